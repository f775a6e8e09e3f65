"""The C-ABI library: loads, exports what include/rsq.h declares, validates on the
host.  No compute call here needs a GPU."""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import ssm_decode_02_b200 as rsq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "rsq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rsq_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert "rsq_decode_step" in names and len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", rsq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (rsq_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(rsq.lib, n)


def test_library_is_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", rsq.LIB_PATH], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    arches = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert arches == {"100a"}, arches


def _create(**kw):
    base = dict(family=rsq.RSQ_GDN, batch=2, heads=4, dk=128, dv=128, head_bits=None,
                rounding=rsq.RSQ_SR, in_dtype=rsq.RSQ_BF16, seed=1, ngroups=1)
    base.update(kw)
    f = base.pop("family")
    return rsq.rsq_create(f, base.pop("batch"), base.pop("heads"), base.pop("dk"), base.pop("dv"), **base)


@pytest.mark.parametrize("kw,status", [
    (dict(family=7), rsq.RSQ_E_INVAL),
    (dict(batch=0), rsq.RSQ_E_INVAL),
    (dict(heads=0), rsq.RSQ_E_INVAL),
    (dict(heads=rsq.RSQ_MAX_HEADS + 1), rsq.RSQ_E_INVAL),
    (dict(dk=100), rsq.RSQ_E_UNSUPPORTED),
    (dict(dk=512), rsq.RSQ_E_UNSUPPORTED),
    (dict(dk=256, window=8), rsq.RSQ_E_UNSUPPORTED),
    (dict(dk=256, key_axis=1), rsq.RSQ_E_UNSUPPORTED),
    (dict(dv=8), rsq.RSQ_E_UNSUPPORTED),
    (dict(rounding=4), rsq.RSQ_E_INVAL),
    (dict(rounding=6), rsq.RSQ_E_INVAL),
    (dict(rounding=-1), rsq.RSQ_E_INVAL),
    (dict(in_dtype=9), rsq.RSQ_E_INVAL),
    (dict(head_bits=[8, 4, 2, 8]), rsq.RSQ_E_INVAL),
    (dict(head_bits=[8, 32, 32, 32]), rsq.RSQ_E_UNSUPPORTED),
    (dict(family=rsq.RSQ_MAMBA2, ngroups=3), rsq.RSQ_E_INVAL),
    (dict(window=3), rsq.RSQ_E_INVAL),
    (dict(window=8, family=rsq.RSQ_MAMBA2), rsq.RSQ_E_UNSUPPORTED),
    (dict(window=8, rounding=rsq.RSQ_BDR), rsq.RSQ_E_UNSUPPORTED),
    (dict(key_axis=2), rsq.RSQ_E_INVAL),
    (dict(key_axis=1, family=rsq.RSQ_KDA), rsq.RSQ_E_UNSUPPORTED),
    (dict(key_axis=1, window=4), rsq.RSQ_E_UNSUPPORTED),
    (dict(key_axis=1, head_bits=[32, 32, 32, 32]), rsq.RSQ_E_UNSUPPORTED),
    (dict(alloc=rsq.rsq_alloc_fn(lambda n, u: None)), rsq.RSQ_E_INVAL),      # hook without release
    (dict(release=rsq.rsq_release_fn(lambda p, u: None)), rsq.RSQ_E_INVAL),  # release without hook
])
def test_create_rejects_bad_configs_on_host(kw, status):
    with pytest.raises(rsq.RsqError) as e:
        _create(**kw)
    assert e.value.status == status
    assert rsq.lib.rsq_last_error().decode()


def test_null_arguments_rejected():
    assert rsq.lib.rsq_create(None, None) == rsq.RSQ_E_INVAL
    assert rsq.lib.rsq_decode_step(None, None, None, None, None, 0, None) == rsq.RSQ_E_INVAL
    assert rsq.lib.rsq_quantize(None, None, None, 0, None) == rsq.RSQ_E_INVAL
    assert rsq.lib.rsq_dequantize(None, None, None, None) == rsq.RSQ_E_INVAL
    assert rsq.lib.rsq_check_flags(None, None, None) == rsq.RSQ_E_INVAL
    rsq.lib.rsq_destroy(None)


def test_reduction_partials():
    assert [rsq.rsq_reduction_partials(d) for d in (16, 32, 64, 128, 256)] == [8, 8, 8, 8, 16]


def test_allocate_bits_matches_oracle_brute_force():
    """Decay-based mixed precision (host logic) against the oracle's brute force."""
    rng = np.random.default_rng(3)
    for H in (1, 4, 32, 80, 512):
        score = rng.uniform(0.5, 1.0, H)
        if H > 3:
            score[1] = score[2]  # tie
        for n_hi in (0, H // 4, H):
            got = rsq.rsq_allocate_bits(score, n_hi)
            want = oracle.allocate_bits(score, n_hi)
            assert np.array_equal(got, want)


def test_allocate_bits_validation():
    with pytest.raises(rsq.RsqError):
        rsq.rsq_allocate_bits(np.ones(4), 5)
    with pytest.raises(rsq.RsqError):
        rsq.rsq_allocate_bits(np.ones(4), 1, high_bits=16)


def test_binding_refuses_host_tensors_for_device_arguments():
    """A CPU or non-contiguous tensor passed where the ABI expects device memory
    is refused by the binding before any call reaches the library."""
    import torch
    with pytest.raises(ValueError):
        rsq.gdn_inputs(torch.zeros(4), 0, 0, 0, 0)
    with pytest.raises(ValueError):
        rsq._state(rsq.State(torch.zeros(8, dtype=torch.uint8), 0))
    with pytest.raises(TypeError):
        rsq.gdn_inputs(object(), 0, 0, 0, 0)
    assert rsq.gdn_inputs(0, 0, 0, 0, 0).q is None


def test_binding_structs_match_the_c_header_layout(tmp_path):
    """Every ctypes struct of the binding has the size and field offsets that a C
    compiler gives the declarations in include/rsq.h."""
    import ctypes
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {"rsq_config": rsq.rsq_config, "rsq_state": rsq.rsq_state, "rsq_gdn_inputs": rsq.rsq_gdn_inputs,
               "rsq_mamba2_inputs": rsq.rsq_mamba2_inputs, "rsq_diag_inputs": rsq.rsq_diag_inputs,
               "rsq_window": rsq.rsq_window}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "rsq.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append('printf("%s %%zu\\n", sizeof(%s));' % (name, name))
        for f in cls._fields_:
            lines.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (name, f[0], name, f[0]))
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c11", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                 check=True).stdout.splitlines())
    for name, cls in structs.items():
        assert int(got[name]) == ctypes.sizeof(cls), name
        for f in cls._fields_:
            assert int(got["%s.%s" % (name, f[0])]) == getattr(cls, f[0]).offset, (name, f[0])
