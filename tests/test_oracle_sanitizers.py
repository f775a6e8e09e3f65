"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

Every oracle entry point runs on small inputs in a subprocess that loads the
sanitizer build of the same C source; any out-of-bounds access, leak of a
heap block's bounds or undefined behaviour aborts the subprocess.  CPU only.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import dataclasses
import os
import numpy as np
import oracle
import workloads as W

assert oracle.lib()._name == os.environ["RSQ_ORACLE_LIB"]

tiny = W.WORKLOADS[0]
hb = np.array([8, 4], np.int8)
for mode in (oracle.PLAIN, oracle.CANONICAL):
    for rnd in (oracle.RTN, oracle.SR, oracle.BDR, oracle.SR_BDR):
        st = oracle.zero_state(1, 2, 16, 16)
        for t in range(3):
            st, _ = oracle.gdn_step(st, W.gdn_inputs(tiny, t), hb, rounding=rnd, seed=1, step=t, mode=mode)
m = dataclasses.replace(W.WORKLOADS[3], B=1, H=2, dk=16, dv=16, in_dtype="f32")
st = oracle.zero_state(1, 2, 16, 16)
for t in range(2):
    st, _ = oracle.mamba2_step(st, W.inputs(m, t), hb, rounding=oracle.SR, seed=1, step=t)
for name in ("gla_b64_h16_d128_int8_sr", "kda_b64_h16_d128_int8_sr"):
    w = dataclasses.replace(W.BY_NAME[name], B=1, H=2, dk=16, dv=16, in_dtype="f32")
    step = oracle.gla_step if w.family == "gla" else oracle.kda_step
    st = oracle.zero_state(1, 2, 16, 16)
    for t in range(2):
        st, _ = step(st, W.inputs(w, t), hb, rounding=oracle.SR, seed=1, step=t)
st, win = oracle.zero_state(1, 2, 16, 16), oracle.zero_window(1, 2, 4, 16, 16)
for t in range(6):
    st, win, _ = oracle.gdn_pw_step(st, win, W.gdn_inputs(tiny, t), hb, rounding=oracle.SR, seed=1, step=t)
ka = oracle.zero_state_ka(1, 2, 16, 16)
for t in range(2):
    ka, _ = oracle.gdn_ka_step(ka, W.gdn_inputs(tiny, t), hb, rounding=oracle.SR, seed=1, step=t)
S = np.random.default_rng(0).standard_normal((1, 2, 16, 16)).astype(np.float32)
q = oracle.quantize(S, hb, rounding=oracle.SR, seed=1, step=0, copy_absmax=np.abs(S).max(axis=2) * 0.5)
oracle.dequantize(q, hb)
oracle.unpack_state(oracle.pack_state(q, hb), q["scales"], hb, 1, 2, 16, 16)
oracle.quantize_ka(S, hb, rounding=oracle.RTN, seed=0, step=0)
# columns whose maxima span the float range, down to scales that underflow to zero
E = np.zeros((1, 1, 16, 16), np.float32)
for j, m in enumerate([0.0, 1e-45, 1e-43, 1e-41, 3e-39, 1e-37, 1e-30, 1.0, 1e30, 3.4e38]):
    E[0, 0, :, j] = np.linspace(-m, m, 16, dtype=np.float64).astype(np.float32)
E[0, 0, 5, 10] = np.float32(3.4028235e38)
for mode in (oracle.PLAIN, oracle.CANONICAL):
    for rnd in (oracle.RTN, oracle.SR):
        for b in (8, 4):
            oracle.quantize(E, np.array([b], np.int8), rounding=rnd, seed=1, step=0, mode=mode)
    oracle.quantize_ka(E, np.array([4], np.int8), rounding=oracle.SR, seed=1, step=0, mode=mode)
    tinyst = oracle.quantize(E, np.array([8], np.int8), rounding=oracle.RTN, seed=1, step=0)
    oracle.gdn_step(tinyst, W.gdn_inputs(dataclasses.replace(tiny, B=1, H=1), 0), np.array([8], np.int8),
                    rounding=oracle.SR_BDR, seed=1, step=0, mode=mode)
[oracle.e4m3_decode(c) for c in range(256)]
[oracle.e4m3_encode(x) for x in (0.0, 1e-9, 0.3, 448.0, 1e6, -3.0)]
oracle.allocate_bits(np.arange(8, dtype=np.float64), 2)
print("sanitized oracle ok")
"""


def test_oracle_under_address_and_undefined_behaviour_sanitizers():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    asan = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    if not asan or not os.path.exists(asan):
        pytest.skip("libasan not available")
    sys.path.insert(0, ROOT)
    from oracle import build as ob
    lib = ob.build_sanitized()
    env = dict(os.environ, RSQ_ORACLE_LIB=lib, LD_PRELOAD=asan,
               ASAN_OPTIONS="detect_leaks=0:abort_on_error=1", UBSAN_OPTIONS="print_stacktrace=1",
               PYTHONPATH=ROOT)
    res = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-4000:]
    assert "sanitized oracle ok" in res.stdout
    assert "runtime error" not in res.stderr
