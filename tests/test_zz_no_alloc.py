"""The decode step that allocates nothing, against the context-based entry point.

rsq_decode_step_noalloc exists for callers that cannot allocate device memory
once they run (serving runtimes that reserve nearly all GPU memory for their
own pools at start-up, embedded hosts with a fixed memory budget): instead of
the context's cudaMalloc'd flag word it uses a static device array.  Here it must produce exactly what rsq_decode_step
produces, on two consecutive decode steps, through the C ABI.  This file is
collected last on purpose, so a run that stops at the first failure has already
run every other test.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, dev, host

pytestmark = pytest.mark.gpu


def _copy(s: rsq.State) -> rsq.State:
    return rsq.State(s.codes.clone(), s.scales.clone())


@pytest.mark.parametrize("family", ["gdn", "mamba2", "gdn_dk256"])
def test_noalloc_step_matches_context_step_twice(family):
    if family == "gdn":
        w = dataclasses.replace(W.WORKLOADS[1], B=6, H=8)
        bits = np.array([8, 4, 8, 4, 4, 8, 4, 4], np.int8)
    elif family == "gdn_dk256":
        w = dataclasses.replace(W.WORKLOADS[1], B=3, H=4, dk=256, dv=64)
        bits = np.array([8, 4, 4, 8], np.int8)
    else:
        w = dataclasses.replace(W.WORKLOADS[3], B=3, H=8)
        bits = np.full(8, 8, np.int8)
    run = Run(w, bits)
    # a non-trivial starting state made by the oracle
    rng = np.random.default_rng(17)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    start = oracle.quantize(S, bits, rounding=run.rounding, seed=run.seed, step=0)
    a = run.upload(start)        # context path
    b = _copy(a)                 # no-allocation path
    for t in (1, 2):
        inp = run.inputs(t)
        ins, keep = run.dev_inputs(inp)
        out_a = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
        out_b = torch.empty_like(out_a)
        run.ctx.decode_step(a, a, ins, out_a, t)
        rsq.rsq_decode_step_noalloc(run.family, run.B, run.H, run.dk, run.dv, b, b, ins, out_b, t,
                                    head_bits=bits, rounding=run.rounding, in_dtype=run.in_dtype,
                                    seed=run.seed, ngroups=w.ngroups)
        torch.cuda.synchronize()
        assert np.array_equal(host(a.codes), host(b.codes)), "codes differ at call %d" % t
        assert np.array_equal(host(a.scales).view(np.uint32), host(b.scales).view(np.uint32)), \
            "scales differ at call %d" % t
        assert np.array_equal(host(out_a).view(np.uint32), host(out_b).view(np.uint32)), \
            "outputs differ at call %d" % t
        del keep


def test_noalloc_rejects_bad_config_on_host():
    st = rsq.State(0, 0)
    with pytest.raises(rsq.RsqError) as e:
        rsq.rsq_decode_step_noalloc(rsq.RSQ_GDN, 1, 2, 100, 128, st, st, rsq.gdn_inputs(0, 0, 0, 0, 0),
                                    0, 0)
    assert e.value.status == rsq.RSQ_E_UNSUPPORTED
