"""The context allocator hook (rsq_config.alloc / release).

A failing hook makes rsq_create return RSQ_E_NOMEM with nothing left
allocated; a hook over PyTorch's caching allocator gives a context that
decodes exactly like one on cudaMalloc, and rsq_destroy hands the word back
once.  The out-of-memory case is simulated on the host: no device allocation
is made to fail.
"""
import dataclasses

import numpy as np
import pytest
import torch

import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal

pytestmark = pytest.mark.gpu


def _ctx(allocator):
    return rsq.Context(rsq.RSQ_GDN, 2, 3, 32, 32, head_bits=[8, 4, 8], rounding=rsq.RSQ_SR, seed=5,
                       allocator=allocator)


def test_failing_hook_reports_out_of_memory():
    released = []
    with pytest.raises(rsq.RsqError) as e:
        _ctx((lambda n: None, released.append))
    assert e.value.status == rsq.RSQ_E_NOMEM
    assert released == []


def test_misaligned_hook_memory_is_refused_and_released():
    base = torch.cuda.caching_allocator_alloc(64)
    released = []
    try:
        with pytest.raises(rsq.RsqError) as e:
            _ctx((lambda n: base + 4, released.append))
        assert e.value.status == rsq.RSQ_E_NOMEM
        assert released == [base + 4]
    finally:
        torch.cuda.caching_allocator_delete(base)


def test_torch_pool_hook_decodes_like_cudamalloc():
    calls = {"alloc": [], "release": []}

    def alloc(n):
        p = torch.cuda.caching_allocator_alloc(n)
        calls["alloc"].append((n, p))
        return p

    def release(p):
        calls["release"].append(p)
        torch.cuda.caching_allocator_delete(p)

    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3, dk=32, dv=32)
    bits = np.array([8, 4, 8], np.int8)
    run = Run(w, bits)
    hooked = rsq.Context(rsq.RSQ_GDN, 2, 3, 32, 32, head_bits=bits, rounding=run.rounding,
                         in_dtype=run.in_dtype, seed=run.seed, allocator=(alloc, release))
    assert len(calls["alloc"]) == 1 and calls["alloc"][0][0] == 4
    st = run.zero()
    a_in, a_out, b_in, b_out = (run.upload(st) for _ in range(4))
    for t in range(3):
        inp = run.inputs(t)
        ins, keep = run.dev_inputs(inp)
        oa = torch.empty((2, 3, 32), dtype=torch.float32, device="cuda")
        ob = torch.empty_like(oa)
        run.ctx.decode_step(a_in, a_out, ins, oa, t)
        hooked.decode_step(b_in, b_out, ins, ob, t)
        torch.cuda.synchronize()
        assert_state_equal(run.download(b_out), run.download(a_out), bits, what="step %d" % t)
        assert_out_equal(ob.cpu().numpy(), oa.cpu().numpy(), what="step %d" % t)
        a_in, a_out, b_in, b_out = a_out, a_in, b_out, b_in
    assert hooked.check_flags() == 0
    hooked.close()
    assert calls["release"] == [calls["alloc"][0][1]]
