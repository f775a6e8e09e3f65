"""Failure detection on the GPU without a fault: a bounded barrier wait runs out.

With the test hook rsq_debug_waits, the second warp of every two-warp block
(d_k = 256) withholds its arrivals on the block's exchange barrier and the
waits are limited to 1024 polls, so both warps' waits run out.  The kernel
must end by itself, report the timeout through rsq_check_flags (RSQ_E_CUDA),
and leave the context usable: with the hook cleared the next step is
bit-exact against the oracle again.  Every wait is bounded, so no step can
hang; the stage copies of a CTA that stops early are waited for (bounded)
before it ends.
"""
import dataclasses
import time

import numpy as np
import pytest
import torch

import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal

pytestmark = pytest.mark.gpu


def test_exchange_wait_runs_out_and_is_reported():
    w = dataclasses.replace(W.BY_NAME["gdn_b64_h8_d256_int8_sr"], B=2, H=2, dv=64)   # d_k = 256
    assert w.dk == 256
    run = Run(w, np.array([8, 4], np.int8))
    st = run.zero()
    inp = run.inputs(0)
    g_in, g_out = run.upload(st), run.upload(st)
    rsq.rsq_debug_waits(run.ctx.ctx, 1024, 1)
    t0 = time.perf_counter()
    run.gpu_step(g_in, g_out, inp, 0)            # synchronizes: the kernel ended by itself
    elapsed = time.perf_counter() - t0
    print("step with the withheld arrival took %.3f s" % elapsed)
    assert elapsed < 60.0
    with pytest.raises(rsq.RsqError) as e:
        run.ctx.check_flags()
    assert e.value.status == rsq.RSQ_E_CUDA and "timed out" in str(e.value)
    # the flag is cleared by the check and the context still works
    rsq.rsq_debug_waits(run.ctx.ctx, 0, 0)
    assert run.ctx.check_flags() == 0
    g_in, g_out = run.upload(st), run.upload(st)
    out = run.gpu_step(g_in, g_out, inp, 0)
    ref, ref_out = run.oracle_step(st, inp, 0)
    assert_state_equal(run.download(g_out), ref, run.head_bits)
    assert_out_equal(out, ref_out)
    assert run.ctx.check_flags() == 0


def test_debug_waits_argument_checks():
    w = dataclasses.replace(W.WORKLOADS[1], B=1, H=2)
    run = Run(w, np.array([8, 8], np.int8))
    with pytest.raises(rsq.RsqError) as e:
        rsq.rsq_debug_waits(run.ctx.ctx, 10, 2)
    assert e.value.status == rsq.RSQ_E_INVAL
