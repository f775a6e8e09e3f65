"""GPU parity of the copy scale (LoReS (4/4), animation details: the scale
taken from an unquantized copy of the state, which removes the scale-state
feedback described in "When Dynamic Scaling Fails") and of the column-maximum
helper, against the CPU oracle.

The quantized trajectory takes each step's scales from the column maxima of the
FP32 trajectory (same kernel with 32-bit heads, same inputs), read on the GPU
with rsq_column_absmax; the oracle runs the same two trajectories.  Both sides
free-run from S_0 = 0 and must agree bit for bit.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal, dev, host

pytestmark = pytest.mark.gpu


def test_column_absmax_matches_dequantized_maxima():
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=4)
    for bits in (np.array([8, 4, 4, 8], np.int8), np.full(4, 32, np.int8)):
        run = Run(w, bits)
        rng = np.random.default_rng(int(bits[0]))
        S = rng.standard_normal((3, 4, 128, 128)).astype(np.float32)
        st = oracle.quantize(S, bits, rounding=oracle.SR, seed=2, step=0)
        got = torch.empty((3, 4, 128), dtype=torch.float32, device="cuda")
        run.ctx.column_absmax(run.upload(st), got)
        want = np.abs(oracle.dequantize(st, bits)).max(axis=2)
        assert np.array_equal(host(got), want)


@pytest.mark.parametrize("family,rounding,bits", [
    ("gdn", rsq.RSQ_SR, [4, 8, 4, 4]), ("gdn", rsq.RSQ_RTN, [4, 4, 8, 8]),
    ("gdn", rsq.RSQ_SR_BDR, [4, 4, 4, 8]), ("mamba2", rsq.RSQ_SR, [8, 4, 4, 8]),
    ("kda", rsq.RSQ_RTN, [4, 8, 4, 8])])
def test_copy_scale_trajectory_bit_exact(family, rounding, bits):
    base = {"gdn": W.WORKLOADS[1], "mamba2": W.WORKLOADS[3],
            "kda": W.BY_NAME["kda_b64_h16_d128_int8_sr"]}[family]
    w = dataclasses.replace(base, B=3, H=4)
    bits = np.array(bits, np.int8)
    q = Run(w, bits, rounding=rounding)
    f = Run(w, np.full(4, 32, np.int8))
    sq, sf = q.zero(), f.zero()
    gq, gf = q.upload(sq), f.upload(sf)
    absmax = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
    clipped = 0
    for t in range(6):
        inp = q.inputs(t)
        decay = None
        if family == "mamba2":
            decay = np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)
        ins, keep = q.dev_inputs(inp, decay)
        out_f = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
        out_q = torch.empty_like(out_f)
        f.ctx.decode_step(gf, gf, ins, out_f, t)
        f.ctx.column_absmax(gf, absmax)
        q.ctx.decode_step_copy_scale(gq, gq, ins, absmax, out_q, t)
        torch.cuda.synchronize()
        # oracle: the FP32 trajectory, its column maxima, the copy-scale step
        sf, _ = f.oracle_step(sf, inp, t, decay=decay)
        m = np.abs(sf["f"]).max(axis=2)
        if family == "gdn":
            sq_new, o = oracle.gdn_step(sq, inp, bits, rounding=rounding, seed=q.seed, step=t, copy_absmax=m)
        elif family == "kda":
            sq_new, o = oracle.kda_step(sq, inp, bits, rounding=rounding, seed=q.seed, step=t, copy_absmax=m)
        else:
            sq_new, o = oracle.mamba2_step(sq, inp, bits, rounding=rounding, seed=q.seed, step=t,
                                           decay=decay, copy_absmax=m)
        assert np.array_equal(host(absmax), m)
        assert_state_equal(q.download(gq), sq_new, bits, what="step %d" % t)
        assert_out_equal(host(out_q), o, what="step %d" % t)
        r = np.array([oracle.rmax(int(b)) for b in bits])[None, :, None, None]
        clipped += int((np.abs(sq_new["codes"]) == r).sum())
        sq = sq_new
        del keep
    assert clipped > 0


def test_copy_scale_rejects_bad_arguments():
    w = dataclasses.replace(W.WORKLOADS[1], B=1, H=2)
    f = Run(w, np.full(2, 32, np.int8))
    st = f.upload(f.zero())
    ins, keep = f.dev_inputs(f.inputs(0))
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(rsq.RsqError) as e:
        f.ctx.decode_step_copy_scale(st, st, ins, out, out, 0)
    assert e.value.status == rsq.RSQ_E_UNSUPPORTED
    q = Run(w, np.array([8, 4], np.int8))
    sq = q.upload(q.zero())
    with pytest.raises(rsq.RsqError) as e:
        q.ctx.decode_step_copy_scale(sq, sq, ins, None, out, 0)
    assert e.value.status == rsq.RSQ_E_INVAL
