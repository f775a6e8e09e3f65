"""GPU parity of Bounded Directional Rounding ("Preserving Updates in Low-Bit
Recurrent State Quantization", abstract) against the CPU oracle.

The CUDA decode step with RSQ_BDR (nearest base rounding) and RSQ_SR_BDR
(stochastic base rounding) must match the oracle's canonical order bit for bit
on free-running trajectories that start from a non-trivial quantized state (so
reversals occur from the first step), and the directional correction must
actually change codes relative to the base rule.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, bits_for, sample_heads
from test_gpu_decode import _trajectory

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def _start(run: Run, seed: int) -> dict:
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    return oracle.quantize(S, run.head_bits, rounding=run.rounding, seed=run.seed, step=0)


@pytest.mark.parametrize("rounding", [rsq.RSQ_BDR, rsq.RSQ_SR_BDR, rsq.RSQ_SR8_BDR])
@pytest.mark.parametrize("family,dk,dv", [("gdn", 128, 128), ("gdn", 32, 16), ("gdn", 64, 256),
                                          ("mamba2", 128, 64), ("mamba2", 16, 32)])
def test_bdr_bit_exact(rounding, family, dk, dv):
    base = WL[1] if family == "gdn" else WL[3]
    w = dataclasses.replace(base, B=3, H=4, dk=dk, dv=dv)
    run = Run(w, np.array([8, 4, 4, 8], np.int8), rounding=rounding)
    _trajectory(run, 4, init=_start(run, dk + dv))


def test_bdr_full_size_sampled_heads():
    """The INT4 long-horizon shape at full batch in the benchmark's launch
    configuration, with the directional rule; sampled heads."""
    w = WL[4]
    run = Run(w, bits_for(w), rounding=rsq.RSQ_SR_BDR)
    heads = sample_heads(run.B, run.H, 48, seed=4)
    _trajectory(run, 3, heads=heads)


@pytest.mark.parametrize("base,bdr", [(rsq.RSQ_RTN, rsq.RSQ_BDR), (rsq.RSQ_SR, rsq.RSQ_SR_BDR), (rsq.RSQ_SR8, rsq.RSQ_SR8_BDR)])
def test_bdr_changes_codes_only_by_one_step(base, bdr):
    """One step from the same state: the rule keeps the scales, moves codes by at
    most one step, and does move some (reversals are common at 4 bits)."""
    w = dataclasses.replace(WL[1], B=4, H=4)
    bits = np.full(4, 4, np.int8)
    rb = Run(w, bits, rounding=base)
    rd = Run(w, bits, rounding=bdr)
    st = _start(rb, 3)
    inp = rb.inputs(0)
    outs = []
    for r in (rb, rd):
        g_in, g_out = r.upload(st), r.upload(st)
        r.gpu_step(g_in, g_out, inp, 0)
        outs.append(r.download(g_out))
    a, b = outs
    assert np.array_equal(a["scales"].view(np.uint32), b["scales"].view(np.uint32))
    d = np.abs(a["codes"].astype(int) - b["codes"].astype(int))
    assert d.max() == 1 and d.sum() > 0
