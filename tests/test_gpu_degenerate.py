"""Degenerate cases of the method, GPU against the CPU oracle (bit for bit).

* Magnitudes across the whole binary32 range: all-zero columns, column maxima
  in the subnormal range (where r/m overflows and the multiplier saturates),
  tiny, unit, huge and FLT_MAX columns -- quantize, dequantize and a decode step
  that starts from such a state.
* Gate extremes: alpha = 0 (the state is forgotten), alpha = 1 (no decay),
  beta = 0 (no write), beta = 1; zero k, v, q vectors; Mamba-2 with dt = 0
  (decay 1, no input), decay 0, zero x, B, C and D; GLA / KDA with per-channel
  decays of exactly 0 and 1; BDR on steps that leave elements unchanged.
* The largest head count a context takes (RSQ_MAX_HEADS), every head compared.
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

TINY = np.finfo(np.float32).smallest_subnormal
FMAX = np.finfo(np.float32).max
MAXIMA = [0.0, TINY, 2 * TINY, 1e-43, 1e-41, 3e-39, 1e-38, 1e-37, 1e-36, 1e-30, 1.0, 1e30, 3e38]


def _extreme_state(B, H, dk, dv, seed, maxima=MAXIMA, fmax=True):
    """Columns with the given maxima (cycled), random signs and sizes below them."""
    rng = np.random.default_rng(seed)
    S = np.zeros((B, H, dk, dv), np.float32)
    for b in range(B):
        for h in range(H):
            for j in range(dv):
                m = np.float32(maxima[(j + 3 * h + b) % len(maxima)])
                col = (rng.uniform(-1, 1, dk) * np.float64(m)).astype(np.float32)
                col[rng.integers(dk)] = m if rng.random() < 0.5 else -m
                S[b, h, :, j] = col
    if fmax:
        S[0, 0, 1, 2] = FMAX
    return S


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_quantize_dequantize_extreme_magnitudes(rounding):
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=4, dk=32, dv=32)
    bits = np.array([8, 4, 4, 8], np.int8)
    run = Run(w, bits, rounding=rounding)
    S = _extreme_state(2, 4, 32, 32, seed=rounding)
    s = run.ctx.alloc_state()
    run.ctx.quantize(dev(S), s, step=3)
    torch.cuda.synchronize()
    ref = oracle.quantize(S, bits, rounding=rounding, seed=run.seed, step=3)
    assert_state_equal(run.download(s), ref, bits, what="quantize")
    D = torch.empty((2, 4, 32, 32), dtype=torch.float32, device="cuda")
    run.ctx.dequantize(s, D)
    torch.cuda.synchronize()
    assert np.array_equal(host(D).view(np.uint32), oracle.dequantize(ref, bits).view(np.uint32))


def _run_steps(run: Run, st: dict, inputs_at, steps: int, decay_at=None):
    g_in, g_out = run.upload(st), run.upload(st)
    for t in range(steps):
        inp = inputs_at(t)
        decay = None if decay_at is None else decay_at(inp, t)
        out = run.gpu_step(g_in, g_out, inp, t, decay=decay)
        st, o = run.oracle_step(st, inp, t, decay=decay)
        assert_state_equal(run.download(g_out), st, run.head_bits, what="step %d" % t)
        assert_out_equal(out, o, what="step %d" % t)
        g_in, g_out = g_out, g_in
    assert run.ctx.check_flags() == 0
    return st


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8, rsq.RSQ_SR8_BDR])
def test_decode_from_extreme_state(rounding):
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=4, dk=32, dv=32, in_dtype="f32")
    bits = np.array([8, 4, 8, 4], np.int8)
    run = Run(w, bits, rounding=rounding)
    # maxima up to 1 (larger ones would overflow the readout to non-finite values)
    small = [m for m in MAXIMA if m <= 1.0]
    st = oracle.quantize(_extreme_state(2, 4, 32, 32, seed=7, maxima=small, fmax=False), bits,
                         rounding=oracle.RTN, seed=1, step=0)
    scale = np.float32(1e-36)

    def inputs_at(t):
        inp = {k: v.copy() for k, v in run.inputs(t).items()}
        inp["v"] = (inp["v"] * scale).astype(np.float32)   # writes as small as the small columns
        inp["alpha"][:, 0] = 1.0                           # head 0 keeps its (extreme) state
        inp["beta"][:, 0] = 0.0
        return inp
    _run_steps(run, st, inputs_at, 3)


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR8, rsq.RSQ_BDR])
def test_gdn_gate_and_vector_extremes(rounding):
    H = 8
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=H, dk=32, dv=64, in_dtype="f32")
    bits = np.array([8, 4, 8, 4, 8, 4, 8, 4], np.int8)
    run = Run(w, bits, rounding=rounding)
    st = oracle.quantize((np.random.default_rng(2).standard_normal((2, H, 32, 64)) * 0.5).astype(np.float32),
                         bits, rounding=oracle.SR, seed=4, step=0)

    def inputs_at(t):
        inp = {k: v.copy() for k, v in run.inputs(t).items()}
        inp["alpha"][:, 0] = 0.0                     # forget everything: S = beta k v^T
        inp["alpha"][:, 1] = 1.0                     # no decay, no write
        inp["beta"][:, 1] = 0.0
        inp["alpha"][:, 2] = 1.0                     # full-strength delta rule
        inp["beta"][:, 2] = 1.0
        inp["k"][:, 3] = 0.0                         # nothing erased, nothing written
        inp["v"][:, 4] = 0.0                         # erase only
        inp["q"][:, 4] = 0.0                         # zero readout
        inp["alpha"][:, 5] = 0.0                     # forget and write nothing: S = 0
        inp["beta"][:, 5] = 0.0
        inp["v"][:, 6] *= np.float32(1e30)           # huge writes
        return inp
    _run_steps(run, st, inputs_at, 4)


def test_mamba2_extremes():
    H = 6
    w = dataclasses.replace(W.WORKLOADS[3], B=2, H=H, dk=32, dv=32, ngroups=3, in_dtype="f32")
    bits = np.array([8, 4, 8, 4, 8, 4], np.int8)
    run = Run(w, bits)
    st = oracle.quantize((np.random.default_rng(3).standard_normal((2, H, 32, 32))).astype(np.float32),
                         bits, rounding=oracle.SR, seed=5, step=0)

    def inputs_at(t):
        inp = {k: v.copy() for k, v in run.inputs(t).items()}
        inp["dt"][:, 0] = 0.0                        # decay exp(0) = 1 and no input
        inp["x"][:, 1] = 0.0                         # decay only
        inp["Bm"][:, 1] = 0.0                        # group 1 (heads 2, 3): no input direction
        inp["Cm"][:, 2] = 0.0                        # group 2 (heads 4, 5): readout D x only
        inp["D"][3] = 0.0
        return inp

    def decay_at(inp, t):
        d = np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)
        d[:, 5] = 0.0                                # state forgotten
        return d
    _run_steps(run, st, inputs_at, 3, decay_at)


@pytest.mark.parametrize("family", ["gla", "kda"])
def test_diagonal_decay_extremes(family):
    w = dataclasses.replace(W.BY_NAME["%s_b64_h16_d128_int8_sr" % family], B=2, H=4, dk=32, dv=32,
                            in_dtype="f32")
    bits = np.array([8, 4, 4, 8], np.int8)
    run = Run(w, bits)
    st = oracle.quantize((np.random.default_rng(4).standard_normal((2, 4, 32, 32))).astype(np.float32),
                         bits, rounding=oracle.SR, seed=6, step=0)

    def inputs_at(t):
        inp = {k: v.copy() for k, v in run.inputs(t).items()}
        inp["alpha"][:, 0, ::2] = 0.0                # every other key channel forgotten
        inp["alpha"][:, 0, 1::2] = 1.0               # the rest kept as is
        inp["alpha"][:, 1] = 0.0                     # the whole state forgotten
        inp["alpha"][:, 2] = 1.0                     # no decay
        inp["k"][:, 3] = 0.0                         # no write (KDA: no erase either)
        if "beta" in inp:
            inp["beta"][:, 2] = 0.0
        return inp
    _run_steps(run, st, inputs_at, 3)


@pytest.mark.parametrize("family", ["gdn", "mamba2"])
def test_maximum_head_count(family):
    H = rsq.RSQ_MAX_HEADS
    base = W.WORKLOADS[1] if family == "gdn" else W.WORKLOADS[3]
    w = dataclasses.replace(base, B=2, H=H, dk=16, dv=16, ngroups=8 if family == "mamba2" else 1)
    bits = np.random.default_rng(H).choice([4, 8], size=H).astype(np.int8)
    run = Run(w, bits)
    st = oracle.quantize((np.random.default_rng(5).standard_normal((2, H, 16, 16))).astype(np.float32),
                         bits, rounding=oracle.SR, seed=7, step=0)
    s = run.ctx.alloc_state()
    run.ctx.quantize(dev(oracle.dequantize(st, bits)), s, step=0)
    torch.cuda.synchronize()
    assert_state_equal(run.download(s), oracle.quantize(oracle.dequantize(st, bits), bits,
                                                        rounding=run.rounding, seed=run.seed, step=0),
                       bits, what="quantize")

    def decay_at(inp, t):
        return np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)
    _run_steps(run, st, lambda t: run.inputs(t), 2, decay_at if family == "mamba2" else None)
