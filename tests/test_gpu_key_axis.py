"""GPU parity of key-axis scale groups (LoReS "(1/4) Scale grouping": one scale
per key row, the grouping ablation) against the CPU oracle.

The key-axis decode kernel (persistent CTAs, one head at a time through a
two-stage ring of bulk copies) and its quantize / dequantize paths must match
the oracle bit for bit on free-running trajectories.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import assert_out_equal, dev, host, sample_heads

pytestmark = pytest.mark.gpu


class KaRun:
    def __init__(self, w, bits, rounding):
        self.w, self.bits, self.rounding = w, np.asarray(bits, np.int8), rounding
        self.B, self.H, self.dk, self.dv = w.B, w.H, w.dk, w.dv
        self.in_dtype = rsq.RSQ_BF16 if w.in_dtype == "bf16" else rsq.RSQ_F32
        self.ctx = rsq.Context(rsq.RSQ_GDN, self.B, self.H, self.dk, self.dv, head_bits=self.bits,
                               rounding=rounding, in_dtype=self.in_dtype, seed=w.sr_seed, key_axis=1)

    def upload(self, st):
        return rsq.State(dev(oracle.pack_state(st, self.bits)), dev(st["scales"]))

    def download(self, s, heads=None):
        dummy = np.zeros((self.B, self.H, self.dv), np.float32)
        st = oracle.unpack_state(host(s.codes), dummy, self.bits, self.B, self.H, self.dk, self.dv,
                                 heads=heads)
        return {"codes": st["codes"], "scales": host(s.scales)}

    def inputs(self, t):
        return W.gdn_inputs(self.w, t)


def _assert_ka_equal(g, o, heads, what):
    for b, h in heads:
        assert np.array_equal(g["codes"][b, h], o["codes"][b, h]), "%s codes (%d,%d)" % (what, b, h)
        assert np.array_equal(g["scales"][b, h].view(np.uint32), o["scales"][b, h].view(np.uint32)), \
            "%s scales (%d,%d)" % (what, b, h)


def _trajectory(run: KaRun, steps, heads=None, seed=5):
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    st = oracle.quantize_ka(S, run.bits, rounding=run.rounding, seed=run.w.sr_seed, step=0)
    g = run.upload(st)
    sel = heads if heads is not None else [(b, h) for b in range(run.B) for h in range(run.H)]
    for t in range(steps):
        inp = run.inputs(t)
        keep = {k: dev(v) for k, v in inp.items()}
        ins = rsq.gdn_inputs(keep["q"], keep["k"], keep["v"], keep["alpha"], keep["beta"])
        out = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
        run.ctx.decode_step(g, g, ins, out, t)
        torch.cuda.synchronize()
        st, o = oracle.gdn_ka_step(st, inp, run.bits, rounding=run.rounding, seed=run.w.sr_seed, step=t,
                                   heads=heads)
        _assert_ka_equal(run.download(g, heads=heads), st, sel, "step %d" % t)
        assert_out_equal(host(out), o, heads=heads, what="step %d" % t)


@pytest.mark.parametrize("dk,dv", [(128, 128), (16, 16), (32, 64), (64, 256), (128, 32)])
@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_key_axis_decode_bit_exact(dk, dv, rounding):
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=4, dk=dk, dv=dv)
    _trajectory(KaRun(w, [8, 4, 4, 8], rounding), 4, seed=dk + dv)


def test_key_axis_f32_inputs():
    w = dataclasses.replace(W.WORKLOADS[0], B=2, H=3)
    _trajectory(KaRun(w, [8, 8, 4], rsq.RSQ_SR), 6)


def test_key_axis_full_size_sampled_heads():
    w = W.WORKLOADS[1]
    run = KaRun(w, np.full(w.H, 8, np.int8), rsq.RSQ_SR)
    _trajectory(run, 2, heads=sample_heads(w.B, w.H, 32, seed=7))


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_key_axis_quantize_dequantize_and_maxima(rounding):
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3, dk=64, dv=128)
    run = KaRun(w, [8, 4, 8], rounding)
    rng = np.random.default_rng(3)
    S = rng.standard_normal((2, 3, 64, 128)).astype(np.float32)
    g = run.ctx.alloc_state()
    run.ctx.quantize(dev(S), g, step=4)
    want = oracle.quantize_ka(S, run.bits, rounding=rounding, seed=w.sr_seed, step=4)
    _assert_ka_equal(run.download(g), want, [(b, h) for b in range(2) for h in range(3)], "quantize")
    D = torch.empty((2, 3, 64, 128), dtype=torch.float32, device="cuda")
    run.ctx.dequantize(g, D)
    assert np.array_equal(host(D), oracle.dequantize_ka(want))
    m = torch.empty((2, 3, 128), dtype=torch.float32, device="cuda")
    run.ctx.column_absmax(g, m)
    assert np.array_equal(host(m), np.abs(oracle.dequantize_ka(want)).max(axis=2))


def test_key_axis_several_heads_per_cta_all_heads():
    """More heads than resident CTAs (d_v = 256: 512-thread CTAs), so every
    persistent CTA takes several heads through its two-stage ring; every head
    compared, mixed widths."""
    w = dataclasses.replace(W.WORKLOADS[1], B=40, H=8, dk=64, dv=256)
    _trajectory(KaRun(w, [8, 4, 4, 8, 8, 4, 8, 4], rsq.RSQ_SR8), 3, seed=11)


def test_key_axis_stage_wait_runs_out_and_is_reported():
    """Failure detection without a fault: with the test hook the first stage of
    every CTA's ring is never filled, so its bounded wait runs out while the
    second stage's copies are in flight.  The kernel must wait for those
    copies, end by itself, report the timeout, and leave the context usable."""
    import time
    w = dataclasses.replace(W.WORKLOADS[1], B=40, H=8, dk=64, dv=256)
    bits = [8, 4, 4, 8, 8, 4, 8, 4]
    run = KaRun(w, bits, rsq.RSQ_SR8)
    rng = np.random.default_rng(2)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    st = oracle.quantize_ka(S, run.bits, rounding=run.rounding, seed=w.sr_seed, step=0)
    inp = run.inputs(0)
    keep = {k: dev(v) for k, v in inp.items()}
    ins = rsq.gdn_inputs(keep["q"], keep["k"], keep["v"], keep["alpha"], keep["beta"])
    out = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
    g = run.upload(st)
    rsq.rsq_debug_waits(run.ctx.ctx, 1024, 1)
    t0 = time.perf_counter()
    run.ctx.decode_step(g, g, ins, out, 0)
    torch.cuda.synchronize()                     # the kernel ended by itself
    assert time.perf_counter() - t0 < 60.0
    with pytest.raises(rsq.RsqError) as e:
        run.ctx.check_flags()
    assert e.value.status == rsq.RSQ_E_CUDA and "timed out" in str(e.value)
    # hook cleared: the same context computes the step bit-exactly again
    rsq.rsq_debug_waits(run.ctx.ctx, 0, 0)
    assert run.ctx.check_flags() == 0            # the flag was cleared by the read above
    g = run.upload(st)
    run.ctx.decode_step(g, g, ins, out, 0)
    torch.cuda.synchronize()
    want, o = oracle.gdn_ka_step(st, inp, run.bits, rounding=run.rounding, seed=w.sr_seed, step=0)
    allh = [(b, h) for b in range(run.B) for h in range(run.H)]
    _assert_ka_equal(run.download(g), want, allh, "after the timeout")
    assert_out_equal(host(out), o, what="after the timeout")
    assert run.ctx.check_flags() == 0


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("rounding", [rsq.RSQ_SR8, rsq.RSQ_RTN])
def test_key_axis_against_the_literal_order(bits, rounding):
    """Key-axis groups against the oracle's literal order at the method's
    tolerance ("(1/4) Scale grouping": s_i = max_j |S_ij| / r, codes
    round(S / s); "(3/4) Rounding").  Teacher-forced on the benchmark head
    shape: each step starts the GPU and the literal order from the canonical
    oracle's state, which the GPU matches bit for bit.  At most 1e-5 of the
    codes differ, each by one step, apart from nearest-rounding boundary cases
    (held to 1e-3); scales agree to 1e-5 relative; outputs and the
    dequantized state of the agreeing codes to 1e-3 normwise relative.  Row
    groups are compared through the transpose, so a group's maximum is the
    column maximum the boundary accounting expects."""
    import plain_order
    w = dataclasses.replace(W.WORKLOADS[1], B=8)
    hb = np.full(w.H, bits, np.int8)
    run = KaRun(w, hb, rounding)
    rng = np.random.default_rng(21 + bits)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    orc_rnd = oracle.SR8 if rounding == rsq.RSQ_SR8 else oracle.RTN
    st = oracle.quantize_ka(S, hb, rounding=orc_rnd, seed=w.sr_seed, step=0)
    b32 = np.full(w.H, 32, np.int8)
    n_other = n_tie = n_tot = 0
    for t in range(4):
        inp = run.inputs(t)
        keep = {k: dev(v) for k, v in inp.items()}
        ins = rsq.gdn_inputs(keep["q"], keep["k"], keep["v"], keep["alpha"], keep["beta"])
        out = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
        g = run.upload(st)
        run.ctx.decode_step(g, g, ins, out, t)
        torch.cuda.synchronize()
        gpu = run.download(g)
        canon, canon_out = oracle.gdn_ka_step(st, inp, hb, rounding=orc_rnd, seed=w.sr_seed, step=t)
        allh = [(b, h) for b in range(run.B) for h in range(run.H)]
        _assert_ka_equal(gpu, canon, allh, "step %d" % t)
        assert_out_equal(host(out), canon_out, what="step %d" % t)
        plain, plain_out = oracle.gdn_ka_step(st, inp, hb, rounding=orc_rnd, seed=w.sr_seed, step=t,
                                              mode=oracle.PLAIN)
        # the literal order's full-precision S_t: the 32-bit plain step of the dequantized state
        f = oracle.zero_state(run.B, run.H, run.dk, run.dv, fp32=True)
        f["f"] = oracle.dequantize_ka(st)
        lit, _ = oracle.gdn_step(f, inp, b32, rounding=oracle.RTN, seed=0, step=0, mode=oracle.PLAIN)
        T = lambda x: np.ascontiguousarray(np.swapaxes(x, 2, 3))
        o, ti, tot = plain_order.compare_codes(T(gpu["codes"]), T(plain["codes"]), T(lit["f"]), hb,
                                               nearest=rounding == rsq.RSQ_RTN)
        n_other, n_tie, n_tot = n_other + o, n_tie + ti, n_tot + tot
        assert np.allclose(gpu["scales"], plain["scales"], rtol=1e-5, atol=0)
        assert plain_order.max_rel(host(out), plain_out) <= 1e-3
        same = gpu["codes"] == plain["codes"]
        dg = np.where(same, oracle.dequantize_ka(gpu), 0.0)
        dp = np.where(same, oracle.dequantize_ka(plain), 0.0)
        rows = np.abs(oracle.dequantize_ka(plain)).max(axis=3, keepdims=True)
        rows[rows == 0] = 1.0
        assert np.max(np.abs(dg - dp) / rows) <= 1e-3
        st = canon
    assert n_tot > 0
    assert n_other <= 1e-5 * n_tot, (n_other, n_tie, n_tot)
    assert n_tie <= 1e-3 * n_tot, (n_other, n_tie, n_tot)
