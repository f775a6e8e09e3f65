"""d_k = 256 (two warps per 16-column block), GPU against the CPU oracle.

At d_k = 256 the library sums over the key axis with R = 16 partials (its two
warps each hold 8 row groups); the oracle's canonical order with R = 16 is
the same order, so codes, scales and outputs must agree bit for bit on
free-running trajectories for every family, rounding rule and state width,
and stay within one code step of the literal order.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal, dev, host, sample_heads
from test_gpu_decode import _trajectory

pytestmark = pytest.mark.gpu

GDN = W.WORKLOADS[1]
MAMBA = W.WORKLOADS[3]


def test_reduction_partials_at_256():
    assert rsq.rsq_reduction_partials(256) == 16


@pytest.mark.parametrize("dv", [16, 32, 64, 256])
@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_gdn_dk256_bit_exact(dv, rounding):
    w = dataclasses.replace(GDN, B=3, H=4, dk=256, dv=dv)
    run = Run(w, np.array([8, 4, 4, 8], np.int8), rounding=rounding)
    assert run.R == 16
    _trajectory(run, 3)


@pytest.mark.parametrize("rounding", [rsq.RSQ_BDR, rsq.RSQ_SR_BDR])
def test_gdn_dk256_bdr_bit_exact(rounding):
    w = dataclasses.replace(GDN, B=2, H=3, dk=256, dv=64)
    run = Run(w, np.array([4, 8, 4], np.int8), rounding=rounding)
    _trajectory(run, 4)


@pytest.mark.parametrize("dv", [32, 64])
def test_mamba2_dk256_groups_bit_exact(dv):
    w = dataclasses.replace(MAMBA, B=2, H=6, dk=256, dv=dv, ngroups=3)
    run = Run(w, np.array([8, 4, 8, 4, 4, 8], np.int8))
    _trajectory(run, 3)


@pytest.mark.parametrize("family", ["gla", "kda"])
def test_diagonal_dk256_bit_exact(family):
    w = dataclasses.replace(W.BY_NAME["%s_b64_h16_d128_int8_sr" % family], B=2, H=3, dk=256, dv=64)
    run = Run(w, np.array([8, 4, 8], np.int8))
    _trajectory(run, 3)


@pytest.mark.parametrize("family", ["gdn", "mamba2", "kda"])
def test_fp32_state_dk256_bit_exact(family):
    base = {"gdn": GDN, "mamba2": MAMBA, "kda": W.BY_NAME["kda_b64_h16_d128_int8_sr"]}[family]
    w = dataclasses.replace(base, B=2, H=3, dk=256, dv=64)
    run = Run(w, np.full(3, 32, np.int8))
    _trajectory(run, 3)


def test_dk256_persistent_grid_sampled():
    """More units than resident CTAs, several grid-stride rounds (every stage
    refilled, the exchange barrier through many phases): sampled heads."""
    w = dataclasses.replace(GDN, B=96, H=8, dk=256, dv=128)
    run = Run(w, np.array([8, 4] * 4, np.int8))
    heads = sample_heads(w.B, w.H, 40, seed=3)
    _trajectory(run, 3, heads=heads)


def test_dk256_plain_order_tolerance():
    """Against the literal order: codes within one step (at most 1e-5 of them
    differ), outputs within 1e-3 relative."""
    w = dataclasses.replace(GDN, B=8, H=4, dk=256, dv=128)
    run = Run(w, np.array([8, 8, 8, 8], np.int8))
    nd, nt = _trajectory(run, 4, check_plain=True)
    assert nd <= 1e-5 * nt, (nd, nt)


def test_dk256_in_place_matches_ping_pong():
    w = dataclasses.replace(GDN, B=2, H=4, dk=256, dv=64)
    run = Run(w, np.array([8, 4, 4, 8], np.int8))
    st = run.zero()
    a, b, c = run.upload(st), run.upload(st), run.upload(st)
    for t in range(3):
        inp = run.inputs(t)
        o1 = run.gpu_step(a, b, inp, t)
        o2 = run.gpu_step(c, c, inp, t)
        assert np.array_equal(host(b.codes), host(c.codes)) and np.array_equal(host(b.scales), host(c.scales))
        assert np.array_equal(o1, o2)
        a, b = b, a


def test_dk256_copy_scale_bit_exact():
    w = dataclasses.replace(GDN, B=2, H=3, dk=256, dv=32)
    bits = np.array([4, 8, 4], np.int8)
    q, f = Run(w, bits), Run(w, np.full(3, 32, np.int8))
    sq, sf = q.zero(), f.zero()
    gq, gf = q.upload(sq), f.upload(sf)
    absmax = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
    for t in range(4):
        inp = q.inputs(t)
        ins, keep = q.dev_inputs(inp)
        out_f = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
        out_q = torch.empty_like(out_f)
        f.ctx.decode_step(gf, gf, ins, out_f, t)
        f.ctx.column_absmax(gf, absmax)
        q.ctx.decode_step_copy_scale(gq, gq, ins, absmax, out_q, t)
        torch.cuda.synchronize()
        sf, _ = f.oracle_step(sf, inp, t)
        m = np.abs(sf["f"]).max(axis=2)
        sq, o = oracle.gdn_step(sq, inp, bits, rounding=q.rounding, seed=q.seed, step=t, copy_absmax=m, R=16)
        assert np.array_equal(host(absmax), m)
        assert_state_equal(q.download(gq), sq, bits, what="step %d" % t)
        assert_out_equal(host(out_q), o, what="step %d" % t)


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_dk256_quantize_dequantize_drift(rounding):
    w = dataclasses.replace(GDN, B=2, H=3, dk=256, dv=64)
    bits = np.array([8, 4, 8], np.int8)
    run = Run(w, bits, rounding=rounding)
    f = Run(w, np.full(3, 32, np.int8))
    rng = np.random.default_rng(rounding)
    S = (rng.standard_normal((2, 3, 256, 64)) * rng.uniform(0.01, 5, (2, 3, 1, 64))).astype(np.float32)
    s = run.ctx.alloc_state()
    run.ctx.quantize(dev(S), s, step=9)
    torch.cuda.synchronize()
    ref = oracle.quantize(S, bits, rounding=rounding, seed=run.seed, step=9)
    assert_state_equal(run.download(s), ref, bits, what="quantize")
    D = torch.empty((2, 3, 256, 64), dtype=torch.float32, device="cuda")
    run.ctx.dequantize(s, D)
    torch.cuda.synchronize()
    deq = oracle.dequantize(ref, bits)
    assert np.array_equal(host(D).view(np.uint32), deq.view(np.uint32))
    fs = oracle.zero_state(2, 3, 256, 64)
    fs["f"] = S
    sums = torch.zeros((2, 3, 2), dtype=torch.float64, device="cuda")
    rsq.rsq_state_drift(run.ctx.ctx, s, f.ctx.ctx, f.upload(fs), sums)
    torch.cuda.synchronize()
    e2 = ((deq.astype(np.float64) - S) ** 2).sum(axis=(2, 3))
    assert np.allclose(host(sums)[..., 0], e2, rtol=1e-12)
