"""GPU parity: the CUDA decode step (through the C ABI) against the CPU oracle.

Bit-exact against the oracle's canonical order (codes, scales, outputs, FP32
states); against the literal order within the method's tolerance (at most 1e-5
of codes differ, by at most one step; outputs within 1e-3 relative).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import (Run, assert_out_equal, assert_state_equal, bits_for, dev, host,
                         sample_heads)

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def _mamba_decay(inp):
    return np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)


def _trajectory(run: Run, steps: int, heads=None, decay_override=True, check_plain=False,
                init=None):
    """Run `steps` decode steps on the GPU and, independently, on the oracle (only
    the listed heads when given; heads are independent).  Both start from the same
    oracle-made state and free-run; every step must agree bit for bit.  With
    check_plain, the literal-order oracle is also stepped from the oracle's state
    and the GPU's codes must stay within one step of it."""
    st = run.zero() if init is None else init
    g_in, g_out = run.upload(st), run.upload(st)
    plain_diff = plain_tot = 0
    for t in range(steps):
        inp = run.inputs(t)
        decay = _mamba_decay(inp) if (run.family == rsq.RSQ_MAMBA2 and decay_override) else None
        out = run.gpu_step(g_in, g_out, inp, t, decay=decay)
        gpu_st = run.download(g_out, heads=heads)
        ref, ref_out = run.oracle_step(st, inp, t, decay=decay, heads=heads)
        assert_state_equal(gpu_st, ref, run.head_bits, heads=heads, what="step %d" % t)
        assert_out_equal(out, ref_out, heads=heads, what="step %d" % t)
        if check_plain:
            pl, pl_out = run.oracle_step(st, inp, t, mode=oracle.PLAIN, decay=decay, heads=heads)
            sel = heads if heads is not None else [(b, h) for b in range(run.B) for h in range(run.H)]
            for b, h in sel:
                d = np.abs(gpu_st["codes"][b, h].astype(int) - pl["codes"][b, h].astype(int))
                assert d.max() <= 1
                plain_diff += int((d != 0).sum())
                plain_tot += d.size
                ref_n = np.max(np.abs(pl_out[b, h])) + 1e-30
                assert np.max(np.abs(out[b, h] - pl_out[b, h])) <= 1e-3 * ref_n
        st = ref
        g_in, g_out = g_out, g_in
    if check_plain:
        return plain_diff, plain_tot
    return None


# ---------------------------------------------------------------------------
# The five evaluation workloads
# ---------------------------------------------------------------------------
def test_gdn_tiny_full_trajectory_bit_exact():
    """GDN B=1 H=2 d=16, INT8 RTN, 64 steps: free-running trajectory, bit-exact."""
    w = WL[0]
    run = Run(w, bits_for(w))
    _trajectory(run, w.steps)


def test_gdn_int8_sr_bit_exact_and_plain_tolerance():
    """GDN d=128 INT8 SR (bf16 inputs), reduced batch: free-running bit-exact, and the
    literal evaluation order within the 1e-5 code tolerance."""
    w = WL[1]
    run = Run(w, bits_for(w), B=8)
    nd, nt = _trajectory(run, 8, check_plain=True)
    assert nd <= 1e-5 * nt, (nd, nt)


def test_gdn_mixed_precision_bit_exact():
    """Decay-based mixed precision: 25% INT8 heads (highest mean alpha) + INT4 rest, SR."""
    w = WL[2]
    bits = bits_for(w)
    assert (bits == 8).sum() == w.H // 4 and (bits == 4).sum() == w.H - w.H // 4
    run = Run(w, bits, B=4)
    _trajectory(run, 5)


def test_mamba2_int8_sr_bit_exact_with_decay():
    w = WL[3]
    run = Run(w, bits_for(w), B=2)
    _trajectory(run, 5)


def test_mamba2_device_expf_within_tolerance():
    """With the decay computed on the device (expf) instead of passed in, codes may
    differ from the host libm result in at most 1e-5 of places by one step.  Each
    step starts the GPU from the oracle's state."""
    w = WL[3]
    run = Run(w, bits_for(w), B=4)
    st = run.zero()
    n_diff = n_tot = 0
    for t in range(4):
        inp = run.inputs(t)
        g_in, g_out = run.upload(st), run.upload(st)
        out = run.gpu_step(g_in, g_out, inp, t)
        gpu = run.download(g_out)
        ref, ref_out = run.oracle_step(st, inp, t)
        d = np.abs(gpu["codes"].astype(int) - ref["codes"].astype(int))
        assert d.max() <= 1
        n_diff += int((d != 0).sum())
        n_tot += d.size
        assert np.allclose(gpu["scales"], ref["scales"], rtol=1e-5, atol=0)
        assert np.max(np.abs(out - ref_out)) <= 1e-3 * np.max(np.abs(ref_out))
        st = ref
    assert n_diff <= 1e-5 * n_tot, (n_diff, n_tot)


def test_gdn_int4_sr_bit_exact():
    w = WL[4]
    run = Run(w, bits_for(w), B=8)
    _trajectory(run, 5)


# ---------------------------------------------------------------------------
# Full sizes, in the launch configuration the benchmark times (sampled heads)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("idx,steps,nsample", [(1, 3, 96), (2, 2, 64), (3, 2, 48), (4, 2, 64)])
def test_full_size_sampled_heads(idx, steps, nsample):
    """Full workload sizes in the benchmark's launch configuration; the oracle
    computes a sample of heads (including the first and last) one by one."""
    w = WL[idx]
    run = Run(w, bits_for(w))
    heads = sample_heads(run.B, run.H, nsample, seed=idx)
    _trajectory(run, steps, heads=heads)


def test_persistent_ragged_all_heads():
    """More units than resident CTAs (several grid-stride rounds and a ragged tail):
    every head compared."""
    w = WL[1]
    run = Run(w, bits_for(w, 9), B=37, H=9)
    assert run.B * run.H * 2 > 148 * 4
    _trajectory(run, 2)


def test_persistent_many_rounds_sampled():
    """At least five units per CTA, so every pipeline stage is refilled and its
    barrier phase flips more than once."""
    w = WL[4]
    run = Run(w, bits_for(w), B=320, H=16)
    heads = sample_heads(run.B, run.H, 80, seed=9)
    _trajectory(run, 2, heads=heads)


# ---------------------------------------------------------------------------
# Shapes, formats and modes
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dk", [16, 32, 64, 128])
@pytest.mark.parametrize("dv", [16, 32, 64, 256])
def test_shapes_gdn(dk, dv):
    w = dataclasses.replace(WL[1], B=3, H=5, dk=dk, dv=dv)
    rng = np.random.default_rng(dk * 1000 + dv)
    bits = rng.choice([4, 8], size=5).astype(np.int8)
    run = Run(w, bits)
    _trajectory(run, 3)


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 32), (128, 128)])
def test_shapes_mamba2_groups(dk, dv):
    w = dataclasses.replace(WL[3], B=2, H=6, dk=dk, dv=dv, ngroups=3)
    run = Run(w, np.array([8, 4, 8, 4, 8, 4], np.int8))
    _trajectory(run, 3)


@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
@pytest.mark.parametrize("in_dtype", [rsq.RSQ_F32, rsq.RSQ_BF16])
def test_rounding_and_input_dtypes(rounding, in_dtype):
    w = dataclasses.replace(WL[1], B=3, H=4)
    run = Run(w, np.array([8, 4, 4, 8], np.int8), rounding=rounding, in_dtype=in_dtype)
    _trajectory(run, 3)


@pytest.mark.parametrize("family", ["gdn", "mamba2"])
def test_fp32_state_bit_exact(family):
    """Full-precision state (no quantization): the decode step against the oracle's
    FP32 mode, bit for bit."""
    w = dataclasses.replace(WL[1] if family == "gdn" else WL[3], B=3, H=4)
    run = Run(w, np.full(4, 32, np.int8))
    _trajectory(run, 4)


def test_in_place_update_matches_ping_pong():
    w = dataclasses.replace(WL[1], B=4, H=8)
    run = Run(w, bits_for(w, 8))
    st = run.zero()
    a, b = run.upload(st), run.upload(st)
    c = run.upload(st)
    for t in range(3):
        inp = run.inputs(t)
        o1 = run.gpu_step(a, b, inp, t)
        o2 = run.gpu_step(c, c, inp, t)
        assert np.array_equal(host(b.codes), host(c.codes))
        assert np.array_equal(host(b.scales), host(c.scales))
        assert np.array_equal(o1, o2)
        a, b = b, a


def test_checkpoint_resume_bit_identical():
    """The quantized state plus (seed, step) is a complete checkpoint: T steps equal
    T/2 steps, a copy to the host and back, and T/2 more."""
    w = dataclasses.replace(WL[4], B=4, H=4)
    run = Run(w, bits_for(w, 4))
    st = run.zero()
    a, b = run.upload(st), run.upload(st)
    for t in range(6):
        run.gpu_step(a, b, run.inputs(t), t)
        a, b = b, a
    full = (host(a.codes), host(a.scales))
    c, d = run.upload(st), run.upload(st)
    for t in range(3):
        run.gpu_step(c, d, run.inputs(t), t)
        c, d = d, c
    ck = (host(c.codes).copy(), host(c.scales).copy())
    del c, d
    e = rsq.State(dev(ck[0]), dev(ck[1]))
    f = rsq.State(dev(ck[0]), dev(ck[1]))
    for t in range(3, 6):
        run.gpu_step(e, f, run.inputs(t), t)
        e, f = f, e
    assert np.array_equal(host(e.codes), full[0]) and np.array_equal(host(e.scales), full[1])


def test_nonfinite_column_flagged_and_zeroed():
    """A NaN in one head's values makes its columns non-finite: scale NaN, zero codes,
    the context flag raised; other heads unaffected."""
    w = dataclasses.replace(WL[1], B=2, H=4)
    run = Run(w, np.array([8, 8, 4, 4], np.int8))
    assert run.ctx.check_flags() == 0
    st = run.zero()
    g_in, g_out = run.upload(st), run.upload(st)
    inp = run.inputs(0)
    v = W.bf16_to_f32(inp["v"]).copy()
    v[1, 2, 5] = np.nan
    inp["v"] = W.bf16_bits(v)
    run.gpu_step(g_in, g_out, inp, 0)
    gpu = run.download(g_out)
    ref, _ = run.oracle_step(st, inp, 0)
    assert_state_equal(gpu, ref, run.head_bits)
    assert np.isnan(gpu["scales"][1, 2, 5]) and not gpu["codes"][1, 2, :, 5].any()
    assert run.ctx.check_flags() == 1
    assert run.ctx.check_flags() == 0


def test_quantize_dequantize_kernels_bit_exact():
    for rounding in (rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8):
        w = dataclasses.replace(WL[1], B=3, H=4, dk=64, dv=128)
        run = Run(w, np.array([8, 4, 8, 4], np.int8), rounding=rounding)
        rng = np.random.default_rng(rounding)
        S = (rng.standard_normal((3, 4, 64, 128)) * rng.uniform(0.01, 5, (3, 4, 1, 128))).astype(np.float32)
        S[0, 1, :, 7] = 0.0  # an all-zero column
        s = run.ctx.alloc_state()
        run.ctx.quantize(dev(S), s, step=11)
        torch.cuda.synchronize()
        got = run.download(s)
        ref = oracle.quantize(S, run.head_bits, rounding=rounding, seed=run.seed, step=11)
        assert_state_equal(got, ref, run.head_bits, what="quantize")
        D = torch.empty((3, 4, 64, 128), dtype=torch.float32, device="cuda")
        run.ctx.dequantize(s, D)
        torch.cuda.synchronize()
        want = oracle.dequantize(ref, run.head_bits)
        assert np.array_equal(host(D).view(np.uint32), want.view(np.uint32))


def test_zero_state_quantizes_to_zero_code():
    w = dataclasses.replace(WL[1], B=2, H=2)
    run = Run(w, np.array([8, 4], np.int8))
    s = run.ctx.alloc_state()
    run.ctx.quantize(torch.zeros((2, 2, 128, 128), device="cuda"), s)
    torch.cuda.synchronize()
    codes = host(s.codes)
    off4 = rsq.rsq_head_offset(run.ctx.ctx, 1)
    assert np.all(codes[:, :off4] == 0x80) and np.all(codes[:, off4:] == 0x88)
    assert not host(s.scales).any()


def test_state_drift_kernel():
    w = dataclasses.replace(WL[4], B=3, H=4)
    q = Run(w, np.full(4, 4, np.int8))
    f = Run(w, np.full(4, 32, np.int8))
    rng = np.random.default_rng(5)
    S = rng.standard_normal((3, 4, 128, 128)).astype(np.float32)
    qs = oracle.quantize(S, q.head_bits, rounding=rsq.RSQ_SR, seed=1, step=0)
    fs = oracle.zero_state(3, 4, 128, 128)
    fs["f"] = S + rng.standard_normal(S.shape).astype(np.float32) * 0.01
    sums = torch.zeros((3, 4, 2), dtype=torch.float64, device="cuda")
    rsq.rsq_state_drift(q.ctx.ctx, q.upload(qs), f.ctx.ctx, f.upload(fs), sums)
    torch.cuda.synchronize()
    deq = oracle.dequantize(qs, q.head_bits).astype(np.float64)
    e2 = ((deq - fs["f"]) ** 2).sum(axis=(2, 3))
    f2 = (fs["f"].astype(np.float64) ** 2).sum(axis=(2, 3))
    got = host(sums)
    assert np.allclose(got[..., 0], e2, rtol=1e-12) and np.allclose(got[..., 1], f2, rtol=1e-12)


def test_misaligned_pointer_rejected_without_launch():
    w = dataclasses.replace(WL[1], B=1, H=2)
    run = Run(w, np.array([8, 8], np.int8))
    s = run.ctx.alloc_state()
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    bad = rsq.State(int(buf.data_ptr()) + 4, s.scales)
    ins, keep = run.dev_inputs(run.inputs(0))
    out = torch.empty((1, 2, 128), device="cuda")
    with pytest.raises(rsq.RsqError) as e:
        run.ctx.decode_step(bad, s, ins, out, 0)
    assert e.value.status == rsq.RSQ_E_INVAL


@pytest.mark.parametrize("family,rounding", [("gdn", rsq.RSQ_RTN), ("gdn", rsq.RSQ_SR), ("gdn", rsq.RSQ_SR8_BDR),
                                             ("mamba2", rsq.RSQ_SR8), ("gla", rsq.RSQ_SR8), ("kda", rsq.RSQ_RTN)])
def test_large_batch_geometry_sampled(family, rounding):
    """Enough units per resident CTA that the library gives each warp two
    blocks per unit (d_k = 128): sampled heads bit-exact against the oracle for
    every family and several rules."""
    base = {"gdn": WL[1], "mamba2": WL[3], "gla": W.BY_NAME["gla_b64_h16_d128_int8_sr"],
            "kda": W.BY_NAME["kda_b64_h16_d128_int8_sr"]}[family]
    w = dataclasses.replace(base, B=320, H=16)
    bits = np.array([8, 4] * 8, np.int8)
    run = Run(w, bits, rounding=rounding)
    heads = sample_heads(run.B, run.H, 40, seed=17)
    _trajectory(run, 2, heads=heads)
