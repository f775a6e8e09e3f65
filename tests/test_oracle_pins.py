"""Pins of the CPU oracle against what the method description and mathematics fix.

Each test names the passage it checks.  None of them re-types the oracle's own
formula: they use closed forms, bounds, exhaustive enumeration, statistical
laws, an independent library implementation, or brute force on tiny inputs.
CPU only.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import workloads as W
import plain_order
import workloads as W_mod

TINY = W.WORKLOADS[0]                      # GDN B=1 H=2 d=16, fp32 inputs, 64 steps
TINY_M = dataclasses.replace(W.WORKLOADS[3], name="mamba2_tiny", B=1, H=2, dk=16, dv=16,
                             steps=64, in_dtype="f32")


def _rel(a, b):
    return float(np.linalg.norm((a - b).ravel()) / np.linalg.norm(b.ravel()))


# ---------------------------------------------------------------------------
# (a) quantization disabled == closed-form unrolled sum of decayed outer products
# ---------------------------------------------------------------------------
def _gdn_closed_form(ins, t_end, b, h):
    """S_t = sum_tau [prod_{s=tau+1..t} alpha_s (I - beta_s k_s k_s^T)] beta_tau k_tau v_tau^T."""
    ks = [np.asarray(i["k"][b, h], np.float64) for i in ins[:t_end]]
    vs = [np.asarray(i["v"][b, h], np.float64) for i in ins[:t_end]]
    al = [float(i["alpha"][b, h]) for i in ins[:t_end]]
    be = [float(i["beta"][b, h]) for i in ins[:t_end]]
    d = ks[0].shape[0]
    S = np.zeros((d, vs[0].shape[0]))
    for tau in range(t_end):
        M = be[tau] * np.outer(ks[tau], vs[tau])
        for s in range(tau + 1, t_end):
            M = al[s] * (M - be[s] * np.outer(ks[s], ks[s] @ M))
        S += M
    return S


@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_gdn_fp32_state_matches_closed_form(mode):
    """Quantization disabled: the closed-form unrolled sum of decayed outer
    products; recurrence of the gated delta rule (Gated DeltaNet)."""
    w = TINY
    ins = [W.gdn_inputs(w, t) for t in range(w.steps)]
    bits = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    for t in range(w.steps):
        st, o = oracle.gdn_step(st, ins[t], bits, rounding=oracle.RTN, seed=0, step=t, mode=mode)
        if t in (0, 7, 31, w.steps - 1):
            for h in range(w.H):
                S_ref = _gdn_closed_form(ins, t + 1, 0, h)
                assert _rel(st["f"][0, h].astype(np.float64), S_ref) <= 1e-5
                o_ref = S_ref.T @ ins[t]["q"][0, h].astype(np.float64)
                assert _rel(o[0, h].astype(np.float64), o_ref) <= 1e-5


@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_gdn_fp32_state_matches_closed_form_dk256(mode):
    """The closed-form unrolled sum at d_k = 256, with the 16-partial canonical order the
    library uses there (rsq_reduction_partials(256) = 16)."""
    w = dataclasses.replace(TINY, B=1, H=2, dk=256, dv=32)
    ins = [W.gdn_inputs(w, t) for t in range(6)]
    bits = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    for t in range(6):
        st, o = oracle.gdn_step(st, ins[t], bits, rounding=oracle.RTN, seed=0, step=t, mode=mode, R=16)
        for h in range(w.H):
            S_ref = _gdn_closed_form(ins, t + 1, 0, h)
            assert _rel(st["f"][0, h].astype(np.float64), S_ref) <= 1e-5
            o_ref = S_ref.T @ ins[t]["q"][0, h].astype(np.float64)
            assert _rel(o[0, h].astype(np.float64), o_ref) <= 1e-5


def _mamba_closed_form(ins, t_end, b, h, D):
    """S_t = sum_tau (prod_{s>tau} exp(dt_s A)) dt_tau B_tau x_tau^T;  y_t = S_t^T C_t + D x_t."""
    S = np.zeros((ins[0]["Bm"].shape[-1], ins[0]["x"].shape[-1]))
    for tau in range(t_end):
        decay = 1.0
        for s in range(tau + 1, t_end):
            decay *= float(np.float32(np.exp(np.float64(ins[s]["dt"][b, h]) * ins[s]["A"][h])))
        S += decay * float(ins[tau]["dt"][b, h]) * np.outer(ins[tau]["Bm"][b, 0], ins[tau]["x"][b, h])
    y = S.T @ ins[t_end - 1]["Cm"][b, 0].astype(np.float64) + D * ins[t_end - 1]["x"][b, h]
    return S, y


@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_mamba2_fp32_state_matches_closed_form(mode):
    """Quantization disabled: the closed-form unrolled sum of decayed outer
    products; Mamba-2 scalar-decay recurrence."""
    w = TINY_M
    ins = [W.mamba2_inputs(w, t) for t in range(w.steps)]
    # exp(dt*A) passed explicitly (correctly rounded) so the closed form uses the same decays
    decays = [np.exp(i["dt"].astype(np.float64) * i["A"][None, :]).astype(np.float32) for i in ins]
    bits = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    for t in range(w.steps):
        st, y = oracle.mamba2_step(st, ins[t], bits, rounding=oracle.RTN, seed=0, step=t, mode=mode,
                                   decay=decays[t])
        if t in (0, 9, w.steps - 1):
            for h in range(w.H):
                S_ref, y_ref = _mamba_closed_form(ins, t + 1, 0, h, float(ins[0]["D"][h]))
                assert _rel(st["f"][0, h].astype(np.float64), S_ref) <= 1e-5
                assert _rel(y[0, h].astype(np.float64), y_ref) <= 1e-5


def test_injected_error_survives_as_alpha_pow_n():
    """(2/4) Mixed precision, animation: one injected error under constant scalar
    decay and no further rounding survives as ||E_n|| / ||E_0|| = alpha^n."""
    w = TINY_M
    a = np.float32(0.75)  # exactly representable; powers of 0.75 stay exact for small n
    rng = np.random.default_rng(5)
    E0 = rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
    bits = np.full(w.H, 32, np.int8)
    s1, s2 = oracle.zero_state(w.B, w.H, w.dk, w.dv), oracle.zero_state(w.B, w.H, w.dk, w.dv)
    s2["f"] = E0.copy()
    for n in range(1, 25):
        inp = W.mamba2_inputs(w, n)
        dec = np.full((w.B, w.H), a, np.float32)
        s1, _ = oracle.mamba2_step(s1, inp, bits, rounding=0, seed=0, step=n, decay=dec)
        s2, _ = oracle.mamba2_step(s2, inp, bits, rounding=0, seed=0, step=n, decay=dec)
        ratio = np.linalg.norm((s2["f"] - s1["f"]).astype(np.float64)) / np.linalg.norm(E0.astype(np.float64))
        assert abs(ratio - 0.75 ** n) <= 1e-5 * 0.75 ** n + 1e-6


def test_gdn_error_contraction_delta_rule():
    """(2/4) Proposition (decaying error) with no further rounding: for unit-norm
    keys and 0 < beta < 2 the transition alpha (I - beta k k^T) has norm <= alpha,
    so a state difference shrinks at least as alpha^n."""
    w = TINY
    bits = np.full(w.H, 32, np.int8)
    rng = np.random.default_rng(6)
    E0 = rng.standard_normal((w.B, w.H, w.dk, w.dv)).astype(np.float32)
    s1, s2 = oracle.zero_state(w.B, w.H, w.dk, w.dv), oracle.zero_state(w.B, w.H, w.dk, w.dv)
    s2["f"] = E0.copy()
    bound = np.ones(w.H)
    for n in range(20):
        inp = W.gdn_inputs(w, n)
        s1, _ = oracle.gdn_step(s1, inp, bits, rounding=0, seed=0, step=n, mode=oracle.PLAIN)
        s2, _ = oracle.gdn_step(s2, inp, bits, rounding=0, seed=0, step=n, mode=oracle.PLAIN)
        bound *= inp["alpha"][0].astype(np.float64)
        for h in range(w.H):
            e = np.linalg.norm((s2["f"][0, h] - s1["f"][0, h]).astype(np.float64))
            assert e <= bound[h] * np.linalg.norm(E0[0, h].astype(np.float64)) * (1 + 1e-4)


# ---------------------------------------------------------------------------
# (b) round-to-nearest error at most half a step; brute-force optimality
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_rtn_error_at_most_half_step(bits, mode):
    """Round-to-nearest error at most half a step; (1/4) Proposition: rounding
    errors within half a grid step."""
    rng = np.random.default_rng(bits)
    S = (rng.standard_normal((3, 4, 32, 24)) * rng.uniform(0.01, 10, (3, 4, 1, 24))).astype(np.float32)
    st = oracle.quantize(S, np.full(4, bits, np.int8), rounding=oracle.RTN, seed=0, step=0, mode=mode)
    deq = oracle.dequantize(st, np.full(4, bits, np.int8)).astype(np.float64)
    s = st["scales"][:, :, None, :].astype(np.float64)
    r = oracle.rmax(bits)
    # reciprocal multiplier and scale each carry <= 1 ulp: slack r * 2^-22 of a step
    assert np.all(np.abs(deq - S) <= s * (0.5 + r * 2.0 ** -22) + 1e-30)
    assert np.abs(st["codes"]).max() <= r
    # scale = absmax / r, and the absmax element gets code +-r
    m = np.abs(S).max(axis=2)
    assert np.allclose(st["scales"], m / r, rtol=2 ** -23, atol=0)
    assert np.all(np.abs(st["codes"]).max(axis=2) == r)


@pytest.mark.parametrize("bits", [8, 4])
def test_rtn_brute_force_nearest_code(bits):
    """Brute force over every code on tiny columns: the RTN code minimises |c*s - S|
    (ties resolved to an even code)."""
    rng = np.random.default_rng(100 + bits)
    r = oracle.rmax(bits)
    for _ in range(300):
        col = rng.standard_normal(4).astype(np.float32) * np.float32(rng.uniform(0.1, 3))
        m = float(np.abs(col).max())
        s = np.float64(np.float32(m / r))
        for S in col:
            c = oracle.quantize_scalar(S, m, bits, oracle.RTN, oracle.CANONICAL)
            errs = np.abs(np.arange(-r, r + 1) * s - np.float64(S))
            best = errs.min()
            # the chosen code is optimal up to the one-ulp multiplier error
            assert errs[c + r] <= best + s * r * 2.0 ** -22


@pytest.mark.parametrize("bits", [8, 4])
def test_subnormal_column_maxima(bits):
    """Columns whose maximum m is so small that r/m overflows binary32.
    Canonical order: the multiplier r/m rounded toward zero saturates at FLT_MAX,
    so codes are the nearest integers of the exact products S * FLT_MAX (closed
    form, float64).  Plain order: once s = m/r underflows to zero, every nonzero
    element gets the code sign(S) r and a zero element 0; the stored scale is 0
    either way, so both orders dequantize such a column to zeros."""
    r = oracle.rmax(bits)
    fmax = np.float64(np.finfo(np.float32).max)
    hb = np.array([bits], np.int8)
    for m in (np.float32(1e-38), np.float32(3e-39), np.float32(1e-40)):
        assert np.float64(r) / np.float64(m) > fmax      # r/m overflows
        col = np.array([m, -m, m / 2, -m / 3, 0, m / 7, -m, m / 5], np.float32)
        S = np.zeros((1, 1, 8, 2), np.float32)
        S[0, 0, :, 0] = col
        st = oracle.quantize(S, hb, rounding=oracle.RTN, seed=0, step=0, mode=oracle.CANONICAL)
        want = np.rint(col.astype(np.float64) * fmax).astype(np.int64)
        assert np.array_equal(st["codes"][0, 0, :, 0], want)
        assert st["scales"][0, 0, 0] == np.float32(m) / np.float32(r)
        assert st["scales"][0, 0, 1] == 0 and not st["codes"][0, 0, :, 1].any()   # all-zero column
    m = np.float32(2 * np.finfo(np.float32).smallest_subnormal)
    assert np.float32(m) / np.float32(r) == 0                                        # s underflows
    col = np.array([m, -m, 0, np.float32(m / 4), -np.float32(m / 2), 0, m, -m], np.float32)
    S = np.zeros((1, 1, 8, 1), np.float32)
    S[0, 0, :, 0] = col
    for rnd in (oracle.RTN, oracle.SR):
        st = oracle.quantize(S, hb, rounding=rnd, seed=3, step=1, mode=oracle.PLAIN)
        assert np.array_equal(st["codes"][0, 0, :, 0], (np.sign(col) * r).astype(np.int64))
        assert st["scales"][0, 0, 0] == 0
        assert not oracle.dequantize(st, hb).any()


# ---------------------------------------------------------------------------
# (c) stochastic rounding is (conditionally) unbiased
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_sr_exhaustive_probability(bits, mode):
    """(3/4) Rounding: SR is conditionally unbiased.  Enumerating all 2^16 uniforms,
    P(round up) equals frac(x) to within 2^-16 for every x."""
    r = oracle.rmax(bits)
    m = float(r)               # column max r -> scale 1 and multiplier 1: x = S exactly
    rng = np.random.default_rng(7 + bits)
    xs = list(rng.uniform(-r, r, 10).astype(np.float32)) + [np.float32(v) for v in
                                                          (0.0, 0.5, -0.5, 3.25, -2.75, r, -r, 1e-3)]
    us = np.arange(65536)
    for x in xs:
        x = float(x)
        lo = np.floor(x)
        codes = np.array([oracle.quantize_scalar(x, m, bits, oracle.SR, mode, int(u)) for u in us[::1]])
        assert set(np.unique(codes)) <= {int(lo), int(lo) + 1}
        p_up = float(np.mean(codes == lo + 1))
        assert abs(p_up - (x - lo)) <= 2.0 ** -16 + 1e-12, (x, p_up)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_sr8_exhaustive_probability(bits, mode):
    """(3/4) Rounding with 8-bit uniforms: enumerating all 256 uniforms, every
    code is floor(x) or floor(x) + 1, P(round up) equals frac(x) to within
    2^-9, and a value within 2^-9 of an integer is never moved off it."""
    r = oracle.rmax(bits)
    m = float(r)               # column max r -> scale 1 and multiplier 1: x = S exactly
    rng = np.random.default_rng(17 + bits)
    xs = list(rng.uniform(-r, r, 24).astype(np.float32)) + [np.float32(v) for v in (
        0.0, 0.5, -0.5, 3.25, -2.75, r, -r, 1e-3, -1e-3, 2.0 - 2.0 ** -10, 1.0 + 2.0 ** -10,
        0.5 + 2.0 ** -9, 0.25 - 2.0 ** -11)]
    for x in xs:
        x = float(x)
        lo = np.floor(x)
        codes = np.array([oracle.quantize_scalar(x, m, bits, oracle.SR8, mode, u) for u in range(256)])
        assert set(np.unique(codes)) <= {int(lo), int(lo) + 1}
        p_up = float(np.mean(codes == lo + 1))
        assert abs(p_up - (x - lo)) <= 2.0 ** -9 + 1e-12, (x, p_up)
        near = np.round(x)
        if abs(x - near) < 2.0 ** -9:
            assert np.all(codes == near), (x, np.unique(codes))


def test_sr8_unbiased_over_draws():
    """Stochastic rounding with 8-bit uniforms is unbiased to within 2^-9 of a
    step: the mean of dequantized values over many draws converges to the value."""
    rng = np.random.default_rng(13)
    S = (rng.standard_normal((1, 2, 16, 16))).astype(np.float32)
    bits = np.full(2, 4, np.int8)
    n = 400
    acc = np.zeros(S.shape)
    for t in range(n):
        st = oracle.quantize(S, bits, rounding=oracle.SR8, seed=4321, step=t, mode=oracle.CANONICAL)
        acc += oracle.dequantize(st, bits).astype(np.float64)
    mean = acc / n
    s = st["scales"][:, :, None, :].astype(np.float64)
    x = S.astype(np.float64) / s
    phi = x - np.floor(x)
    sigma = s * np.sqrt(np.maximum(phi * (1 - phi), 1.0 / n) / n)
    assert np.all(np.abs(mean - S) <= 5 * sigma + s * 2.0 ** -9)


@pytest.mark.parametrize("bits", [8, 4])
def test_sr8_quantize_dequantize_idempotent(bits):
    """With 8-bit uniforms (values within 2^-9 of an integer stay on it),
    quantize o dequantize is idempotent for stochastic rounding: the codes of
    Q(D(Q(S))) equal those of Q(S) whatever the second draw."""
    rng = np.random.default_rng(41 + bits)
    S = (rng.standard_normal((4, 4, 64, 64)) * 2).astype(np.float32)
    hb = np.full(4, bits, np.int8)
    for mode in (oracle.PLAIN, oracle.CANONICAL):
        q1 = oracle.quantize(S, hb, rounding=oracle.SR8, seed=9, step=1, mode=mode)
        q2 = oracle.quantize(oracle.dequantize(q1, hb), hb, rounding=oracle.SR8, seed=9, step=2, mode=mode)
        assert np.array_equal(q1["codes"], q2["codes"])


def test_sr_unbiased_over_draws():
    """Stochastic rounding is unbiased: the mean of SR-dequantized values over many independent
    draws (steps) converges to the value (5 sigma)."""
    rng = np.random.default_rng(11)
    S = (rng.standard_normal((1, 2, 16, 16))).astype(np.float32)
    bits = np.full(2, 4, np.int8)
    n = 400
    acc = np.zeros(S.shape)
    for t in range(n):
        st = oracle.quantize(S, bits, rounding=oracle.SR, seed=1234, step=t, mode=oracle.CANONICAL)
        d = oracle.dequantize(st, bits).astype(np.float64)
        acc += d
    mean = acc / n
    s = st["scales"][:, :, None, :].astype(np.float64)
    x = S.astype(np.float64) / s
    phi = x - np.floor(x)
    sigma = s * np.sqrt(np.maximum(phi * (1 - phi), 1.0 / n) / n)   # Bernoulli(phi) law of SR
    assert np.all(np.abs(mean - S) <= 5 * sigma + s * 2.0 ** -15)


# ---------------------------------------------------------------------------
# (d) quantize o dequantize is idempotent
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [8, 4])
def test_rtn_quantize_dequantize_idempotent(bits):
    """quantize o dequantize is idempotent: Q(D(Q(S))) == Q(S) for round-to-nearest (codes bit-exact,
    scales within one ulp)."""
    rng = np.random.default_rng(21 + bits)
    S = (rng.standard_normal((2, 3, 32, 64)) * 3).astype(np.float32)
    hb = np.full(3, bits, np.int8)
    q1 = oracle.quantize(S, hb, rounding=oracle.RTN, seed=0, step=0)
    q2 = oracle.quantize(oracle.dequantize(q1, hb), hb, rounding=oracle.RTN, seed=0, step=0)
    assert np.array_equal(q1["codes"], q2["codes"])
    ulp = np.spacing(q1["scales"])
    assert np.all(np.abs(q1["scales"] - q2["scales"]) <= ulp)


@pytest.mark.parametrize("bits", [8, 4])
def test_sr_quantize_dequantize_nearly_idempotent(bits):
    """Idempotence for stochastic rounding: re-quantizing dequantized codes moves
    at most a 1e-5 fraction of the codes, each by at most one step."""
    rng = np.random.default_rng(31 + bits)
    S = (rng.standard_normal((4, 4, 64, 64)) * 2).astype(np.float32)
    hb = np.full(4, bits, np.int8)
    q1 = oracle.quantize(S, hb, rounding=oracle.SR, seed=9, step=1)
    q2 = oracle.quantize(oracle.dequantize(q1, hb), hb, rounding=oracle.SR, seed=9, step=2)
    diff = np.abs(q1["codes"].astype(int) - q2["codes"].astype(int))
    assert diff.max() <= 1
    assert np.mean(diff != 0) <= 1e-5


def test_zero_state_quantizes_to_zero():
    """S_0 = 0: scales 0, codes 0 (a zero column has no usable scale)."""
    st = oracle.quantize(np.zeros((1, 2, 16, 16), np.float32), np.array([8, 4], np.int8),
                         rounding=oracle.SR, seed=1, step=0)
    assert not st["codes"].any() and not st["scales"].any()


# ---------------------------------------------------------------------------
# First step from S_0 = 0 (closed form of the quantizer on a rank-one state)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_first_step_rank_one_codes(mode):
    """From S_0 = 0 the delta rule gives S_1 = beta k v^T (rank one), so every
    column's codes are round(r * k_i * sign(v_j) / max|k|) and its scale is
    beta |v_j| max|k| / r -- identical columns up to sign."""
    w = TINY
    inp = W.gdn_inputs(w, 0)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    hb = np.full(w.H, 8, np.int8)
    st1, o = oracle.gdn_step(st, inp, hb, rounding=oracle.RTN, seed=0, step=0, mode=mode)
    for h in range(w.H):
        k = inp["k"][0, h].astype(np.float64)
        v = inp["v"][0, h].astype(np.float64)
        beta = float(inp["beta"][0, h])
        expect = 127 * np.outer(k, np.sign(v)) / np.abs(k).max()
        assert np.all(np.abs(st1["codes"][0, h] - expect) <= 0.5 + 1e-4)
        s_expect = beta * np.abs(v) * np.abs(k).max() / 127
        assert np.allclose(st1["scales"][0, h], s_expect, rtol=1e-5)
        # readout from the full-precision S_1 = beta k v^T: o = beta (k.q) v
        o_expect = beta * float(k @ inp["q"][0, h]) * v
        assert np.allclose(o[0, h], o_expect, rtol=1e-5, atol=1e-6)


# ---------------------------------------------------------------------------
# Statistical laws of the method description
# ---------------------------------------------------------------------------
def test_value_axis_readout_error_variance():
    """(1/4) Proposition (per-channel readout error), value-axis grouping:
    E[e_j^2] = M_j^2 / (12 r^2) for a unit-norm query (within 10%)."""
    rng = np.random.default_rng(41)
    bits, r = 8, 127
    ratios = []
    for rep in range(40):
        S = rng.standard_normal((1, 1, 64, 64)).astype(np.float32)
        st = oracle.quantize(S, np.array([bits], np.int8), rounding=oracle.RTN, seed=0, step=0)
        E = (oracle.dequantize(st, np.array([bits], np.int8)) - S)[0, 0].astype(np.float64)
        q = rng.standard_normal((64, 64))
        q /= np.linalg.norm(q, axis=0, keepdims=True)      # 64 unit-norm queries
        e = E.T @ q                                          # e[j, n] = sum_i E_ij q_in
        M = np.abs(S[0, 0]).max(axis=0).astype(np.float64)
        ratios.append(np.mean(e ** 2, axis=1) / (M ** 2 / (12 * r * r)))
    assert abs(np.mean(ratios) - 1.0) <= 0.10


def _gdn_traj(w, steps, bits_h, rounding, seed, mode):
    ins = [W.gdn_inputs(w, t) for t in range(steps)]
    hb = np.full(w.H, bits_h, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    out = []
    for t in range(steps):
        st, _ = oracle.gdn_step(st, ins[t], hb, rounding=rounding, seed=seed, step=t, mode=mode)
        out.append(oracle.copy_state(st))
    return ins, out


@pytest.mark.parametrize("rounding", [oracle.RTN, oracle.SR, oracle.SR8])
def test_decaying_error_bound(rounding):
    """(2/4) Proposition (decaying error): ||E_t||_F <= sum_tau alpha^(t-tau) ||eps_tau||_F
    with alpha = max alpha_t, unit-norm keys and 0 < beta < 2."""
    w = TINY
    T = 48
    ins, traj = _gdn_traj(w, T, 4, rounding, 77, oracle.PLAIN)
    hb32 = np.full(w.H, 32, np.int8)
    hb4 = np.full(w.H, 4, np.int8)
    ref = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    prev = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    amax = max(float(i["alpha"].max()) for i in ins)
    acc = np.zeros(w.H)
    for t in range(T):
        ref, _ = oracle.gdn_step(ref, ins[t], hb32, rounding=0, seed=0, step=t, mode=oracle.PLAIN)
        # S_pre: full-precision update of the previous dequantized state
        pre_in = oracle.zero_state(w.B, w.H, w.dk, w.dv)
        pre_in["f"] = oracle.dequantize(prev, hb4) if t else pre_in["f"]
        pre, _ = oracle.gdn_step(pre_in, ins[t], hb32, rounding=0, seed=0, step=t, mode=oracle.PLAIN)
        deq = oracle.dequantize(traj[t], hb4).astype(np.float64)
        eps = np.linalg.norm((deq - pre["f"]).reshape(w.H, -1), axis=1)
        acc = amax * acc + eps
        E = np.linalg.norm((deq - ref["f"]).reshape(w.H, -1), axis=1)
        assert np.all(E <= acc * (1 + 1e-3) + 1e-6)
        prev = traj[t]


@pytest.mark.slow
def test_sr_cross_terms_vanish_in_expectation():
    """(3/4) Proposition (repeated quantization): with scalar decay, no delta
    correction and writes fixed independently of rounding, the remainder
    R_t = E_t^2 - sum_tau gamma^2 eps_tau^2 has zero mean under SR."""
    w = dataclasses.replace(TINY_M, H=1, dk=4, dv=4)
    T, n_seeds = 40, 150
    hb4, hb32 = np.array([4], np.int8), np.array([32], np.int8)
    ins = [W.mamba2_inputs(w, t) for t in range(T)]
    dec = [np.full((1, 1), 0.9, np.float32) for _ in range(T)]
    ref = oracle.zero_state(1, 1, 4, 4)
    refs = []
    for t in range(T):
        ref, _ = oracle.mamba2_step(ref, ins[t], hb32, rounding=0, seed=0, step=t, decay=dec[t])
        refs.append(ref["f"].astype(np.float64))
    Rs = []
    for seed in range(n_seeds):
        st = oracle.zero_state(1, 1, 4, 4)
        acc = np.zeros((4, 4))
        for t in range(T):
            pre_in = oracle.zero_state(1, 1, 4, 4)
            pre_in["f"] = oracle.dequantize(st, hb4)
            pre, _ = oracle.mamba2_step(pre_in, ins[t], hb32, rounding=0, seed=0, step=t, decay=dec[t])
            st, _ = oracle.mamba2_step(st, ins[t], hb4, rounding=oracle.SR, seed=seed, step=t,
                                       mode=oracle.PLAIN, decay=dec[t])
            eps = oracle.dequantize(st, hb4).astype(np.float64) - pre["f"]
            acc = 0.81 * acc + eps ** 2
        E = oracle.dequantize(st, hb4).astype(np.float64) - refs[-1]
        Rs.append(float((E ** 2 - acc).sum()))
    Rs = np.array(Rs)
    assert abs(Rs.mean()) <= 5 * Rs.std() / np.sqrt(n_seeds)


# ---------------------------------------------------------------------------
# Philox4x32-10 against an independent library implementation
# ---------------------------------------------------------------------------
def test_philox_matches_triton_cpu_interpreter():
    """Counter-based RNG: the oracle's Philox4x32-10 equals the Philox block of an
    independent implementation (Triton's random module run by its CPU interpreter)."""
    import os
    import subprocess
    import sys
    import json
    rng = np.random.default_rng(3)
    ctr = rng.integers(0, 2 ** 32, (64, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, (64, 2), dtype=np.uint64)
    ctr[0] = 0; key[0] = 0
    ctr[1] = 2 ** 32 - 1; key[1] = 2 ** 32 - 1
    script = r'''
import os, sys, json
os.environ["TRITON_INTERPRET"] = "1"
import torch, triton, triton.language as tl
@triton.jit
def kern(c0p, c1p, c2p, c3p, k0p, k1p, o0, o1, o2, o3, N: tl.constexpr):
    i = tl.arange(0, N)
    a, b, c, d = tl.random.philox_impl(tl.load(c0p + i), tl.load(c1p + i), tl.load(c2p + i),
                                       tl.load(c3p + i), tl.load(k0p + i), tl.load(k1p + i), 10)
    tl.store(o0 + i, a); tl.store(o1 + i, b); tl.store(o2 + i, c); tl.store(o3 + i, d)
d = json.loads(sys.stdin.read())
t = [torch.tensor(c, dtype=torch.int64).to(torch.uint32) for c in d["cols"]]
outs = [torch.zeros(len(d["cols"][0]), dtype=torch.uint32) for _ in range(4)]
kern[(1,)](*t, *outs, N=len(d["cols"][0]))
print(json.dumps([[int(v) & 0xffffffff for v in o.tolist()] for o in outs]))
'''
    cols = [ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3], key[:, 0], key[:, 1]]
    payload = json.dumps({"cols": [[int(v) for v in c] for c in cols]})
    env = dict(os.environ, TRITON_INTERPRET="1", CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", script], input=payload, capture_output=True,
                         text=True, env=env, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    tri = np.array(json.loads(res.stdout.strip().splitlines()[-1]), dtype=np.uint64).T
    ours = oracle.philox4x32_10(ctr.astype(np.uint32), key.astype(np.uint32)).astype(np.uint64)
    assert np.array_equal(ours, tri)


def test_sr_uniforms_distinct_per_element():
    """Each element of a head draws its own 16-bit chunk: over one head the
    (Philox block, chunk) pairs are all distinct, and the uniforms are uniform."""
    dk, dv = 32, 16
    seen = set()
    vals = []
    for i in range(dk):
        for j in range(dv):
            blk = (i % (dk // 2), j // 4)
            chunk = 4 * (i >= dk // 2) + j % 4
            assert (blk, chunk) not in seen
            seen.add((blk, chunk))
            vals.append(oracle.sr_uniform16(99, 3, 5, 7, dk, i, j))
    vals = np.array(vals)
    assert vals.min() >= 0 and vals.max() < 65536
    # coarse uniformity: 16 bins, chi-square well below the 1e-6 tail
    hist = np.bincount(vals >> 12, minlength=16)
    chi2 = float(((hist - len(vals) / 16) ** 2 / (len(vals) / 16)).sum())
    assert chi2 < 60


def test_sr8_uniforms_distinct_per_element():
    """With 8-bit uniforms each element of a head draws its own byte of a
    Philox block: counter {i mod dk/4 | (j/4) << 16, h, b, step}, word i div
    dk/4, byte j mod 4.  Over one head the (block, byte) pairs are all
    distinct, each uniform is that byte of the oracle's (Triton-pinned) Philox
    output, and the uniforms are uniform."""
    for dk in (16, 128):
        dv = 32
        seen = set()
        vals = []
        for i in range(dk):
            for j in range(dv):
                blk = (i % (dk // 4), j // 4)
                slot = 4 * (i // (dk // 4)) + j % 4
                assert (blk, slot) not in seen
                seen.add((blk, slot))
                u = oracle.sr_uniform8(77, 2, 6, 9, dk, i, j)
                vals.append(u)
        if dk == 128:
            for i, j in ((0, 0), (37, 5), (127, 31), (64, 17)):
                ctr = np.array([(i % 32) | ((j // 4) << 16), 6, 2, 9], np.uint32)
                out = oracle.philox4x32_10(ctr, np.array([77, 0], np.uint32))[0]
                assert oracle.sr_uniform8(77, 2, 6, 9, dk, i, j) == (int(out[i // 32]) >> (8 * (j % 4))) & 0xFF
        vals = np.array(vals)
        assert vals.min() >= 0 and vals.max() < 256
        hist = np.bincount(vals >> 4, minlength=16)
        chi2 = float(((hist - len(vals) / 16) ** 2 / (len(vals) / 16)).sum())
        assert chi2 < 60


# ---------------------------------------------------------------------------
# Reduction order, mixed precision allocation, storage format
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("family", ["gdn", "mamba2"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("rounding", [oracle.RTN, oracle.SR, oracle.SR8])
def test_canonical_and_plain_agree_teacher_forced(family, bits, rounding):
    """Both evaluation orders compute the same mathematics ("(1/4) Scale
    grouping": s = max|S| / r, codes round(S / s); "(3/4) Rounding"): from the
    same input state at most 1e-5 of the codes differ, each by one step, apart
    from exact ties of nearest rounding (an element exactly a half-integer
    number of steps), which the two orders break differently; scales and
    outputs agree to 1e-5 relative."""
    base = W.WORKLOADS[1] if family == "gdn" else W.WORKLOADS[3]
    w = dataclasses.replace(base, B=8, H=8)
    hb = np.full(w.H, bits, np.int8)
    rng = np.random.default_rng(51 + bits + 7 * rounding)
    S = (rng.standard_normal((w.B, w.H, w.dk, w.dv)) * 0.1).astype(np.float32)
    st = oracle.quantize(S, hb, rounding=rounding, seed=1, step=0)
    step = oracle.gdn_step if family == "gdn" else oracle.mamba2_step
    n_other = n_tie = n_tot = 0
    for t in range(1, 5):
        inp = W.inputs(w, t, B=w.B)
        a, oa = step(st, inp, hb, rounding=rounding, seed=5, step=t, mode=oracle.PLAIN)
        b, ob = step(st, inp, hb, rounding=rounding, seed=5, step=t, mode=oracle.CANONICAL)
        S_lit = plain_order.literal_state(family, st, inp, hb)
        o, ti, tot = plain_order.compare_codes(b["codes"], a["codes"], S_lit, hb,
                                               nearest=rounding == oracle.RTN)
        n_other, n_tie, n_tot = n_other + o, n_tie + ti, n_tot + tot
        assert plain_order.max_rel(ob, oa) <= 1e-5
        assert np.allclose(a["scales"], b["scales"], rtol=1e-5, atol=0)
        st = b
    assert n_other <= 1e-5 * n_tot, (n_other, n_tie, n_tot)
    assert n_tie <= 1e-3 * n_tot, (n_other, n_tie, n_tot)


def test_exact_tie_broken_toward_zero_by_the_canonical_order():
    """An element exactly half its column's maximum (x = S / s = r / 2) is an
    exact tie of nearest rounding: the literal order's float scale and
    quotient decide it, the canonical order's multiplier r / m rounded toward
    zero rounds it toward zero unless r / m is exact in binary32, when the
    product is the tie itself and goes to even ("(1/4) Scale grouping";
    nearest with ties to even)."""
    for bits in (4, 8):
        r = (1 << (bits - 1)) - 1
        for m in (1.0, 0.5, 0.75, 3.0e-3, 1.7):
            m = float(np.float32(m))
            S = m / 2.0                                  # exact
            exact = float(np.float32(r / m)) == r / m    # r / m representable
            want_c = (r + 1) // 2 if exact else (r - 1) // 2   # even (4 / 64) or toward zero
            assert oracle.quantize_scalar(S, m, bits, oracle.RTN, oracle.CANONICAL) == want_c
            assert oracle.quantize_scalar(-S, m, bits, oracle.RTN, oracle.CANONICAL) == -want_c
            # the literal order: x = S / fl(m / r), nearest, ties to even
            s = np.float32(np.float32(m) / np.float32(r))
            x = np.float32(np.float32(S) / s)
            want = int(np.rint(np.float64(x)))
            assert oracle.quantize_scalar(S, m, bits, oracle.RTN, oracle.PLAIN) == want
            assert want in ((r - 1) // 2, (r + 1) // 2)


def test_allocation_matches_sort():
    """(2/4) Mixed precision: the n_hi slowest-decaying heads (largest mean alpha)
    keep 8 bits; checked against a stable sort."""
    rng = np.random.default_rng(61)
    for H in (4, 32, 80):
        score = rng.uniform(0.5, 1.0, H)
        score[H // 3] = score[H // 2]                   # a tie
        n_hi = H // 4
        got = oracle.allocate_bits(score, n_hi)
        order = sorted(range(H), key=lambda h: (-score[h], h))
        want = np.full(H, 4, np.int8)
        want[order[:n_hi]] = 8
        assert np.array_equal(got, want)


def test_storage_format_golden():
    """Byte format of the library (declared in include/rsq.h), pinned by a hand-written
    fixture: tests/golden/pack_format.txt."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "pack_format.txt")
    cases = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, key, val = line.split(None, 2)
        cases.setdefault(name, {})[key] = val
    for name, c in cases.items():
        dk, dv, bits = int(c["dk"]), int(c["dv"]), int(c["bits"])
        codes = np.array([int(v) for v in c["codes"].split()], np.int8).reshape(1, 1, dk, dv)
        st = oracle.zero_state(1, 1, dk, dv)
        st["codes"] = codes
        packed = oracle.pack_state(st, np.array([bits], np.int8))[0]
        want = bytes.fromhex(c["bytes"].replace(" ", ""))
        assert packed.tobytes() == want, name
        back = oracle.unpack_state(packed[None], np.zeros((1, 1, dv), np.float32),
                                   np.array([bits], np.int8), 1, 1, dk, dv)
        assert np.array_equal(back["codes"], codes)


def test_pack_roundtrip_mixed():
    rng = np.random.default_rng(71)
    B, H, dk, dv = 2, 3, 16, 128
    hb = np.array([8, 4, 32], np.int8)
    st = oracle.zero_state(B, H, dk, dv)
    st["codes"][:, 0] = rng.integers(-127, 128, (B, dk, dv))
    st["codes"][:, 1] = rng.integers(-7, 8, (B, dk, dv))
    st["f"][:, 2] = rng.standard_normal((B, dk, dv))
    buf = oracle.pack_state(st, hb)
    assert buf.shape == (B, dk * dv * (8 + 4 + 32) // 8)
    back = oracle.unpack_state(buf, st["scales"], hb, B, H, dk, dv)
    assert np.array_equal(back["codes"][:, :2], st["codes"][:, :2])
    assert np.array_equal(back["f"][:, 2], st["f"][:, 2])


# ---------------------------------------------------------------------------
# Bounded Directional Rounding ("Preserving Updates in Low-Bit Recurrent State
# Quantization", abstract): an element whose rounding moves it opposite to its
# update is rounded toward the update instead; the error stays below one step.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_bdr_worked_scalar_cases(mode):
    """Column maximum 127 at 8 bits: scale 1, so x = S.  Hand-derived cases."""
    m = 127.0
    rtn = lambda S: oracle.quantize_scalar(S, m, 8, oracle.RTN, mode)
    # update +0.1 from 0.3 to 0.4: nearest rounding gives 0, below the old value -> reversed -> 1
    assert rtn(0.4) == 0 and oracle.bdr_adjust(0, 0.4, 0.3, m, 8, mode) == 1
    # the mirror image: from -0.3 down to -0.4
    assert oracle.bdr_adjust(0, -0.4, -0.3, m, 8, mode) == -1
    # update from 0.5 down to 0.4: rounding to 0 moves down as well -> kept
    assert oracle.bdr_adjust(0, 0.4, 0.5, m, 8, mode) == 0
    # a lost update (0.0 -> 0.4 rounds back to 0.0) is not a reversal -> kept
    assert oracle.bdr_adjust(0, 0.4, 0.0, m, 8, mode) == 0
    # no update: kept whatever the code
    assert oracle.bdr_adjust(3, 2.6, 2.6, m, 8, mode) == 3
    # next to the column maximum the corrected code is still within [-r, r]
    assert oracle.bdr_adjust(126, 126.4, 126.3, m, 8, mode) == 127


def _one_step_f64(st, inp, b, h):
    """Full-precision update of the previous dequantized state, in float64 (the
    gated delta rule written out: S = alpha S^ + k (beta (v - alpha S^T k))^T)."""
    Sh = (st["codes"][b, h].astype(np.float64) * st["scales"][b, h].astype(np.float64))
    k = oracle.widen(inp["k"])[b, h].astype(np.float64)
    v = oracle.widen(inp["v"])[b, h].astype(np.float64)
    a, be = float(inp["alpha"][b, h]), float(inp["beta"][b, h])
    w = be * (v - a * (Sh.T @ k))
    return a * Sh + np.outer(k, w), Sh


@pytest.mark.parametrize("base", [oracle.RTN, oracle.SR, oracle.SR8])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_bdr_properties_on_trajectories(base, bits, mode):
    """On free-running trajectories, against the base rounding from the same state:
    (1) scales are unchanged and codes move by at most one step (bounded);
    (2) no element is left moving opposite to its update (checked against a
        float64 update, away from ties);
    (3) where the base rounding had no reversal the code is the base code;
    (4) reversals of the base rounding occur and every one is corrected."""
    w = dataclasses.replace(TINY, B=2, H=2, dk=16, dv=16)
    hb = np.full(w.H, bits, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    n_rev = n_fixed = 0
    for t in range(40):
        inp = W.gdn_inputs(w, t)
        kw = dict(seed=91, step=t, mode=mode)
        nb, _ = oracle.gdn_step(st, inp, hb, rounding=base, **kw)
        nd, _ = oracle.gdn_step(st, inp, hb, rounding=base | oracle.BDR, **kw)
        assert np.array_equal(nb["scales"], nd["scales"])
        dc = nd["codes"].astype(int) - nb["codes"].astype(int)
        assert np.abs(dc).max() <= 1
        for b in range(w.B):
            for h in range(w.H):
                S, prev = _one_step_f64(st, inp, b, h)
                s = nd["scales"][b, h].astype(np.float64)
                scale = np.abs(S).max()
                tol = 1e-5 * max(scale, 1e-30)
                clear = (np.abs(S - prev) > tol)
                up, down = clear & (S > prev), clear & (S < prev)
                base_now = nb["codes"][b, h] * s
                bdr_now = nd["codes"][b, h] * s
                far = lambda now: np.abs(now - prev) > tol
                rev_base = (up & (base_now < prev) & far(base_now)) | (down & (base_now > prev) & far(base_now))
                rev_bdr = (up & (bdr_now < prev) & far(bdr_now)) | (down & (bdr_now > prev) & far(bdr_now))
                assert not rev_bdr.any()
                ok_base = clear & ~rev_base & ~(np.abs(base_now - prev) <= tol)
                assert np.array_equal(nd["codes"][b, h][ok_base], nb["codes"][b, h][ok_base])
                n_rev += int(rev_base.sum())
                n_fixed += int((rev_base & (dc[b, h] != 0)).sum())
        st = nd
    assert n_rev > 0 and n_fixed == n_rev


# ---------------------------------------------------------------------------
# Diagonal-decay recurrences of the mixer zoo (LoReS Table 1: GLA, KDA)
# ---------------------------------------------------------------------------
TINY_GLA = dataclasses.replace(W.BY_NAME["gla_b64_h16_d128_int8_sr"], B=1, H=2, dk=16, dv=16,
                               in_dtype="f32")
TINY_KDA = dataclasses.replace(W.BY_NAME["kda_b64_h16_d128_int8_sr"], B=1, H=2, dk=16, dv=16,
                               in_dtype="f32")


def _gla_closed_form(ins, t_end, b, h):
    """S_t = sum_tau diag(prod_{s=tau+1..t} alpha_s) k_tau v_tau^T (cumulative decay products)."""
    S = 0.0
    for tau in range(t_end):
        decay = np.ones(ins[0]["alpha"].shape[-1])
        for s in range(tau + 1, t_end):
            decay *= np.asarray(ins[s]["alpha"][b, h], np.float64)
        S = S + np.outer(decay * np.asarray(ins[tau]["k"][b, h], np.float64),
                         np.asarray(ins[tau]["v"][b, h], np.float64))
    return S


def _kda_closed_form(ins, t_end, b, h):
    """S_t = sum_tau [prod_{s=tau+1..t} (I - beta_s k_s k_s^T) diag(alpha_s)] beta_tau k_tau v_tau^T."""
    S = 0.0
    for tau in range(t_end):
        k0 = np.asarray(ins[tau]["k"][b, h], np.float64)
        M = float(ins[tau]["beta"][b, h]) * np.outer(k0, np.asarray(ins[tau]["v"][b, h], np.float64))
        for s in range(tau + 1, t_end):
            a = np.asarray(ins[s]["alpha"][b, h], np.float64)
            ks = np.asarray(ins[s]["k"][b, h], np.float64)
            Dm = a[:, None] * M
            M = Dm - float(ins[s]["beta"][b, h]) * np.outer(ks, ks @ Dm)
        S = S + M
    return S


@pytest.mark.parametrize("family", ["gla", "kda"])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_diag_decay_fp32_state_matches_closed_form(family, mode):
    """(a) for the diagonal-decay mixers: with quantization disabled the state and
    readout equal the unrolled sums of decayed outer products."""
    w = TINY_GLA if family == "gla" else TINY_KDA
    step = oracle.gla_step if family == "gla" else oracle.kda_step
    close = _gla_closed_form if family == "gla" else _kda_closed_form
    T = 48
    ins = [W.inputs(w, t) for t in range(T)]
    hb = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    for t in range(T):
        st, o = step(st, ins[t], hb, rounding=0, seed=0, step=t, mode=mode)
        if (t + 1) % 8 == 0:
            for h in range(w.H):
                ref = close(ins, t + 1, 0, h)
                assert _rel(st["f"][0, h], ref) <= 1e-5
                assert _rel(o[0, h], ref.T @ np.asarray(ins[t]["q"][0, h], np.float64)) <= 1e-5


def test_gla_constant_decay_is_the_scalar_decay_step():
    """GLA with the same decay on every key channel is RetNet's recurrence, i.e.
    the Mamba-2 step with B = k, C = q, x = v, dt = 1, decay = gamma and D = 0:
    both evaluation orders reduce to the same operations, state for state."""
    w = dataclasses.replace(TINY_GLA, B=2, H=3)
    hb = np.array([8, 4, 32], np.int8)
    a = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    m = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    for t in range(12):
        inp = W.inputs(w, t)
        gamma = inp["alpha"][:, :, 0].copy()
        inp["alpha"] = np.repeat(gamma[:, :, None], w.dk, axis=2)
        a, o_a = oracle.gla_step(a, inp, hb, rounding=oracle.SR, seed=5, step=t)
        mi = {"x": inp["v"], "Bm": inp["k"], "Cm": inp["q"], "dt": np.ones((w.B, w.H), np.float32),
              "A": np.zeros(w.H, np.float32), "D": np.zeros(w.H, np.float32)}
        m, o_m = oracle.mamba2_step(m, mi, hb, rounding=oracle.SR, seed=5, step=t, ngroups=w.H,
                                    decay=gamma)
        assert np.array_equal(a["codes"], m["codes"]) and np.array_equal(a["scales"], m["scales"])
        assert np.array_equal(a["f"], m["f"]) and np.array_equal(o_a, o_m)


# ---------------------------------------------------------------------------
# Copy scale (LoReS (4/4), animation details: the scale taken from an
# unquantized copy of the state; "When Dynamic Scaling Fails", key points: the
# dynamic scale feeds back on the state it is derived from)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rounding", [oracle.RTN, oracle.SR, oracle.SR8])
@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_copy_scale_equal_to_own_maximum_is_the_noisy_quantizer(rounding, mode):
    rng = np.random.default_rng(3)
    S = (rng.standard_normal((2, 3, 16, 32)) * 0.3).astype(np.float32)
    hb = np.array([8, 4, 8], np.int8)
    own = np.abs(S).max(axis=2)                      # exact column maxima
    a = oracle.quantize(S, hb, rounding=rounding, seed=4, step=2, mode=mode)
    b = oracle.quantize(S, hb, rounding=rounding, seed=4, step=2, mode=mode, copy_absmax=own)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


@pytest.mark.parametrize("bits", [8, 4])
def test_copy_scale_clips_beyond_the_copy_maximum(bits):
    """A copy maximum below the column's own: elements beyond it clip to +-r, the
    others keep the half-step bound of nearest rounding."""
    rng = np.random.default_rng(bits)
    S = rng.standard_normal((1, 2, 32, 16)).astype(np.float32)
    hb = np.full(2, bits, np.int8)
    mc = (np.abs(S).max(axis=2) * 0.5).astype(np.float32)
    st = oracle.quantize(S, hb, rounding=oracle.RTN, seed=0, step=0, copy_absmax=mc)
    r = oracle.rmax(bits)
    s = st["scales"].astype(np.float64)[:, :, None, :]
    c = st["codes"].astype(np.float64)
    assert np.abs(c).max() == r
    inside = np.abs(S) <= mc[:, :, None, :]
    err = np.abs(c * s - S)
    assert np.all(err[inside] <= (s / 2 * (1 + 1e-6) + 0 * err)[inside])
    assert np.array_equal(c[~inside], r * np.sign(S[~inside]))


def test_copy_scale_removes_the_error_dependence_of_the_scale():
    """With the copy scale the scales follow the unquantized trajectory whatever
    the rounding draws; with the state's own (noisy) scale they do not."""
    w = dataclasses.replace(TINY, B=1, H=2)
    hb4 = np.full(w.H, 4, np.int8)
    hb32 = np.full(w.H, 32, np.int8)
    ref = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    cp = {s: oracle.zero_state(w.B, w.H, w.dk, w.dv) for s in (1, 2)}
    ny = {s: oracle.zero_state(w.B, w.H, w.dk, w.dv) for s in (1, 2)}
    noisy_differ = False
    for t in range(24):
        inp = W.gdn_inputs(w, t)
        ref, _ = oracle.gdn_step(ref, inp, hb32, rounding=0, seed=0, step=t)
        m = np.abs(ref["f"]).max(axis=2)
        for seed in (1, 2):
            cp[seed], _ = oracle.gdn_step(cp[seed], inp, hb4, rounding=oracle.SR, seed=seed, step=t,
                                          copy_absmax=m)
            ny[seed], _ = oracle.gdn_step(ny[seed], inp, hb4, rounding=oracle.SR, seed=seed, step=t)
        assert np.array_equal(cp[1]["scales"], cp[2]["scales"])
        assert np.array_equal(cp[1]["scales"], (m / np.float32(7)).astype(np.float32))
        noisy_differ |= not np.array_equal(ny[1]["scales"], ny[2]["scales"])
    assert noisy_differ


# ---------------------------------------------------------------------------
# Pure-write window ("Low-Bit GDN Recurrent-State Quantization: ... Pure-Write
# Sliding Windows", abstract) and its FP8 E4M3 vectors
# ---------------------------------------------------------------------------
def test_e4m3_decode_table_matches_torch():
    """All 256 codes against PyTorch's float8_e4m3fn (an independent implementation)."""
    import torch
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float32)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.array_equal(ref[~np.isnan(ref)], got[~np.isnan(got)])


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    """Round to nearest even against PyTorch on random values, every tie between
    neighbouring codes and the subnormal range; beyond 448 the codec saturates."""
    import torch
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(4000) * 30, rng.uniform(-0.02, 0.02, 2000),
                        rng.uniform(-463.9, 463.9, 2000)]).astype(np.float32)
    vals = np.array([oracle.e4m3_decode(c) for c in range(127)], np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)          # exact ties (binary32 holds them)
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], np.uint8)
    assert np.array_equal(ref, got)
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-500.0) == 0xFE


@pytest.mark.parametrize("W", [4, 8])
def test_pure_write_window_decomposition_is_exact(W):
    """With binary32 vectors and history, H + sum_w a_w b_w^T is the Gated DeltaNet
    state (closed form in float64) at every step, before and after slots start to
    merge, and the readout is S_t^T q."""
    w = TINY
    T = 3 * W + 5
    ins = [W_inputs for W_inputs in (W_mod.gdn_inputs(w, t) for t in range(T))]
    hb = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    win = oracle.zero_window(w.B, w.H, W, w.dk, w.dv, fp32=True)
    for t in range(T):
        st, win, o = oracle.gdn_pw_step(st, win, ins[t], hb, rounding=0, seed=0, step=t,
                                        fp32window=True)
        full = oracle.window_full_state(st, win, hb, fp32window=True)
        for h in range(w.H):
            ref = _gdn_closed_form(ins, t + 1, 0, h)
            assert _rel(full[0, h], ref) <= 1e-5
            assert _rel(o[0, h], ref.T @ np.asarray(ins[t]["q"][0, h], np.float64)) <= 1e-5


def test_pure_write_window_fp8_error_is_bounded():
    """FP8 vectors (3 mantissa bits, one scale per vector) keep the full state
    within a few percent of the exact one."""
    w = TINY
    T, W = 40, 8
    ins = [W_mod.gdn_inputs(w, t) for t in range(T)]
    hb = np.full(w.H, 32, np.int8)
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    win = oracle.zero_window(w.B, w.H, W, w.dk, w.dv)
    for t in range(T):
        st, win, _ = oracle.gdn_pw_step(st, win, ins[t], hb, rounding=0, seed=0, step=t)
    full = oracle.window_full_state(st, win, hb)
    for h in range(w.H):
        assert _rel(full[0, h], _gdn_closed_form(ins, T, 0, h)) <= 0.08


# ---------------------------------------------------------------------------
# Key-axis scale groups (LoReS (1/4) Scale grouping: the alternative grouping,
# one scale per key row)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [8, 4])
def test_key_axis_quantizer_is_the_value_axis_quantizer_transposed(bits):
    """Rows of S grouped by key are the columns of S^T: nearest rounding of S with
    key-axis scales equals the (pinned) value-axis quantizer applied to S^T."""
    rng = np.random.default_rng(bits + 1)
    S = rng.standard_normal((2, 3, 32, 48)).astype(np.float32)
    hb = np.full(3, bits, np.int8)
    ka = oracle.quantize_ka(S, hb, rounding=oracle.RTN, seed=0, step=0)
    va = oracle.quantize(np.ascontiguousarray(S.transpose(0, 1, 3, 2)), hb, rounding=oracle.RTN, seed=0,
                         step=0)
    assert np.array_equal(ka["codes"], va["codes"].transpose(0, 1, 3, 2))
    assert np.array_equal(ka["scales"], va["scales"])


@pytest.mark.parametrize("mode", [oracle.PLAIN, oracle.CANONICAL])
def test_key_axis_first_step_rank_one_codes(mode):
    """From S_0 = 0, S_1 = beta k v^T: every row's codes are round(r * v_j *
    sign(k_i) / max|v|) and its scale beta |k_i| max|v| / r."""
    w = TINY
    inp = W.gdn_inputs(w, 0)
    hb = np.full(w.H, 8, np.int8)
    st1, o = oracle.gdn_ka_step(oracle.zero_state_ka(w.B, w.H, w.dk, w.dv), inp, hb, rounding=oracle.RTN,
                                seed=0, step=0, mode=mode)
    for h in range(w.H):
        k = inp["k"][0, h].astype(np.float64)
        v = inp["v"][0, h].astype(np.float64)
        beta = float(inp["beta"][0, h])
        expect = 127 * np.outer(np.sign(k), v) / np.abs(v).max()
        assert np.all(np.abs(st1["codes"][0, h] - expect) <= 0.5 + 1e-4)
        assert np.allclose(st1["scales"][0, h], beta * np.abs(k) * np.abs(v).max() / 127, rtol=1e-5)
        assert np.allclose(o[0, h], beta * float(k @ inp["q"][0, h]) * v, rtol=1e-5, atol=1e-6)


def test_key_axis_readout_error_variance():
    """With key-axis groups the readout error of column j mixes the row scales:
    E[e_j^2] = sum_i q_i^2 s_i^2 / 12 under uniform rounding error (within 10%) --
    the quantity the value-axis proposition of (1/4) compares against."""
    rng = np.random.default_rng(43)
    ratios = []
    for rep in range(40):
        S = rng.standard_normal((1, 1, 64, 64)).astype(np.float32)
        st = oracle.quantize_ka(S, np.array([8], np.int8), rounding=oracle.RTN, seed=0, step=0)
        E = (oracle.dequantize_ka(st) - S)[0, 0].astype(np.float64)
        q = rng.standard_normal((64, 64))
        q /= np.linalg.norm(q, axis=0, keepdims=True)
        e = E.T @ q                                          # e[j, n] = sum_i E_ij q_in
        s = st["scales"][0, 0].astype(np.float64)
        pred = (q ** 2 * (s ** 2)[:, None]).sum(axis=0) / 12  # per query n
        ratios.append(np.mean(e ** 2, axis=0) / pred)
    assert abs(np.mean(ratios) - 1.0) <= 0.10


def test_key_axis_step_plain_and_canonical_agree():
    """The literal and the canonical evaluation order of the key-axis step differ
    only by rounding: codes within one step, readouts within 1e-5 relative."""
    w = dataclasses.replace(TINY, B=2, H=2)
    hb = np.full(w.H, 8, np.int8)
    rng = np.random.default_rng(9)
    st = oracle.quantize_ka((rng.standard_normal((2, 2, 16, 16)) * 0.3).astype(np.float32), hb,
                            rounding=oracle.RTN, seed=0, step=0)
    for t in range(8):
        inp = W.gdn_inputs(w, t)
        a, oa = oracle.gdn_ka_step(st, inp, hb, rounding=oracle.SR, seed=3, step=t, mode=oracle.CANONICAL)
        b, ob = oracle.gdn_ka_step(st, inp, hb, rounding=oracle.SR, seed=3, step=t, mode=oracle.PLAIN)
        assert np.abs(a["codes"].astype(int) - b["codes"].astype(int)).max() <= 1
        assert _rel(oa, ob) <= 1e-5
        st = a
