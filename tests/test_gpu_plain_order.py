"""GPU parity against the oracle's literal evaluation order at the method's tolerance.

Every benchmark workload and both code widths: each step the GPU and the
literal-order oracle start from the same state (the canonical oracle's, which
the GPU matches bit for bit), and
  * at most 1e-5 of the codes differ from the literal order's, each by one
    step, apart from exact ties of nearest rounding (tests/plain_order.py);
  * scales agree to 1e-5 relative, and the dequantized state of every code that
    agrees, and the outputs, to 1e-3 normwise relative (max |a - b| / max |b|
    per head vector).
Definitions: "Quantizing Recurrent Language Models Is Easier Than You Think",
"(1/4) Scale grouping" (s = max|S| / r, codes round(S / s)) and "(3/4)
Rounding" (stochastic rounding); the recurrences of "Preserving Updates in
Low-Bit Recurrent State Quantization", abstract.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
import plain_order
from gpu_harness import Run, assert_out_equal, assert_state_equal, bits_for

pytestmark = pytest.mark.gpu

WL = W.WORKLOADS


def _decay(inp):
    return np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)


def _against_plain(run: Run, steps: int, decay_override: bool = True, bit_exact: bool = True):
    """Teacher-forced: every step starts both sides from the canonical oracle's
    state.  Returns (codes differing away from ties, at ties, codes compared)."""
    family = {rsq.RSQ_GDN: "gdn", rsq.RSQ_MAMBA2: "mamba2", rsq.RSQ_GLA: "gla", rsq.RSQ_KDA: "kda"}[run.family]
    nearest = (run.rounding & rsq.RSQ_SR) == 0   # nearest rounding, with or without BDR
    st = run.zero()
    n_other = n_tie = n_tot = 0
    for t in range(steps):
        inp = run.inputs(t)
        decay = _decay(inp) if (family == "mamba2" and decay_override) else None
        g_in, g_out = run.upload(st), run.upload(st)
        out = run.gpu_step(g_in, g_out, inp, t, decay=decay)
        gpu = run.download(g_out)
        canon, canon_out = run.oracle_step(st, inp, t, decay=decay)
        if bit_exact:
            assert_state_equal(gpu, canon, run.head_bits, what="step %d" % t)
            assert_out_equal(out, canon_out, what="step %d" % t)
        plain, plain_out = run.oracle_step(st, inp, t, mode=oracle.PLAIN, decay=decay)
        S_lit = plain_order.literal_state(family, st, inp, run.head_bits, ngroups=run.w.ngroups, decay=decay)
        o, ti, tot = plain_order.compare_codes(gpu["codes"], plain["codes"], S_lit, run.head_bits,
                                               nearest=nearest)
        n_other, n_tie, n_tot = n_other + o, n_tie + ti, n_tot + tot
        assert np.allclose(gpu["scales"], plain["scales"], rtol=1e-5, atol=0)
        assert plain_order.max_rel(out, plain_out) <= 1e-3
        # dequantized state wherever the codes agree
        same = gpu["codes"] == plain["codes"]
        dg = np.where(same, oracle.dequantize(gpu, run.head_bits), 0.0)
        dp = np.where(same, oracle.dequantize(plain, run.head_bits), 0.0)
        cols = np.abs(oracle.dequantize(plain, run.head_bits)).max(axis=2, keepdims=True)
        cols[cols == 0] = 1.0
        assert np.max(np.abs(dg - dp) / cols) <= 1e-3
        st = canon
    return n_other, n_tie, n_tot


def _check(res):
    n_other, n_tie, n_tot = res
    assert n_tot > 0
    assert n_other <= 1e-5 * n_tot, res
    assert n_tie <= 1e-3 * n_tot, res


def test_gdn_int8_sr_plain():
    """Gated DeltaNet, INT8, stochastic rounding, bf16 inputs (the B=64 workload's head shape)."""
    w = WL[1]
    _check(_against_plain(Run(w, bits_for(w), B=8), 6))


def test_gdn_mixed_sr_plain():
    """Decay-based mixed precision (8 INT8 + 24 INT4 heads), stochastic rounding."""
    w = WL[2]
    _check(_against_plain(Run(w, bits_for(w), B=4), 5))


@pytest.mark.parametrize("decay_override", [True, False])
def test_mamba2_int8_sr_plain(decay_override):
    """Mamba-2 INT8, stochastic rounding; with the decay passed in, and computed
    by the device's expf (the literal order then uses the host's libm expf, so
    the GPU is compared with the literal order only)."""
    w = WL[3]
    run = Run(w, bits_for(w), B=4)
    _check(_against_plain(run, 5, decay_override=decay_override, bit_exact=decay_override))


def test_gdn_int4_sr_plain():
    """Gated DeltaNet, packed INT4, stochastic rounding (the B=1024 workload's head shape)."""
    w = WL[4]
    _check(_against_plain(Run(w, bits_for(w), B=8), 5))


@pytest.mark.parametrize("bits", [4, 8])
def test_gdn_rtn_plain(bits):
    """Nearest rounding, 4- and 8-bit codes, bf16 inputs."""
    w = dataclasses.replace(WL[1], rounding="rtn")
    _check(_against_plain(Run(w, np.full(w.H, bits, np.int8), B=8), 5))


@pytest.mark.parametrize("bits", [4, 8])
def test_mamba2_rtn_plain(bits):
    w = dataclasses.replace(WL[3], rounding="rtn")
    _check(_against_plain(Run(w, np.full(w.H, bits, np.int8), B=4), 5))


def test_mixed_bit_map_from_the_runs_gates():
    """(2/4) Mixed precision: the oracle's allocation over the gates of the run
    itself (every request and step of this reduced run) equals the library's,
    and the run with that map is bit-exact against the oracle."""
    w = WL[2]
    B, steps = 4, 5
    score = np.zeros(w.H, np.float64)
    for t in range(steps):
        score += W.gdn_inputs(w, t, B=B)["alpha"].astype(np.float64).sum(axis=0)
    score /= B * steps
    n_hi = int(w.H * w.high_frac)
    want = oracle.allocate_bits(score, n_hi)
    got = rsq.rsq_allocate_bits(score, n_hi)
    assert np.array_equal(np.asarray(got, np.int8), want)
    assert (want == 8).sum() == w.H // 4
    run = Run(w, want, B=B)
    st = run.zero()
    g_in, g_out = run.upload(st), run.upload(st)
    for t in range(steps):
        inp = run.inputs(t)
        out = run.gpu_step(g_in, g_out, inp, t)
        st, ref_out = run.oracle_step(st, inp, t)
        assert_state_equal(run.download(g_out), st, run.head_bits, what="step %d" % t)
        assert_out_equal(out, ref_out, what="step %d" % t)
        g_in, g_out = g_out, g_in


@pytest.mark.parametrize("name", ["gla_b64_h16_d128_int8_sr", "kda_b64_h16_d128_int8_sr"], ids=["gla", "kda"])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rounding", ["sr", "rtn"])
def test_diag_families_plain(name, bits, rounding):
    """GLA and KDA (a decay per key channel), 4- and 8-bit codes, stochastic
    (8-bit uniforms) and nearest rounding, bf16 inputs."""
    w = dataclasses.replace(W.BY_NAME[name], rounding=rounding)
    _check(_against_plain(Run(w, np.full(w.H, bits, np.int8), B=8), 4))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rounding", ["sr", "rtn"])
def test_dk256_plain(bits, rounding):
    """d_k = 256 (two warps per block, the 16-partial canonical order), 4- and
    8-bit codes, stochastic (8-bit uniforms) and nearest rounding."""
    w = dataclasses.replace(W.BY_NAME["gdn_b64_h8_d256_int8_sr"], rounding=rounding)
    _check(_against_plain(Run(w, np.full(w.H, bits, np.int8), B=8), 3))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rounding", [rsq.RSQ_BDR, rsq.RSQ_SR8_BDR], ids=["bdr", "sr8_bdr"])
def test_bdr_plain(bits, rounding):
    """Bounded Directional Rounding on nearest and on stochastic rounding (8-bit
    uniforms), 4- and 8-bit codes.  In the literal order the reversal test
    compares c s_new with c_prev s_prev from the float scales and takes ceil or
    floor of S / s; the canonical order uses the multiplier."""
    w = W.WORKLOADS[1]
    _check(_against_plain(Run(w, np.full(w.H, bits, np.int8), B=8, rounding=rounding), 4))
