"""Seeded synthetic workloads for the quantized recurrent-state decode step.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds ONLY workload definitions and seeded input generation (normal draws,
L2 normalisation, sigmoid/softplus gates, bf16 rounding of the drawn values).
It contains none of the decode method's arithmetic: no dequantisation, no
recurrence, no readout, no scale computation, no rounding of the state.

Input distributions follow the five workloads the method is evaluated on:

* Gated DeltaNet: q, k ~ N(0, 1) then L2-normalised over the key axis,
  v ~ N(0, 1), alpha = sigmoid(N(3, 1)), beta = sigmoid(N(0, 1)).
* Mamba-2: A_h = -exp(U(0, 2.8)), dt = softplus(N(-2, 1)), x, B, C ~ N(0, 1),
  D_h ~ N(1, 0.1).
* GLA / KDA (diagonal decay): q, k, v as for Gated DeltaNet, a decay per key
  channel alpha_i = sigmoid(N(3, 1)) (the GDN gate law per channel), and for
  KDA beta = sigmoid(N(0, 1)).

Every quantity of every decode step is drawn from its own numpy stream keyed
on (input_seed, step, quantity), so any step can be regenerated alone and any
slice of heads taken from it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Stream identifiers: one independent numpy stream per drawn quantity.
_Q, _K, _V, _ALPHA, _BETA, _X, _BMAT, _CMAT, _DT, _STATIC = range(10)


@dataclass(frozen=True)
class Workload:
    """One decode workload: family, shapes, horizon, state format, input law."""

    name: str
    family: str          # "gdn", "mamba2", "gla" or "kda"
    B: int               # batch (independent requests)
    H: int               # heads
    dk: int              # GDN key dim d_k; Mamba-2 state dim N (rows of the stored state)
    dv: int              # GDN value dim d_v; Mamba-2 head dim P (columns; one scale each)
    steps: int           # decode horizon
    state: str           # "int8", "int4", "mixed" (25% int8 + 75% int4 by decay), "fp32"
    rounding: str        # "rtn" or "sr"
    in_dtype: str        # "f32" or "bf16" for q/k/v (GDN) and x/B/C (Mamba-2)
    input_seed: int
    sr_seed: int
    ngroups: int = 1     # Mamba-2 B/C groups
    high_frac: float = 0.25  # mixed: fraction of heads kept at 8 bits
    notes: str = field(default="", compare=False)

    @property
    def head_updates_per_step(self) -> int:
        return self.B * self.H


# The five evaluation workloads (index 0 is the small exact-parity case).
WORKLOADS = [
    Workload("gdn_b1_h2_d16_int8_rtn", "gdn", 1, 2, 16, 16, 64, "int8", "rtn", "f32",
             input_seed=0, sr_seed=1000),
    Workload("gdn_b64_h16_d128_int8_sr", "gdn", 64, 16, 128, 128, 1024, "int8", "sr", "bf16",
             input_seed=1, sr_seed=1001),
    Workload("gdn_b256_h32_d128_mixed_sr", "gdn", 256, 32, 128, 128, 256, "mixed", "sr", "bf16",
             input_seed=2, sr_seed=1002),
    Workload("mamba2_b128_h80_p64_n128_int8_sr", "mamba2", 128, 80, 128, 64, 512, "int8", "sr",
             "bf16", input_seed=3, sr_seed=1003),
    Workload("gdn_b1024_h16_d128_int4_sr_long", "gdn", 1024, 16, 128, 128, 4096, "int4", "sr",
             "bf16", input_seed=4, sr_seed=1004),
]
# Further recurrence families on the decode shape of the benchmark workload.
EXTRA_WORKLOADS = [
    Workload("gla_b64_h16_d128_int8_sr", "gla", 64, 16, 128, 128, 1024, "int8", "sr", "bf16",
             input_seed=5, sr_seed=1005),
    Workload("kda_b64_h16_d128_int8_sr", "kda", 64, 16, 128, 128, 1024, "int8", "sr", "bf16",
             input_seed=6, sr_seed=1006),
    # d_k = 256 (two warps per block): Gated DeltaNet with 256-wide heads, and
    # Mamba-2 with a 256-wide SSM state (N = 256)
    Workload("gdn_b64_h8_d256_int8_sr", "gdn", 64, 8, 256, 256, 1024, "int8", "sr", "bf16",
             input_seed=7, sr_seed=1007),
    Workload("mamba2_b128_h80_p64_n256_int8_sr", "mamba2", 128, 80, 256, 64, 512, "int8", "sr",
             "bf16", input_seed=8, sr_seed=1008),
]
BY_NAME = {w.name: w for w in WORKLOADS + EXTRA_WORKLOADS}


def _rng(seed: int, step: int, qty: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(step), int(qty)])


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


def _softplus(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float64)
    return (np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))).astype(np.float32)


def _l2_normalise(z: np.ndarray) -> np.ndarray:
    z64 = z.astype(np.float64)
    return (z64 / np.linalg.norm(z64, axis=-1, keepdims=True)).astype(np.float32)


def _vec(w: Workload, x: np.ndarray):
    """Return the vector input in the workload's storage dtype (float32 or bf16 bits)."""
    if w.in_dtype == "bf16":
        return bf16_bits(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def gdn_inputs(w: Workload, step: int, B: int | None = None) -> dict:
    """Inputs of one Gated DeltaNet decode step.

    Returns q, k: [B][H][dk], v: [B][H][dv] (float32 or bf16 bits), alpha, beta: [B][H] float32.
    ``B`` may be smaller than the workload's batch to draw only the leading requests
    (the draws of the first B rows are identical to those of the full batch).
    """
    assert w.family == "gdn"
    B = w.B if B is None else B
    s = w.input_seed
    q = _rng(s, step, _Q).standard_normal((w.B, w.H, w.dk), dtype=np.float32)[:B]
    k = _rng(s, step, _K).standard_normal((w.B, w.H, w.dk), dtype=np.float32)[:B]
    v = _rng(s, step, _V).standard_normal((w.B, w.H, w.dv), dtype=np.float32)[:B]
    alpha = _sigmoid(_rng(s, step, _ALPHA).normal(3.0, 1.0, (w.B, w.H)))[:B]
    beta = _sigmoid(_rng(s, step, _BETA).normal(0.0, 1.0, (w.B, w.H)))[:B]
    return {
        "q": _vec(w, _l2_normalise(q)),
        "k": _vec(w, _l2_normalise(k)),
        "v": _vec(w, v),
        "alpha": np.ascontiguousarray(alpha),
        "beta": np.ascontiguousarray(beta),
    }


def diag_inputs(w: Workload, step: int, B: int | None = None) -> dict:
    """Inputs of one GLA / KDA decode step: q, k: [B][H][dk], v: [B][H][dv]
    (float32 or bf16 bits), alpha: [B][H][dk] float32 (decay per key channel),
    beta: [B][H] float32 (KDA only)."""
    assert w.family in ("gla", "kda")
    B = w.B if B is None else B
    s = w.input_seed
    q = _rng(s, step, _Q).standard_normal((w.B, w.H, w.dk), dtype=np.float32)[:B]
    k = _rng(s, step, _K).standard_normal((w.B, w.H, w.dk), dtype=np.float32)[:B]
    v = _rng(s, step, _V).standard_normal((w.B, w.H, w.dv), dtype=np.float32)[:B]
    alpha = _sigmoid(_rng(s, step, _ALPHA).normal(3.0, 1.0, (w.B, w.H, w.dk)))[:B]
    out = {"q": _vec(w, _l2_normalise(q)), "k": _vec(w, _l2_normalise(k)), "v": _vec(w, v),
           "alpha": np.ascontiguousarray(alpha)}
    if w.family == "kda":
        out["beta"] = np.ascontiguousarray(_sigmoid(_rng(s, step, _BETA).normal(0.0, 1.0, (w.B, w.H)))[:B])
    return out


def gdn_alpha(w: Workload, step: int) -> np.ndarray:
    """Only the alpha gates of one GDN step ([B][H] float32), same values as gdn_inputs."""
    return _sigmoid(_rng(w.input_seed, step, _ALPHA).normal(3.0, 1.0, (w.B, w.H)))


def mamba2_static(w: Workload) -> dict:
    """Per-head constants of a Mamba-2 workload: A_h = -exp(U(0, 2.8)), D_h ~ N(1, 0.1)."""
    assert w.family == "mamba2"
    g = _rng(w.input_seed, 0, _STATIC)
    A = (-np.exp(g.uniform(0.0, 2.8, w.H))).astype(np.float32)
    D = g.normal(1.0, 0.1, w.H).astype(np.float32)
    return {"A": A, "D": D}


def mamba2_inputs(w: Workload, step: int, B: int | None = None) -> dict:
    """Inputs of one Mamba-2 decode step.

    Returns x: [B][H][P], Bm, Cm: [B][G][N] (float32 or bf16 bits), dt: [B][H] float32,
    plus the static A, D: [H] float32.
    """
    assert w.family == "mamba2"
    B = w.B if B is None else B
    s = w.input_seed
    x = _rng(s, step, _X).standard_normal((w.B, w.H, w.dv), dtype=np.float32)[:B]
    Bm = _rng(s, step, _BMAT).standard_normal((w.B, w.ngroups, w.dk), dtype=np.float32)[:B]
    Cm = _rng(s, step, _CMAT).standard_normal((w.B, w.ngroups, w.dk), dtype=np.float32)[:B]
    dt = _softplus(_rng(s, step, _DT).normal(-2.0, 1.0, (w.B, w.H)))[:B]
    out = {"x": _vec(w, x), "Bm": _vec(w, Bm), "Cm": _vec(w, Cm), "dt": np.ascontiguousarray(dt)}
    out.update(mamba2_static(w))
    return out


def inputs(w: Workload, step: int, B: int | None = None) -> dict:
    if w.family == "gdn":
        return gdn_inputs(w, step, B)
    if w.family == "mamba2":
        return mamba2_inputs(w, step, B)
    return diag_inputs(w, step, B)


def mean_alpha_per_head(w: Workload, steps: int | None = None) -> np.ndarray:
    """Mean of the generated alpha gates over all requests and steps, per head ([H] float64).

    This is the decay statistic a mixed-precision allocation ranks heads by.
    """
    steps = w.steps if steps is None else steps
    acc = np.zeros(w.H, dtype=np.float64)
    for t in range(steps):
        acc += gdn_alpha(w, t).astype(np.float64).sum(axis=0)
    return acc / (steps * w.B)


def head_bits_for(w: Workload, bits_map: np.ndarray | None = None) -> np.ndarray:
    """Per-head bit widths for a workload whose state format is uniform (int8/int4/fp32).

    Mixed workloads need an allocation (computed by the library or the oracle from
    ``mean_alpha_per_head``) and must pass it as ``bits_map``.
    """
    if w.state == "mixed":
        assert bits_map is not None, "mixed precision needs an allocation"
        return np.asarray(bits_map, dtype=np.int8)
    width = {"int8": 8, "int4": 4, "fp32": 32}[w.state]
    return np.full(w.H, width, dtype=np.int8)
