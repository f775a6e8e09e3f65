"""Comparison with the oracle's literal evaluation order at the method's tolerance.

The oracle's plain mode evaluates the definitions as written ("Quantizing
Recurrent Language Models Is Easier Than You Think", "(1/4) Scale grouping":
s = max|S| / r, codes round(S / s); "(3/4) Rounding": floor(S / s + u)).  The
library and the oracle's canonical mode evaluate the same mathematics in a
fixed binary32 order of their own.  Two orders give codes that differ where
the full-precision value lies within a rounding error of a decision boundary:
at most 1e-5 of the codes, each by one step, is the parity bar.

Nearest rounding has boundary cases that are not generic rounding noise: an
element whose value is a half-integer number of steps (S * r = (n + 1/2) * m,
m the column maximum), exactly or to within the rounding of the products
that formed it.  bf16 inputs make these common at x = r / 2: an element half
its column's maximum, e.g. two keys whose bf16 values differ by a factor of
two; from a zero state the first update is rank one (S = k w^T), so such a
pair puts every column of the head on the boundary at once.  The literal
order decides them through the roundings of its float scale and quotient, the
canonical order (its multiplier r / m rounded toward zero) toward zero.
Differences within a few ulps of x = n + 1/2 are counted separately and are
not held to the 1e-5 bar.

Test code only: imports the oracle, never the library.
"""
from __future__ import annotations

import numpy as np

import oracle


def literal_state(family: str, st: dict, inp: dict, head_bits, *, ngroups: int = 1,
                  decay=None) -> np.ndarray:
    """Full-precision S_t of the literal order from the quantized state ``st``:
    the 32-bit-state step (plain mode) of the dequantized state, which is the
    literal order's own update before its quantizer.  float32 [B][H][dk][dv]."""
    B, H, dk, dv = st["codes"].shape
    f = oracle.zero_state(B, H, dk, dv, fp32=True)
    f["f"] = oracle.dequantize(st, head_bits)
    b32 = np.full(H, 32, np.int8)
    if family == "gdn":
        out, _ = oracle.gdn_step(f, inp, b32, rounding=oracle.RTN, seed=0, step=0, mode=oracle.PLAIN)
    elif family == "mamba2":
        out, _ = oracle.mamba2_step(f, inp, b32, rounding=oracle.RTN, seed=0, step=0, mode=oracle.PLAIN,
                                    ngroups=ngroups, decay=decay)
    elif family in ("gla", "kda"):
        step = oracle.gla_step if family == "gla" else oracle.kda_step
        out, _ = step(f, inp, b32, rounding=oracle.RTN, seed=0, step=0, mode=oracle.PLAIN)
    else:
        raise ValueError(family)
    return out["f"]


def compare_codes(codes: np.ndarray, plain_codes: np.ndarray, S_lit: np.ndarray, head_bits,
                  heads=None, nearest: bool = True) -> tuple[int, int, int]:
    """Codes of another order against the literal order's codes, per (b, h) in
    ``heads`` (default all).  Asserts every difference is one step.  Returns
    (differences away from nearest-rounding boundary cases, differences at
    them, codes compared): a boundary case is an element whose literal value
    x = S * r / m lies within 2^-19 |x| of the half-integer between the two
    codes (a few ulps of binary32).  With ``nearest`` False (stochastic
    rounding) every difference counts."""
    B, H = codes.shape[:2]
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    n_other = n_tie = n_tot = 0
    for b, h in pairs:
        bits = int(head_bits[h])
        if bits == 32:
            continue
        r = float((1 << (bits - 1)) - 1)
        a = codes[b, h].astype(np.int64)
        p = plain_codes[b, h].astype(np.int64)
        d = a != p
        n_tot += d.size
        if not d.any():
            continue
        assert np.abs(a - p).max() <= 1, "codes (%d,%d) differ by more than one step" % (b, h)
        S = S_lit[b, h].astype(np.float64)
        m = np.abs(S).max(axis=0, keepdims=True)          # column maxima (exact)
        half = np.minimum(a, p).astype(np.float64) + 0.5
        # S*r and half*m are exact in binary64 (31 and 33 significant bits)
        tie = (np.abs(S * r - half * m) <= 2.0 ** -19 * np.abs(half) * m) if nearest else np.zeros_like(d)
        n_tie += int((d & tie).sum())
        n_other += int((d & ~tie).sum())
    return n_other, n_tie, n_tot


def max_rel(a: np.ndarray, ref: np.ndarray, heads=None) -> float:
    """max |a - ref| / max |ref| over each head's vector (normwise max relative error)."""
    B, H = ref.shape[:2]
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    worst = 0.0
    for b, h in pairs:
        den = float(np.max(np.abs(ref[b, h])))
        if den == 0.0:
            assert float(np.max(np.abs(a[b, h]))) == 0.0
            continue
        worst = max(worst, float(np.max(np.abs(a[b, h].astype(np.float64) - ref[b, h]))) / den)
    return worst
