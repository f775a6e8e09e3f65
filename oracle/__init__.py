"""Python binding of the CPU oracle (ctypes over oracle/librsq_oracle.so).

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm import this package.  It shares no
code with the CUDA library and never imports it.

The oracle works on LOGICAL state arrays:
    codes  int8    [B][H][dk][dv]   symmetric codes c in [-r, r] (4/8-bit heads)
    scales float32 [B][H][dv]       one scale per value column
    f      float32 [B][H][dk][dv]   full-precision state (32-bit heads)
and converts to / from the library's byte format with ``pack_state`` /
``unpack_state`` (written independently from the format's description).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

PLAIN, CANONICAL = 0, 1
RTN, SR = 0, 1
BDR, SR_BDR = 2, 3      # nearest / stochastic base rounding + Bounded Directional Rounding
U8 = 4                  # stochastic rounding with 8-bit uniforms (SR alone: 16-bit uniforms)
SR8, SR8_BDR = SR | U8, SR_BDR | U8


class _Head(ctypes.Structure):
    _fields_ = [("dk", ctypes.c_int), ("dv", ctypes.c_int), ("bits", ctypes.c_int),
                ("rounding", ctypes.c_int), ("mode", ctypes.c_int), ("R", ctypes.c_int),
                ("seed", ctypes.c_uint64), ("b", ctypes.c_uint32), ("h", ctypes.c_uint32),
                ("step", ctypes.c_uint32), ("m_copy", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        # RSQ_ORACLE_LIB selects another build of the same source (the sanitizer build)
        path = os.environ.get("RSQ_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_sr_uniform16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                       ctypes.c_uint32, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_sr_uniform16.restype = ctypes.c_uint32
        L.orc_sr_uniform8.argtypes = L.orc_sr_uniform16.argtypes
        L.orc_sr_uniform8.restype = ctypes.c_uint32
        L.orc_bf16_to_f32.argtypes = [P, P, ctypes.c_int64]
        L.orc_gdn_head_step.argtypes = [ctypes.POINTER(_Head), P, P, P, P, P, P, ctypes.c_float,
                                        ctypes.c_float, P, P, P, P]
        L.orc_gdn_head_step.restype = ctypes.c_int
        L.orc_mamba2_head_step.argtypes = [ctypes.POINTER(_Head), P, P, P, P, P, P, ctypes.c_float,
                                           ctypes.c_float, ctypes.c_float, ctypes.c_float, P, P,
                                           P, P]
        L.orc_mamba2_head_step.restype = ctypes.c_int
        L.orc_diag_head_step.argtypes = [ctypes.POINTER(_Head), ctypes.c_int, P, P, P, P, P, P, P,
                                         ctypes.c_float, P, P, P, P]
        L.orc_diag_head_step.restype = ctypes.c_int
        L.orc_quantize_head.argtypes = [ctypes.POINTER(_Head), P, P, P]
        L.orc_quantize_head.restype = ctypes.c_int
        L.orc_dequantize_head.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
        L.orc_head_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_head_bytes.restype = ctypes.c_int64
        L.orc_pack_head.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        L.orc_unpack_head.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        L.orc_quantize_scalar.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_uint32]
        L.orc_quantize_scalar.restype = ctypes.c_int
        L.orc_bdr_adjust.argtypes = [ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                     ctypes.c_int, ctypes.c_int]
        L.orc_bdr_adjust.restype = ctypes.c_int
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_float
        L.orc_gdn_pw_head_step.argtypes = [ctypes.POINTER(_Head), ctypes.c_int, ctypes.c_int, P, P, P, P,
                                           P, P, P, P, P, P, ctypes.c_float, ctypes.c_float, P, P, P,
                                           P, P, P, P, P]
        L.orc_gdn_pw_head_step.restype = ctypes.c_int
        L.orc_gdn_ka_head_step.argtypes = [ctypes.POINTER(_Head), P, P, P, P, P, ctypes.c_float,
                                           ctypes.c_float, P, P, P]
        L.orc_gdn_ka_head_step.restype = ctypes.c_int
        L.orc_quantize_ka_head.argtypes = [ctypes.POINTER(_Head), P, P, P]
        L.orc_quantize_ka_head.restype = ctypes.c_int
        L.orc_allocate_bits.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# Random numbers
# ---------------------------------------------------------------------------
def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 blocks for counters ``ctr`` [n][4] and keys ``key`` [n][2] (uint32)."""
    ctr = _c(np.atleast_2d(ctr), np.uint32)
    key = _c(np.atleast_2d(key), np.uint32)
    out = np.zeros((ctr.shape[0], 4), dtype=np.uint32)
    L = lib()
    for n in range(ctr.shape[0]):
        c, k, o = ctr[n].copy(), key[n].copy(), np.zeros(4, np.uint32)
        L.orc_philox4x32_10(_p(c), _p(k), _p(o))
        out[n] = o
    return out


def sr_uniform16(seed: int, b: int, h: int, step: int, dk: int, i: int, j: int) -> int:
    return int(lib().orc_sr_uniform16(seed, b, h, step, dk, i, j))


def sr_uniform8(seed: int, b: int, h: int, step: int, dk: int, i: int, j: int) -> int:
    return int(lib().orc_sr_uniform8(seed, b, h, step, dk, i, j))


def quantize_scalar(S: float, m: float, bits: int, rounding: int, mode: int, u: int = 0) -> int:
    """Code of one element S of a column with absolute maximum m (> 0), given its
    uniform u (16 bits wide, or 8 bits when ``rounding`` has the U8 bit)."""
    return int(lib().orc_quantize_scalar(float(S), float(m), int(bits), int(rounding), int(mode),
                                         int(u)))


def bdr_adjust(c: int, S: float, prev: float, m: float, bits: int, mode: int = CANONICAL) -> int:
    """Bounded Directional Rounding of one element: base code c of S (column
    maximum m), previous dequantized value prev."""
    return int(lib().orc_bdr_adjust(int(c), float(S), float(prev), float(m), int(bits), int(mode)))


def widen(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 through the oracle; float32 passes through."""
    if x.dtype == np.uint16:
        src = _c(x, np.uint16)
        dst = np.empty(src.shape, dtype=np.float32)
        lib().orc_bf16_to_f32(_p(src), _p(dst), src.size)
        return dst
    return _c(x, np.float32)


def rmax(bits: int) -> int:
    return (1 << (bits - 1)) - 1


# ---------------------------------------------------------------------------
# State containers
# ---------------------------------------------------------------------------
def zero_state(B: int, H: int, dk: int, dv: int, fp32: bool = True) -> dict:
    """S_0 = 0: all codes 0, all scales 0; the full-precision part (used by 32-bit
    heads) is allocated only when ``fp32``."""
    return {"codes": np.zeros((B, H, dk, dv), np.int8), "scales": np.zeros((B, H, dv), np.float32),
            "f": np.zeros((B, H, dk, dv), np.float32) if fp32 else None}


def copy_state(st: dict) -> dict:
    return {k: (None if v is None else v.copy()) for k, v in st.items()}


def _f_in(state, b, h, dk, dv):
    if state["f"] is None:
        return np.zeros((dk, dv), np.float32)
    return _c(state["f"][b, h], np.float32)


def _head(dk, dv, bits, rounding, mode, R, seed, b, h, step) -> _Head:
    return _Head(dk, dv, int(bits), int(rounding), int(mode), int(R), int(seed) & (2**64 - 1),
                 int(b), int(h), int(step) & 0xFFFFFFFF)


def _heads(B, H, heads):
    return [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)


# ---------------------------------------------------------------------------
# Decode steps
# ---------------------------------------------------------------------------
def gdn_step(state: dict, inp: dict, head_bits, *, rounding: int, seed: int, step: int,
             mode: int = CANONICAL, R: int = 8, heads=None, copy_absmax=None):
    """One Gated DeltaNet decode step over the given (b, h) heads (default: all).

    Returns (new_state, o) with o float32 [B][H][dv]; heads not processed keep
    their old state and a zero output.  ``copy_absmax`` ([B][H][dv] float32)
    switches to the copy scale: the column maxima of an unquantized copy.
    """
    B, H, dk, dv = state["codes"].shape
    q, k, v = widen(inp["q"]), widen(inp["k"]), widen(inp["v"])
    alpha, beta = _c(inp["alpha"], np.float32), _c(inp["beta"], np.float32)
    new = copy_state(state)
    o = np.zeros((B, H, dv), np.float32)
    L = lib()
    for b, h in _heads(B, H, heads):
        bits = int(head_bits[h])
        hd = _head(dk, dv, bits, rounding, mode, R, seed, b, h, step)
        mc = None
        if copy_absmax is not None:
            mc = _c(copy_absmax[b, h], np.float32)
            hd.m_copy = mc.ctypes.data
        c_in, s_in, f_in = (_c(state["codes"][b, h], np.int8), _c(state["scales"][b, h], np.float32),
                            _f_in(state, b, h, dk, dv))
        c_out = np.zeros((dk, dv), np.int8)
        s_out = np.zeros(dv, np.float32)
        f_out = np.zeros((dk, dv), np.float32)
        o_h = np.zeros(dv, np.float32)
        qh, kh, vh = _c(q[b, h], np.float32), _c(k[b, h], np.float32), _c(v[b, h], np.float32)
        rc = L.orc_gdn_head_step(ctypes.byref(hd), _p(c_in), _p(s_in), _p(f_in), _p(qh), _p(kh),
                                 _p(vh), float(alpha[b, h]), float(beta[b, h]), _p(c_out),
                                 _p(s_out), _p(f_out), _p(o_h))
        assert rc == 0
        if bits == 32:
            new["f"][b, h] = f_out
        else:
            new["codes"][b, h] = c_out
            new["scales"][b, h] = s_out
        o[b, h] = o_h
    return new, o


def mamba2_step(state: dict, inp: dict, head_bits, *, rounding: int, seed: int, step: int,
                mode: int = CANONICAL, R: int = 8, ngroups: int = 1, decay=None, heads=None,
                copy_absmax=None):
    """One Mamba-2 decode step.  ``decay`` ([B][H] float32) replaces exp(dt*A) when given."""
    B, H, dk, dv = state["codes"].shape
    x, Bm, Cm = widen(inp["x"]), widen(inp["Bm"]), widen(inp["Cm"])
    dt, A, D = _c(inp["dt"], np.float32), _c(inp["A"], np.float32), _c(inp["D"], np.float32)
    new = copy_state(state)
    y = np.zeros((B, H, dv), np.float32)
    L = lib()
    heads_per_group = H // ngroups
    for b, h in _heads(B, H, heads):
        bits = int(head_bits[h])
        g = h // heads_per_group
        hd = _head(dk, dv, bits, rounding, mode, R, seed, b, h, step)
        mc = None
        if copy_absmax is not None:
            mc = _c(copy_absmax[b, h], np.float32)
            hd.m_copy = mc.ctypes.data
        c_in, s_in, f_in = (_c(state["codes"][b, h], np.int8), _c(state["scales"][b, h], np.float32),
                            _f_in(state, b, h, dk, dv))
        c_out = np.zeros((dk, dv), np.int8)
        s_out = np.zeros(dv, np.float32)
        f_out = np.zeros((dk, dv), np.float32)
        y_h = np.zeros(dv, np.float32)
        xh, bh, ch = _c(x[b, h], np.float32), _c(Bm[b, g], np.float32), _c(Cm[b, g], np.float32)
        dec = -1.0 if decay is None else float(decay[b, h])
        rc = L.orc_mamba2_head_step(ctypes.byref(hd), _p(c_in), _p(s_in), _p(f_in), _p(xh),
                                    _p(bh), _p(ch), float(dt[b, h]), float(A[h]), float(D[h]),
                                    dec, _p(c_out), _p(s_out), _p(f_out), _p(y_h))
        assert rc == 0
        if bits == 32:
            new["f"][b, h] = f_out
        else:
            new["codes"][b, h] = c_out
            new["scales"][b, h] = s_out
        y[b, h] = y_h
    return new, y


def _diag_step(delta: int, state: dict, inp: dict, head_bits, rounding, seed, step, mode, R, heads,
               copy_absmax=None):
    B, H, dk, dv = state["codes"].shape
    q, k, v = widen(inp["q"]), widen(inp["k"]), widen(inp["v"])
    alpha = _c(inp["alpha"], np.float32)            # [B][H][dk]
    beta = _c(inp["beta"], np.float32) if delta else np.zeros((B, H), np.float32)
    new = copy_state(state)
    o = np.zeros((B, H, dv), np.float32)
    L = lib()
    for b, h in _heads(B, H, heads):
        bits = int(head_bits[h])
        hd = _head(dk, dv, bits, rounding, mode, R, seed, b, h, step)
        mc = None
        if copy_absmax is not None:
            mc = _c(copy_absmax[b, h], np.float32)
            hd.m_copy = mc.ctypes.data
        c_in, s_in, f_in = (_c(state["codes"][b, h], np.int8), _c(state["scales"][b, h], np.float32),
                            _f_in(state, b, h, dk, dv))
        c_out = np.zeros((dk, dv), np.int8)
        s_out = np.zeros(dv, np.float32)
        f_out = np.zeros((dk, dv), np.float32)
        o_h = np.zeros(dv, np.float32)
        qh, kh, vh = _c(q[b, h], np.float32), _c(k[b, h], np.float32), _c(v[b, h], np.float32)
        ah = _c(alpha[b, h], np.float32)
        rc = L.orc_diag_head_step(ctypes.byref(hd), int(delta), _p(c_in), _p(s_in), _p(f_in), _p(qh),
                                  _p(kh), _p(vh), _p(ah), float(beta[b, h]), _p(c_out), _p(s_out),
                                  _p(f_out), _p(o_h))
        assert rc == 0
        if bits == 32:
            new["f"][b, h] = f_out
        else:
            new["codes"][b, h] = c_out
            new["scales"][b, h] = s_out
        o[b, h] = o_h
    return new, o


def gla_step(state: dict, inp: dict, head_bits, *, rounding: int, seed: int, step: int,
             mode: int = CANONICAL, R: int = 8, heads=None, copy_absmax=None):
    """One GLA decode step (decay vector alpha [B][H][dk] over the key axis, no delta rule)."""
    return _diag_step(0, state, inp, head_bits, rounding, seed, step, mode, R, heads, copy_absmax)


def kda_step(state: dict, inp: dict, head_bits, *, rounding: int, seed: int, step: int,
             mode: int = CANONICAL, R: int = 8, heads=None, copy_absmax=None):
    """One KDA decode step (delta rule with a decay vector alpha [B][H][dk] and gate beta [B][H])."""
    return _diag_step(1, state, inp, head_bits, rounding, seed, step, mode, R, heads, copy_absmax)


def zero_state_ka(B: int, H: int, dk: int, dv: int) -> dict:
    """S_0 = 0 with key-axis scales: codes [B][H][dk][dv], scales [B][H][dk]."""
    return {"codes": np.zeros((B, H, dk, dv), np.int8), "scales": np.zeros((B, H, dk), np.float32),
            "f": None}


def gdn_ka_step(state: dict, inp: dict, head_bits, *, rounding: int, seed: int, step: int,
                mode: int = CANONICAL, R: int = 8, heads=None):
    """One Gated DeltaNet decode step with key-axis scales (one per row i)."""
    B, H, dk, dv = state["codes"].shape
    q, k, v = widen(inp["q"]), widen(inp["k"]), widen(inp["v"])
    alpha, beta = _c(inp["alpha"], np.float32), _c(inp["beta"], np.float32)
    new = {"codes": state["codes"].copy(), "scales": state["scales"].copy(), "f": None}
    o = np.zeros((B, H, dv), np.float32)
    L = lib()
    for b, h in _heads(B, H, heads):
        hd = _head(dk, dv, int(head_bits[h]), rounding, mode, R, seed, b, h, step)
        c_in, s_in = _c(state["codes"][b, h], np.int8), _c(state["scales"][b, h], np.float32)
        c_out = np.zeros((dk, dv), np.int8)
        s_out = np.zeros(dk, np.float32)
        o_h = np.zeros(dv, np.float32)
        qh, kh, vh = _c(q[b, h], np.float32), _c(k[b, h], np.float32), _c(v[b, h], np.float32)
        assert L.orc_gdn_ka_head_step(ctypes.byref(hd), _p(c_in), _p(s_in), _p(qh), _p(kh), _p(vh),
                                      float(alpha[b, h]), float(beta[b, h]), _p(c_out), _p(s_out),
                                      _p(o_h)) == 0
        new["codes"][b, h], new["scales"][b, h], o[b, h] = c_out, s_out, o_h
    return new, o


def quantize_ka(S: np.ndarray, head_bits, *, rounding: int, seed: int, step: int,
                mode: int = CANONICAL) -> dict:
    """Quantize a full-precision state [B][H][dk][dv] with key-axis scales."""
    B, H, dk, dv = S.shape
    st = zero_state_ka(B, H, dk, dv)
    L = lib()
    for b in range(B):
        for h in range(H):
            hd = _head(dk, dv, int(head_bits[h]), rounding, mode, 1, seed, b, h, step)
            c_out = np.zeros((dk, dv), np.int8)
            s_out = np.zeros(dk, np.float32)
            assert L.orc_quantize_ka_head(ctypes.byref(hd), _p(_c(S[b, h], np.float32)), _p(c_out),
                                          _p(s_out)) == 0
            st["codes"][b, h], st["scales"][b, h] = c_out, s_out
    return st


def dequantize_ka(st: dict) -> np.ndarray:
    """Key-axis state -> float32 [B][H][dk][dv]: c_ij * s_i (binary32 products)."""
    return (st["codes"].astype(np.float32) * st["scales"][..., :, None]).astype(np.float32)


def e4m3_encode(x: float) -> int:
    """FP8 E4M3 code of x (round to nearest even, saturating to +-448)."""
    return int(lib().orc_e4m3_encode(float(x)))


def e4m3_decode(code: int) -> float:
    return float(lib().orc_e4m3_decode(int(code)))


def zero_window(B: int, H: int, W: int, dk: int, dv: int, fp32: bool = False) -> dict:
    """An empty pure-write window (all slots zero): a [B][H][W][dk], b [B][H][W][dv]
    as FP8 codes with scales as [B][H][W], bs [B][H][W] (binary32 vectors when fp32)."""
    t = np.float32 if fp32 else np.uint8
    return {"a": np.zeros((B, H, W, dk), t), "as": np.zeros((B, H, W), np.float32),
            "b": np.zeros((B, H, W, dv), t), "bs": np.zeros((B, H, W), np.float32)}


def gdn_pw_step(state: dict, window: dict, inp: dict, head_bits, *, rounding: int, seed: int,
                step: int, mode: int = CANONICAL, R: int = 8, heads=None, fp32window: bool = False):
    """One Gated DeltaNet decode step with a pure-write window (slot step % W is
    merged into the history and takes the new write).  Returns (state, window, o)."""
    B, H, dk, dv = state["codes"].shape
    W = window["a"].shape[2]
    q, k, v = widen(inp["q"]), widen(inp["k"]), widen(inp["v"])
    alpha, beta = _c(inp["alpha"], np.float32), _c(inp["beta"], np.float32)
    new = copy_state(state)
    win = {key: val.copy() for key, val in window.items()}
    o = np.zeros((B, H, dv), np.float32)
    L = lib()
    vt = np.float32 if fp32window else np.uint8
    for b, h in _heads(B, H, heads):
        bits = int(head_bits[h])
        hd = _head(dk, dv, bits, rounding, mode, R, seed, b, h, step)
        c_in, s_in, f_in = (_c(state["codes"][b, h], np.int8), _c(state["scales"][b, h], np.float32),
                            _f_in(state, b, h, dk, dv))
        a_in, as_in = _c(window["a"][b, h], vt), _c(window["as"][b, h], np.float32)
        b_in, bs_in = _c(window["b"][b, h], vt), _c(window["bs"][b, h], np.float32)
        c_out = np.zeros((dk, dv), np.int8)
        s_out = np.zeros(dv, np.float32)
        f_out = np.zeros((dk, dv), np.float32)
        a_out, as_out = np.zeros_like(a_in), np.zeros_like(as_in)
        b_out, bs_out = np.zeros_like(b_in), np.zeros_like(bs_in)
        o_h = np.zeros(dv, np.float32)
        qh, kh, vh = _c(q[b, h], np.float32), _c(k[b, h], np.float32), _c(v[b, h], np.float32)
        rc = L.orc_gdn_pw_head_step(ctypes.byref(hd), int(W), int(fp32window), _p(c_in), _p(s_in),
                                    _p(f_in), _p(a_in), _p(as_in), _p(b_in), _p(bs_in), _p(qh),
                                    _p(kh), _p(vh), float(alpha[b, h]), float(beta[b, h]),
                                    _p(c_out), _p(s_out), _p(f_out), _p(a_out), _p(as_out),
                                    _p(b_out), _p(bs_out), _p(o_h))
        assert rc == 0
        if bits == 32:
            new["f"][b, h] = f_out
        else:
            new["codes"][b, h] = c_out
            new["scales"][b, h] = s_out
        win["a"][b, h], win["as"][b, h], win["b"][b, h], win["bs"][b, h] = a_out, as_out, b_out, bs_out
        o[b, h] = o_h
    return new, win, o


def window_full_state(state: dict, window: dict, head_bits, fp32window: bool = False) -> np.ndarray:
    """The full state H + sum_w a_w b_w^T (float64) of a state with a pure-write window."""
    Hs = dequantize(state, head_bits).astype(np.float64)
    if fp32window:
        a, b = window["a"].astype(np.float64), window["b"].astype(np.float64)
    else:
        dec = np.vectorize(e4m3_decode, otypes=[np.float32])
        a = (dec(window["a"]) * window["as"][..., None]).astype(np.float64)
        b = (dec(window["b"]) * window["bs"][..., None]).astype(np.float64)
    return Hs + np.einsum("bhwi,bhwj->bhij", a, b)


def quantize(S: np.ndarray, head_bits, *, rounding: int, seed: int, step: int,
             mode: int = CANONICAL, copy_absmax=None) -> dict:
    """Quantize a full-precision state [B][H][dk][dv]; 32-bit heads are copied.
    ``copy_absmax`` ([B][H][dv]) replaces each column's own maximum in the scale."""
    B, H, dk, dv = S.shape
    st = zero_state(B, H, dk, dv, fp32=any(int(b) == 32 for b in head_bits))
    L = lib()
    for b in range(B):
        for h in range(H):
            bits = int(head_bits[h])
            if bits == 32:
                st["f"][b, h] = S[b, h]
                continue
            hd = _head(dk, dv, bits, rounding, mode, 1, seed, b, h, step)
            mc = None
            if copy_absmax is not None:
                mc = _c(copy_absmax[b, h], np.float32)
                hd.m_copy = mc.ctypes.data
            src = _c(S[b, h], np.float32)
            c_out = np.zeros((dk, dv), np.int8)
            s_out = np.zeros(dv, np.float32)
            assert L.orc_quantize_head(ctypes.byref(hd), _p(src), _p(c_out), _p(s_out)) == 0
            st["codes"][b, h] = c_out
            st["scales"][b, h] = s_out
    return st


def dequantize(st: dict, head_bits) -> np.ndarray:
    """Logical state -> float32 [B][H][dk][dv] (c_ij * s_j, or the stored value for 32-bit heads)."""
    B, H, dk, dv = st["codes"].shape
    out = np.zeros((B, H, dk, dv), np.float32)
    L = lib()
    for b in range(B):
        for h in range(H):
            if int(head_bits[h]) == 32:
                out[b, h] = st["f"][b, h]
                continue
            c = _c(st["codes"][b, h], np.int8)
            s = _c(st["scales"][b, h], np.float32)
            o = np.zeros((dk, dv), np.float32)
            L.orc_dequantize_head(dk, dv, _p(c), _p(s), _p(o))
            out[b, h] = o
    return out


# ---------------------------------------------------------------------------
# Storage format
# ---------------------------------------------------------------------------
def head_bytes(dk: int, dv: int, bits: int) -> int:
    return int(lib().orc_head_bytes(dk, dv, int(bits)))


def pack_state(st: dict, head_bits) -> np.ndarray:
    """Logical state -> library byte buffer uint8 [B][row_bytes] (heads concatenated per row)."""
    B, H, dk, dv = st["codes"].shape
    sizes = [head_bytes(dk, dv, int(b)) for b in head_bits]
    out = np.zeros((B, sum(sizes)), np.uint8)
    L = lib()
    for b in range(B):
        off = 0
        for h in range(H):
            buf = np.zeros(sizes[h], np.uint8)
            c = _c(st["codes"][b, h], np.int8)
            f = _f_in(st, b, h, dk, dv)
            L.orc_pack_head(dk, dv, int(head_bits[h]), _p(c), _p(f), _p(buf))
            out[b, off:off + sizes[h]] = buf
            off += sizes[h]
    return out


def unpack_state(buf: np.ndarray, scales: np.ndarray, head_bits, B: int, H: int, dk: int,
                 dv: int, heads=None) -> dict:
    """Library byte buffer [B][row_bytes] + scales [B][H][dv] -> logical state
    (only the listed (b, h) heads when ``heads`` is given; the others stay zero)."""
    sizes = [head_bytes(dk, dv, int(b)) for b in head_bits]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    buf = _c(buf, np.uint8).reshape(B, int(offs[-1]))
    st = zero_state(B, H, dk, dv, fp32=any(int(b) == 32 for b in head_bits))
    st["scales"] = _c(scales, np.float32).reshape(B, H, dv).copy()
    L = lib()
    for b, h in _heads(B, H, heads):
        src = _c(buf[b, offs[h]:offs[h + 1]], np.uint8)
        c = np.zeros((dk, dv), np.int8)
        f = np.zeros((dk, dv), np.float32)
        L.orc_unpack_head(dk, dv, int(head_bits[h]), _p(src), _p(c), _p(f))
        st["codes"][b, h] = c
        if st["f"] is not None:
            st["f"][b, h] = f
    return st


def allocate_bits(score, n_hi: int, hi: int = 8, lo: int = 4) -> np.ndarray:
    """Decay-based mixed precision: the n_hi heads with the largest score get ``hi`` bits."""
    s = _c(score, np.float64)
    out = np.zeros(s.shape[0], np.int8)
    lib().orc_allocate_bits(_p(s), s.shape[0], int(n_hi), int(hi), int(lo), _p(out))
    return out
