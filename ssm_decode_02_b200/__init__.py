"""Quantized recurrent-state decode step for B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI of ``librsq.so`` (declared in include/rsq.h).
The functions keep the C names (``rsq_create``, ``rsq_decode_step``, ...) and
only marshal arguments: tensors become device pointers, streams become
``cudaStream_t`` handles.  Every step of the decode path runs in the library's
CUDA kernels; there is no fallback, and importing this package on a machine
where the library cannot be loaded raises.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librsq.so")

RSQ_GDN, RSQ_MAMBA2, RSQ_GLA, RSQ_KDA = 0, 1, 2, 3
RSQ_RTN, RSQ_SR, RSQ_BDR, RSQ_SR_BDR = 0, 1, 2, 3
RSQ_SR8, RSQ_SR8_BDR = 5, 7   # stochastic rounding with 8-bit uniforms (RSQ_SR: 16-bit)
RSQ_F32, RSQ_BF16 = 0, 1
RSQ_OK, RSQ_E_INVAL, RSQ_E_UNSUPPORTED, RSQ_E_CUDA, RSQ_E_NOMEM, RSQ_E_NONFINITE = range(6)
RSQ_MAX_HEADS = 512


class RsqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("rsq status %d (%s): %s" % (status, _status_name(status), message))
        self.status = status


rsq_alloc_fn = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p)
rsq_release_fn = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_void_p)


class rsq_config(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int), ("batch", ctypes.c_int), ("heads", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("head_bits", ctypes.POINTER(ctypes.c_int8)), ("rounding", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("seed", ctypes.c_uint64), ("window", ctypes.c_int),
                ("key_axis", ctypes.c_int), ("alloc", rsq_alloc_fn), ("release", rsq_release_fn),
                ("alloc_user", ctypes.c_void_p)]


class rsq_state(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class rsq_gdn_inputs(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p)]


class rsq_mamba2_inputs(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("Bm", ctypes.c_void_p), ("Cm", ctypes.c_void_p),
                ("dt", ctypes.c_void_p), ("A", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("decay", ctypes.c_void_p)]


class rsq_window(ctypes.Structure):
    _fields_ = [("a", ctypes.c_void_p), ("a_scale", ctypes.c_void_p), ("b", ctypes.c_void_p),
                ("b_scale", ctypes.c_void_p)]


class rsq_diag_inputs(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p)]


_EXPORTS = ["rsq_create", "rsq_destroy", "rsq_state_bytes", "rsq_head_offset", "rsq_decode_step",
            "rsq_quantize", "rsq_dequantize", "rsq_state_drift", "rsq_check_flags",
            "rsq_allocate_bits", "rsq_reduction_partials", "rsq_status_string", "rsq_last_error",
            "rsq_version", "rsq_decode_step_noalloc", "rsq_decode_step_copy_scale",
            "rsq_column_absmax", "rsq_window_bytes", "rsq_decode_step_window", "rsq_debug_waits"]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("librsq.so not built (run python -m ssm_decode_02_b200.build): %s" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, C = ctypes.c_void_p, ctypes.c_int
    sig = {
        "rsq_create": ([ctypes.POINTER(rsq_config), ctypes.POINTER(P)], C),
        "rsq_destroy": ([P], None),
        "rsq_state_bytes": ([P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)], C),
        "rsq_head_offset": ([P, C, ctypes.POINTER(ctypes.c_size_t)], C),
        "rsq_decode_step": ([P, ctypes.POINTER(rsq_state), ctypes.POINTER(rsq_state), P, P,
                             ctypes.c_uint32, P], C),
        "rsq_quantize": ([P, P, ctypes.POINTER(rsq_state), ctypes.c_uint32, P], C),
        "rsq_dequantize": ([P, ctypes.POINTER(rsq_state), P, P], C),
        "rsq_state_drift": ([P, ctypes.POINTER(rsq_state), P, ctypes.POINTER(rsq_state), P, P], C),
        "rsq_check_flags": ([P, ctypes.POINTER(C), P], C),
        "rsq_allocate_bits": ([P, C, C, C, C, P], C),
        "rsq_reduction_partials": ([C], C),
        "rsq_status_string": ([C], ctypes.c_char_p),
        "rsq_last_error": ([], ctypes.c_char_p),
        "rsq_version": ([], ctypes.c_char_p),
        "rsq_decode_step_noalloc": ([ctypes.POINTER(rsq_config), ctypes.POINTER(rsq_state),
                                     ctypes.POINTER(rsq_state), P, P, ctypes.c_uint32, P], C),
        "rsq_decode_step_copy_scale": ([P, ctypes.POINTER(rsq_state), ctypes.POINTER(rsq_state), P, P,
                                        P, ctypes.c_uint32, P], C),
        "rsq_column_absmax": ([P, ctypes.POINTER(rsq_state), P, P], C),
        "rsq_window_bytes": ([P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t),
                              ctypes.POINTER(ctypes.c_size_t)], C),
        "rsq_decode_step_window": ([P, ctypes.POINTER(rsq_state), ctypes.POINTER(rsq_state),
                                    ctypes.POINTER(rsq_window), ctypes.POINTER(rsq_window), P, P,
                                    ctypes.c_uint32, P], C),
        "rsq_host_input_layout": ([P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t),
                                   ctypes.POINTER(ctypes.c_size_t)], C),
        "rsq_pipe_create": ([P, ctypes.POINTER(P)], C),
        "rsq_pipe_destroy": ([P], None),
        "rsq_pipe_step": ([P, ctypes.POINTER(rsq_state), ctypes.POINTER(rsq_state), ctypes.POINTER(rsq_window),
                           ctypes.POINTER(rsq_window), P, P, ctypes.c_uint32], C),
        "rsq_pipe_sync": ([P], C),
        "rsq_pipe_streams": ([P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P)], C),
        "rsq_debug_waits": ([P, ctypes.c_uint32, C], C),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _status_name(s: int) -> str:
    return lib.rsq_status_string(int(s)).decode()


def _check(status: int) -> int:
    if status != RSQ_OK:
        raise RsqError(status, lib.rsq_last_error().decode())
    return status


def _ptr(t) -> int | None:
    """Host address of a numpy array (host arguments); ints pass through; None stays None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return int(t.ctypes.data)
    if hasattr(t, "data_ptr"):
        return int(t.data_ptr())
    raise TypeError("cannot take the address of %r" % type(t))


def _dptr(t) -> int | None:
    """Device address of a CUDA tensor argument; a CPU or non-contiguous tensor is
    refused here instead of reaching the kernel.  Ints (raw device addresses) pass
    through; None stays None."""
    if t is None or isinstance(t, int):
        return t
    if not hasattr(t, "data_ptr"):
        raise TypeError("expected a CUDA tensor, got %r" % type(t))
    if not getattr(t, "is_cuda", False):
        raise ValueError("expected a CUDA tensor, got one on %s" % getattr(t, "device", "the host"))
    if not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return int(t.data_ptr())


def _hptr(t) -> int:
    """Host address of a host buffer argument (numpy array or CPU tensor); a CUDA
    tensor is refused here."""
    if getattr(t, "is_cuda", False):
        raise ValueError("expected a host buffer, got a CUDA tensor")
    if isinstance(t, np.ndarray) and not t.flags.c_contiguous:
        raise ValueError("expected a contiguous host buffer")
    if hasattr(t, "is_contiguous") and not t.is_contiguous():
        raise ValueError("expected a contiguous host buffer")
    p = _ptr(t)
    if not p:
        raise ValueError("null host buffer")
    return p


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


# ---------------------------------------------------------------------------
# C functions under their own names (argument marshalling only)
# ---------------------------------------------------------------------------
def rsq_create(family: int, batch: int, heads: int, dk: int, dv: int, *, head_bits=None,
               rounding: int = RSQ_SR8, in_dtype: int = RSQ_BF16, seed: int = 0,
               ngroups: int = 1, window: int = 0, key_axis: int = 0, alloc=None, release=None) -> int:
    """``alloc`` / ``release``: rsq_alloc_fn / rsq_release_fn objects (the
    allocator hook; the caller keeps them alive as long as the context)."""
    cfg, bits_arr = _config(family, batch, heads, dk, dv, head_bits, rounding, in_dtype, seed, ngroups,
                            window, key_axis)
    if alloc is not None:
        cfg.alloc = alloc
    if release is not None:
        cfg.release = release
    out = ctypes.c_void_p()
    _check(lib.rsq_create(ctypes.byref(cfg), ctypes.byref(out)))
    return int(out.value)


def _config(family, batch, heads, dk, dv, head_bits, rounding, in_dtype, seed, ngroups, window=0,
            key_axis=0):
    bits_arr = None
    if head_bits is not None:
        bits_arr = (ctypes.c_int8 * heads)(*[int(b) for b in head_bits])
    cfg = rsq_config(int(family), int(batch), int(heads), int(dk), int(dv), int(ngroups),
                     ctypes.cast(bits_arr, ctypes.POINTER(ctypes.c_int8)) if bits_arr else None,
                     int(rounding), int(in_dtype), int(seed) & (2 ** 64 - 1), int(window),
                     int(key_axis))
    return cfg, bits_arr


def rsq_decode_step_noalloc(family: int, batch: int, heads: int, dk: int, dv: int, state_in,
                            state_out, inputs, out, step: int, *, head_bits=None,
                            rounding: int = RSQ_SR8, in_dtype: int = RSQ_BF16, seed: int = 0,
                            ngroups: int = 1, stream=None) -> None:
    """Decode step without a context and without any device allocation (the
    kernel's flag word lives in a static device array; see include/rsq.h)."""
    cfg, keep = _config(family, batch, heads, dk, dv, head_bits, rounding, in_dtype, seed, ngroups)
    si, so = _state(state_in), _state(state_out)
    _check(lib.rsq_decode_step_noalloc(ctypes.byref(cfg), ctypes.byref(si), ctypes.byref(so),
                                       ctypes.byref(inputs), _dptr(out), int(step) & 0xFFFFFFFF,
                                       _stream(stream)))
    del keep


def rsq_destroy(ctx: int) -> None:
    lib.rsq_destroy(ctx)


def rsq_state_bytes(ctx: int) -> tuple[int, int]:
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.rsq_state_bytes(ctx, ctypes.byref(a), ctypes.byref(b)))
    return int(a.value), int(b.value)


def rsq_head_offset(ctx: int, h: int) -> int:
    o = ctypes.c_size_t()
    _check(lib.rsq_head_offset(ctx, int(h), ctypes.byref(o)))
    return int(o.value)


def _state(st) -> rsq_state:
    return rsq_state(_dptr(st.codes), _dptr(st.scales))


def rsq_decode_step(ctx: int, state_in, state_out, inputs, out, step: int, stream=None) -> None:
    """inputs: rsq_gdn_inputs / rsq_mamba2_inputs / rsq_diag_inputs (see gdn_inputs,
    mamba2_inputs, diag_inputs)."""
    si, so = _state(state_in), _state(state_out)
    _check(lib.rsq_decode_step(ctx, ctypes.byref(si), ctypes.byref(so), ctypes.byref(inputs),
                               _dptr(out), int(step) & 0xFFFFFFFF, _stream(stream)))


def rsq_decode_step_copy_scale(ctx: int, state_in, state_out, inputs, copy_absmax, out, step: int,
                               stream=None) -> None:
    """Decode step whose scales come from copy_absmax ([B][H][dv], column maxima of an
    unquantized copy of the state) instead of the state's own columns."""
    si, so = _state(state_in), _state(state_out)
    _check(lib.rsq_decode_step_copy_scale(ctx, ctypes.byref(si), ctypes.byref(so), ctypes.byref(inputs),
                                          _dptr(copy_absmax), _dptr(out), int(step) & 0xFFFFFFFF,
                                          _stream(stream)))


def rsq_column_absmax(ctx: int, state, absmax, stream=None) -> None:
    """Column maxima of |S^| of a stored state into absmax ([B][H][dv] float32, device)."""
    si = _state(state)
    _check(lib.rsq_column_absmax(ctx, ctypes.byref(si), _dptr(absmax), _stream(stream)))


def rsq_window_bytes(ctx: int) -> tuple[int, int, int]:
    a, b, sc = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.rsq_window_bytes(ctx, ctypes.byref(a), ctypes.byref(b), ctypes.byref(sc)))
    return int(a.value), int(b.value), int(sc.value)


def _window(win) -> rsq_window:
    return rsq_window(_dptr(win.a), _dptr(win.a_scale), _dptr(win.b), _dptr(win.b_scale))


def rsq_decode_step_window(ctx: int, state_in, state_out, win_in, win_out, inputs, out, step: int,
                           stream=None) -> None:
    si, so = _state(state_in), _state(state_out)
    wi, wo = _window(win_in), _window(win_out)
    _check(lib.rsq_decode_step_window(ctx, ctypes.byref(si), ctypes.byref(so), ctypes.byref(wi),
                                      ctypes.byref(wo), ctypes.byref(inputs), _dptr(out),
                                      int(step) & 0xFFFFFFFF, _stream(stream)))


def rsq_host_input_layout(ctx: int) -> tuple[list[int], list[int], int]:
    """(offsets, sizes, total) of the packed host input buffer of one step."""
    off = (ctypes.c_size_t * 6)()
    size = (ctypes.c_size_t * 6)()
    total = ctypes.c_size_t()
    _check(lib.rsq_host_input_layout(ctx, off, size, ctypes.byref(total)))
    return list(off), list(size), int(total.value)


def rsq_pipe_create(ctx: int) -> int:
    out = ctypes.c_void_p()
    _check(lib.rsq_pipe_create(ctx, ctypes.byref(out)))
    return int(out.value)


def rsq_pipe_destroy(pipe: int) -> None:
    lib.rsq_pipe_destroy(pipe)


def rsq_pipe_step(pipe: int, state_in, state_out, host_inputs, host_out, step: int, win_in=None,
                  win_out=None) -> None:
    """host_inputs: the packed host buffer (pack_host_inputs); host_out: host float [B][H][dv]."""
    si, so = _state(state_in), _state(state_out)
    wi = ctypes.byref(_window(win_in)) if win_in is not None else None
    wo = ctypes.byref(_window(win_out)) if win_out is not None else None
    _check(lib.rsq_pipe_step(pipe, ctypes.byref(si), ctypes.byref(so), wi, wo, _hptr(host_inputs),
                             _hptr(host_out), int(step) & 0xFFFFFFFF))


def rsq_pipe_sync(pipe: int) -> None:
    _check(lib.rsq_pipe_sync(pipe))


def rsq_pipe_streams(pipe: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib.rsq_pipe_streams(pipe, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return int(a.value), int(b.value), int(c.value)


def rsq_quantize(ctx: int, S, state_out, step: int, stream=None) -> None:
    so = _state(state_out)
    _check(lib.rsq_quantize(ctx, _dptr(S), ctypes.byref(so), int(step) & 0xFFFFFFFF, _stream(stream)))


def rsq_dequantize(ctx: int, state_in, S_out, stream=None) -> None:
    si = _state(state_in)
    _check(lib.rsq_dequantize(ctx, ctypes.byref(si), _dptr(S_out), _stream(stream)))


def rsq_state_drift(q_ctx: int, q_state, f_ctx: int, f_state, sums, stream=None) -> None:
    a, b = _state(q_state), _state(f_state)
    _check(lib.rsq_state_drift(q_ctx, ctypes.byref(a), f_ctx, ctypes.byref(b), _dptr(sums),
                               _stream(stream)))


def rsq_check_flags(ctx: int, stream=None) -> int:
    """Returns 1 if a non-finite column was seen since the last check (and clears it)."""
    seen = ctypes.c_int(0)
    st = lib.rsq_check_flags(ctx, ctypes.byref(seen), _stream(stream))
    if st not in (RSQ_OK, RSQ_E_NONFINITE):
        _check(st)
    return int(seen.value)


def rsq_debug_waits(ctx: int, wait_iters: int, withhold: int) -> None:
    """Failure-detection tests: limit the kernels' bounded waits and withhold an
    exchange-barrier arrival (see rsq.h)."""
    _check(lib.rsq_debug_waits(ctx, int(wait_iters), int(withhold)))


def rsq_allocate_bits(score, n_high: int, high_bits: int = 8, low_bits: int = 4) -> np.ndarray:
    s = np.ascontiguousarray(score, dtype=np.float64)
    out = np.zeros(s.shape[0], dtype=np.int8)
    _check(lib.rsq_allocate_bits(_ptr(s), s.shape[0], int(n_high), int(high_bits), int(low_bits),
                                 _ptr(out)))
    return out


def rsq_reduction_partials(dk: int) -> int:
    return int(lib.rsq_reduction_partials(int(dk)))


def rsq_version() -> str:
    return lib.rsq_version().decode()


# ---------------------------------------------------------------------------
# Convenience containers (torch tensors for device memory)
# ---------------------------------------------------------------------------
class State:
    """A stored state: codes uint8 [B][row_bytes] and scales float32 [B][H][dv] (device)."""

    def __init__(self, codes, scales):
        self.codes = codes
        self.scales = scales


class Window:
    """A pure-write window (device): a uint8 [B][H][W][dk], a_scale float [B][H][W],
    b uint8 [B][H][dv/16][W][16], b_scale float [B][H][W]."""

    def __init__(self, a, a_scale, b, b_scale):
        self.a, self.a_scale, self.b, self.b_scale = a, a_scale, b, b_scale


def gdn_inputs(q, k, v, alpha, beta) -> rsq_gdn_inputs:
    return rsq_gdn_inputs(_dptr(q), _dptr(k), _dptr(v), _dptr(alpha), _dptr(beta))


def diag_inputs(q, k, v, alpha, beta=None) -> rsq_diag_inputs:
    """GLA / KDA inputs: alpha is the decay per key channel ([B][H][dk] float32)."""
    return rsq_diag_inputs(_dptr(q), _dptr(k), _dptr(v), _dptr(alpha), _dptr(beta))


def mamba2_inputs(x, Bm, Cm, dt, A, D, decay=None) -> rsq_mamba2_inputs:
    return rsq_mamba2_inputs(_dptr(x), _dptr(Bm), _dptr(Cm), _dptr(dt), _dptr(A), _dptr(D), _dptr(decay))


class Context:
    """Owns one rsq_ctx (one layer configuration)."""

    def __init__(self, family: int, batch: int, heads: int, dk: int, dv: int, *, head_bits=None,
                 rounding: int = RSQ_SR8, in_dtype: int = RSQ_BF16, seed: int = 0, ngroups: int = 1,
                 window: int = 0, key_axis: int = 0, allocator=None):
        """``allocator``: optional (alloc(nbytes) -> device address or None,
        release(address)) pair for the context's own device word."""
        self.family, self.batch, self.heads, self.dk, self.dv = family, batch, heads, dk, dv
        self.head_bits = None if head_bits is None else np.asarray(head_bits, np.int8)
        self.rounding, self.in_dtype, self.seed, self.ngroups = rounding, in_dtype, seed, ngroups
        self.window, self.key_axis = window, key_axis
        self._hooks = (None, None)
        if allocator is not None:
            a, r = allocator
            self._hooks = (rsq_alloc_fn(lambda n, _u: a(int(n))), rsq_release_fn(lambda p, _u: r(int(p))))
        self.ctx = rsq_create(family, batch, heads, dk, dv, head_bits=head_bits, rounding=rounding,
                              in_dtype=in_dtype, seed=seed, ngroups=ngroups, window=window,
                              key_axis=key_axis, alloc=self._hooks[0], release=self._hooks[1])
        self.code_bytes, self.scale_bytes = rsq_state_bytes(self.ctx)

    def close(self):
        if getattr(self, "ctx", None):
            rsq_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc_state(self, device="cuda") -> State:
        import torch
        codes = torch.empty((self.batch, self.code_bytes // self.batch), dtype=torch.uint8, device=device)
        scales = torch.empty((self.batch, self.heads, self.dk if self.key_axis else self.dv),
                             dtype=torch.float32, device=device)
        return State(codes, scales)

    def decode_step(self, state_in: State, state_out: State, inputs, out, step: int, stream=None):
        rsq_decode_step(self.ctx, state_in, state_out, inputs, out, step, stream)

    def alloc_window(self, device="cuda") -> Window:
        """An empty (all-zero) pure-write window."""
        import torch
        B, H, W = self.batch, self.heads, self.window
        return Window(torch.zeros((B, H, W, self.dk), dtype=torch.uint8, device=device),
                      torch.zeros((B, H, W), dtype=torch.float32, device=device),
                      torch.zeros((B, H, self.dv // 16, W, 16), dtype=torch.uint8, device=device),
                      torch.zeros((B, H, W), dtype=torch.float32, device=device))

    def decode_step_window(self, state_in: State, state_out: State, win_in: Window, win_out: Window,
                           inputs, out, step: int, stream=None):
        rsq_decode_step_window(self.ctx, state_in, state_out, win_in, win_out, inputs, out, step, stream)

    def decode_step_copy_scale(self, state_in: State, state_out: State, inputs, copy_absmax, out,
                               step: int, stream=None):
        rsq_decode_step_copy_scale(self.ctx, state_in, state_out, inputs, copy_absmax, out, step, stream)

    def column_absmax(self, state: State, absmax, stream=None):
        rsq_column_absmax(self.ctx, state, absmax, stream)

    def quantize(self, S, state_out: State, step: int = 0, stream=None):
        rsq_quantize(self.ctx, S, state_out, step, stream)

    def dequantize(self, state_in: State, S_out, stream=None):
        rsq_dequantize(self.ctx, state_in, S_out, stream)

    def check_flags(self, stream=None) -> int:
        return rsq_check_flags(self.ctx, stream)


def pack_host_inputs(ctx: "Context", inputs: dict, out=None):
    """Pack one step's host input arrays (numpy; bf16 as uint16 bits) into the
    library's host layout (rsq_host_input_layout), in page-locked memory.
    Marshalling only: each array is copied byte for byte to its offset."""
    import torch
    names = (("x", "Bm", "Cm", "dt", "A", "D") if ctx.family == RSQ_MAMBA2
             else ("q", "k", "v", "alpha", "beta"))
    off, size, total = rsq_host_input_layout(ctx.ctx)
    if out is None:
        out = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    buf = out.numpy()
    for f, name in enumerate(names):
        if size[f] == 0:
            continue
        a = np.ascontiguousarray(inputs[name]).reshape(-1).view(np.uint8)
        if a.size != size[f]:
            raise ValueError("input %s has %d bytes, the layout expects %d" % (name, a.size, size[f]))
        buf[off[f]:off[f] + size[f]] = a
    return out


class Pipe:
    """An end-to-end pipeline over host buffers for one Context (rsq_pipe)."""

    def __init__(self, ctx: "Context"):
        self.context = ctx  # the pipe borrows the context: keep it alive
        self.pipe = rsq_pipe_create(ctx.ctx)
        self.copy_in, self.compute, self.copy_out = rsq_pipe_streams(self.pipe)

    def step(self, state_in: State, state_out: State, host_inputs, host_out, step: int, win_in=None,
             win_out=None):
        rsq_pipe_step(self.pipe, state_in, state_out, host_inputs, host_out, step, win_in, win_out)

    def sync(self):
        rsq_pipe_sync(self.pipe)

    def close(self):
        if getattr(self, "pipe", None):
            rsq_pipe_destroy(self.pipe)
            self.pipe = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
