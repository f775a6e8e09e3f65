"""Test harness: run the CUDA library and the CPU oracle on the same seeded inputs.

Converts between the oracle's logical state and device buffers, uploads the
seeded inputs of ``workloads`` and compares results.  Test code only.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W

DEV = "cuda"


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> device tensor with the same bytes (uint16 bf16 bits travel as int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a.copy()).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


class Run:
    """One layer configuration on the GPU plus its oracle twin."""

    def __init__(self, w: W.Workload, head_bits, *, B=None, H=None, rounding=None, seed=None,
                 in_dtype=None):
        self.w = w
        self.B = w.B if B is None else B
        self.H = w.H if H is None else H
        self.dk, self.dv = w.dk, w.dv
        self.head_bits = np.asarray(head_bits, np.int8)
        assert self.head_bits.shape == (self.H,)
        # the workloads' stochastic rounding is the 8-bit-uniform rule; "sr16" the 16-bit one
        self.rounding = ({"rtn": rsq.RSQ_RTN, "sr": rsq.RSQ_SR8, "sr16": rsq.RSQ_SR}[w.rounding]
                         if rounding is None else rounding)
        self.seed = w.sr_seed if seed is None else seed
        self.in_dtype = {"f32": rsq.RSQ_F32, "bf16": rsq.RSQ_BF16}[w.in_dtype] if in_dtype is None else in_dtype
        self.family = {"gdn": rsq.RSQ_GDN, "mamba2": rsq.RSQ_MAMBA2, "gla": rsq.RSQ_GLA,
                       "kda": rsq.RSQ_KDA}[w.family]
        self.ctx = rsq.Context(self.family, self.B, self.H, self.dk, self.dv, head_bits=self.head_bits,
                               rounding=self.rounding, in_dtype=self.in_dtype, seed=self.seed,
                               ngroups=w.ngroups)
        self.R = rsq.rsq_reduction_partials(self.dk)
        self.f32 = bool(np.all(self.head_bits == 32))

    # -- state transfer ----------------------------------------------------
    def upload(self, st: dict) -> rsq.State:
        codes = oracle.pack_state(st, self.head_bits)
        return rsq.State(dev(codes), dev(np.ascontiguousarray(st["scales"], np.float32)))

    def download(self, s: rsq.State, heads=None) -> dict:
        return oracle.unpack_state(host(s.codes), host(s.scales), self.head_bits, self.B, self.H,
                                   self.dk, self.dv, heads=heads)

    def zero(self) -> dict:
        return oracle.zero_state(self.B, self.H, self.dk, self.dv, fp32=self.f32)

    # -- inputs --------------------------------------------------------------
    def inputs(self, t: int) -> dict:
        inp = W.inputs(self.w, t, B=self.B)
        if self.H != self.w.H:
            for key in ("q", "k", "v", "alpha", "beta", "x", "dt"):
                if key in inp:
                    inp[key] = np.ascontiguousarray(inp[key][:, :self.H])
            for key in ("A", "D"):
                if key in inp:
                    inp[key] = np.ascontiguousarray(inp[key][:self.H])
        if self.in_dtype == rsq.RSQ_F32:
            for key in ("q", "k", "v", "x", "Bm", "Cm"):
                if key in inp and inp[key].dtype == np.uint16:
                    inp[key] = W.bf16_to_f32(inp[key])
        return inp

    def dev_inputs(self, inp: dict, decay=None):
        keep = {k: dev(v) for k, v in inp.items()}
        if self.family == rsq.RSQ_GDN:
            s = rsq.gdn_inputs(keep["q"], keep["k"], keep["v"], keep["alpha"], keep["beta"])
        elif self.family in (rsq.RSQ_GLA, rsq.RSQ_KDA):
            s = rsq.diag_inputs(keep["q"], keep["k"], keep["v"], keep["alpha"], keep.get("beta"))
        else:
            dd = None if decay is None else dev(np.ascontiguousarray(decay, np.float32))
            keep["decay"] = dd
            s = rsq.mamba2_inputs(keep["x"], keep["Bm"], keep["Cm"], keep["dt"], keep["A"], keep["D"], dd)
        return s, keep

    # -- one step on each side -----------------------------------------------
    def gpu_step(self, s_in: rsq.State, s_out: rsq.State, inp: dict, t: int, decay=None):
        ins, keep = self.dev_inputs(inp, decay)
        out = torch.empty((self.B, self.H, self.dv), dtype=torch.float32, device=DEV)
        self.ctx.decode_step(s_in, s_out, ins, out, t)
        torch.cuda.synchronize()
        del keep
        return host(out)

    def oracle_step(self, st: dict, inp: dict, t: int, mode=oracle.CANONICAL, decay=None, heads=None):
        if self.family == rsq.RSQ_GDN:
            return oracle.gdn_step(st, inp, self.head_bits, rounding=self.rounding, seed=self.seed,
                                   step=t, mode=mode, R=self.R, heads=heads)
        if self.family in (rsq.RSQ_GLA, rsq.RSQ_KDA):
            step = oracle.gla_step if self.family == rsq.RSQ_GLA else oracle.kda_step
            return step(st, inp, self.head_bits, rounding=self.rounding, seed=self.seed, step=t,
                        mode=mode, R=self.R, heads=heads)
        return oracle.mamba2_step(st, inp, self.head_bits, rounding=self.rounding, seed=self.seed,
                                  step=t, mode=mode, R=self.R, ngroups=self.w.ngroups, decay=decay,
                                  heads=heads)


def mixed_bits(w: W.Workload, H: int | None = None) -> np.ndarray:
    """Decay-based allocation of a mixed workload (library host routine)."""
    score = W.mean_alpha_per_head(w, steps=min(w.steps, 32))
    H = w.H if H is None else H
    return rsq.rsq_allocate_bits(score[:H], int(H * w.high_frac))


def bits_for(w: W.Workload, H: int | None = None) -> np.ndarray:
    H = w.H if H is None else H
    if w.state == "mixed":
        return mixed_bits(w, H)
    return W.head_bits_for(w)[:H]


def assert_state_equal(a: dict, b: dict, head_bits, heads=None, what=""):
    """Bit-exact comparison of two logical states (codes; scales bitwise incl. NaN)."""
    B, H = a["codes"].shape[:2]
    pairs = [(bb, hh) for bb in range(B) for hh in range(H)] if heads is None else heads
    for bb, hh in pairs:
        if int(head_bits[hh]) == 32:
            fa, fb = a["f"][bb, hh], b["f"][bb, hh]
            assert np.array_equal(fa.view(np.uint32), fb.view(np.uint32)), "%s f32 state (%d,%d)" % (what, bb, hh)
            continue
        ca, cb = a["codes"][bb, hh], b["codes"][bb, hh]
        sa, sb = a["scales"][bb, hh], b["scales"][bb, hh]
        nan = np.isnan(sa) | np.isnan(sb)
        assert np.array_equal(np.isnan(sa), np.isnan(sb)), "%s scale NaN (%d,%d)" % (what, bb, hh)
        assert np.array_equal(sa[~nan].view(np.uint32), sb[~nan].view(np.uint32)), \
            "%s scales (%d,%d)" % (what, bb, hh)
        if not np.array_equal(ca, cb):
            d = np.argwhere(ca != cb)
            raise AssertionError("%s codes (%d,%d): %d differ, first %s gpu=%d oracle=%d"
                                 % (what, bb, hh, len(d), d[0], ca[tuple(d[0])], cb[tuple(d[0])]))


def assert_out_equal(a: np.ndarray, b: np.ndarray, heads=None, what=""):
    if heads is not None:
        idx = tuple(np.array(heads).T)
        a, b = a[idx], b[idx]
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), \
        "%s outputs differ: max abs %g" % (what, float(np.nanmax(np.abs(a - b))))


def sample_heads(B: int, H: int, n: int, seed: int = 0):
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * H, size=min(n, B * H), replace=False)
    flat = np.unique(np.concatenate([flat, [0, B * H - 1]]))
    return [(int(f // H), int(f % H)) for f in flat]
