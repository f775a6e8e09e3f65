"""Out-of-bounds checks of every entry point, without a memory checker.

Each device buffer an entry point reads or writes is placed inside a larger
allocation, with poisoned margins on both sides: input margins hold 0xFF
bytes (NaN as float32 and bf16, code -1), output margins and payloads 0xA5.
After the calls, (1) no margin byte has changed, (2) every input payload is
unchanged (inputs are read only), and (3) the results still match the CPU
oracle bit for bit, so a read that strayed into a poisoned margin would have
shown up as a NaN or a wrong code.  Shapes are ragged on purpose: several
heads and batches, units of one, two and four 16-column blocks, mixed head
widths, grids with more CTAs than units.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal, host

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes on each side; the payload starts 4096-byte aligned
IN_POISON, OUT_POISON = 0xFF, 0xA5

_TORCH = {np.dtype(np.float32): torch.float32, np.dtype(np.float64): torch.float64,
          np.dtype(np.uint8): torch.uint8, np.dtype(np.int16): torch.int16}


class Zones:
    """Device buffers with poisoned margins, checked after the calls."""

    def __init__(self):
        self.bufs = []

    @staticmethod
    def _alloc(nbytes, poison):
        return torch.full((MARGIN + nbytes + MARGIN,), poison, dtype=torch.uint8, device="cuda")

    def put(self, a: np.ndarray, name: str) -> torch.Tensor:
        """An input: its bytes in the payload, 0xFF margins; must stay unchanged."""
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        raw = a.reshape(-1).view(np.uint8)
        big = self._alloc(raw.size, IN_POISON)
        big[MARGIN:MARGIN + raw.size].copy_(torch.from_numpy(raw.copy()))
        self.bufs.append((name, big, raw.size, IN_POISON, raw.copy()))
        return big[MARGIN:MARGIN + raw.size].view(_TORCH[a.dtype]).view(a.shape)

    def out(self, shape, dtype, name: str) -> torch.Tensor:
        """An output: payload and margins 0xA5; only the margins are checked."""
        dt = np.dtype(dtype)
        n = int(np.prod(shape)) * dt.itemsize
        big = self._alloc(n, OUT_POISON)
        self.bufs.append((name, big, n, OUT_POISON, None))
        return big[MARGIN:MARGIN + n].view(_TORCH[dt]).view(tuple(shape))

    def check(self):
        torch.cuda.synchronize()
        for name, big, n, poison, payload in self.bufs:
            h = host(big)
            lo, hi = h[:MARGIN], h[MARGIN + n:]
            assert np.all(lo == poison), "%s: %d bytes written before the buffer" % (name, int((lo != poison).sum()))
            assert np.all(hi == poison), "%s: %d bytes written after the buffer (first at +%d)" % (
                name, int((hi != poison).sum()), int(np.argmax(hi != poison)))
            if payload is not None:
                assert np.array_equal(h[MARGIN:MARGIN + n], payload), "%s: input modified" % name


def _state_in(z: Zones, run: Run, st: dict, name: str) -> rsq.State:
    return rsq.State(z.put(oracle.pack_state(st, run.head_bits), name + ".codes"),
                     z.put(np.ascontiguousarray(st["scales"], np.float32), name + ".scales"))


def _state_out(z: Zones, ctx: rsq.Context, name: str, scale_len: int) -> rsq.State:
    return rsq.State(z.out((ctx.batch, ctx.code_bytes // ctx.batch), np.uint8, name + ".codes"),
                     z.out((ctx.batch, ctx.heads, scale_len), np.float32, name + ".scales"))


def _inputs(z: Zones, run: Run, inp: dict, t: int, decay=None):
    d = {k: z.put(v, "%s@%d" % (k, t)) for k, v in inp.items()}
    if run.family == rsq.RSQ_GDN:
        return rsq.gdn_inputs(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    if run.family in (rsq.RSQ_GLA, rsq.RSQ_KDA):
        return rsq.diag_inputs(d["q"], d["k"], d["v"], d["alpha"], d.get("beta"))
    dd = None if decay is None else z.put(np.ascontiguousarray(decay, np.float32), "decay@%d" % t)
    return rsq.mamba2_inputs(d["x"], d["Bm"], d["Cm"], d["dt"], d["A"], d["D"], dd)


def _random_state(run: Run, seed: int) -> dict:
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.3).astype(np.float32)
    if run.f32:
        st = oracle.zero_state(run.B, run.H, run.dk, run.dv, fp32=True)
        st["f"] = S
        return st
    return oracle.quantize(S, run.head_bits, rounding=oracle.SR, seed=3, step=0)


def _mamba_decay(inp):
    return np.exp(inp["dt"].astype(np.float64) * inp["A"][None, :].astype(np.float64)).astype(np.float32)


CASES = [
    # (workload, B, H, dk, dv, bits, rounding, ngroups)
    ("gdn_b64_h16_d128_int8_sr", 3, 5, 32, 16, [8, 4, 4, 8, 4], rsq.RSQ_SR, 1),
    ("gdn_b64_h16_d128_int8_sr", 2, 3, 64, 32, [4, 8, 4], rsq.RSQ_RTN, 1),
    ("gdn_b64_h16_d128_int8_sr", 2, 3, 128, 256, [8, 4, 8], rsq.RSQ_SR, 1),
    ("gdn_b64_h16_d128_int8_sr", 3, 2, 16, 64, [8, 4], rsq.RSQ_SR_BDR, 1),
    ("gdn_b64_h16_d128_int8_sr", 2, 3, 64, 64, [32, 32, 32], rsq.RSQ_SR, 1),
    ("gla_b64_h16_d128_int8_sr", 2, 3, 32, 64, [8, 4, 8], rsq.RSQ_BDR, 1),
    ("kda_b64_h16_d128_int8_sr", 3, 2, 64, 32, [4, 8], rsq.RSQ_SR, 1),
    ("gdn_b64_h8_d256_int8_sr", 3, 3, 256, 16, [8, 4, 8], rsq.RSQ_SR_BDR, 1),   # two warps per block
    ("gdn_b64_h8_d256_int8_sr", 2, 2, 256, 64, [32, 32], rsq.RSQ_SR, 1),
    ("kda_b64_h16_d128_int8_sr", 2, 3, 256, 32, [4, 8, 4], rsq.RSQ_SR, 1),
]


@pytest.mark.parametrize("case", range(len(CASES) + 2))
def test_decode_step_stays_inside_its_buffers(case):
    if case < len(CASES):
        name, B, H, dk, dv, bits, rnd, ng = CASES[case]
        base = W.BY_NAME[name]
    elif case == len(CASES):  # Mamba-2 with shared B/C groups and a ragged group count
        base, B, H, dk, dv, bits, rnd, ng = W.WORKLOADS[3], 2, 6, 32, 64, [8, 4, 8, 4, 4, 8], rsq.RSQ_SR, 3
    else:  # Mamba-2 with a 256-wide state
        base, B, H, dk, dv, bits, rnd, ng = W.WORKLOADS[3], 2, 4, 256, 32, [8, 4, 4, 8], rsq.RSQ_RTN, 2
    w = dataclasses.replace(base, B=B, H=H, dk=dk, dv=dv, ngroups=ng)
    bits = np.array(bits, np.int8)
    run = Run(w, bits, rounding=rnd)
    z = Zones()
    st = _random_state(run, case)
    cur = _state_in(z, run, st, "state0")
    for t in range(3):
        inp = run.inputs(t)
        decay = _mamba_decay(inp) if run.family == rsq.RSQ_MAMBA2 else None
        ins = _inputs(z, run, inp, t, decay)
        nxt = _state_out(z, run.ctx, "state%d" % (t + 1), dv)
        out = z.out((B, H, dv), np.float32, "out@%d" % t)
        run.ctx.decode_step(cur, nxt, ins, out, t)
        z.check()
        st, o = run.oracle_step(st, inp, t, decay=decay)
        assert_state_equal(run.download(nxt), st, bits, what="step %d" % t)
        assert_out_equal(host(out), o, what="step %d" % t)
        cur = nxt
    assert run.ctx.check_flags() == 0


def test_mamba2_device_decay_stays_inside_its_buffers():
    w = dataclasses.replace(W.WORKLOADS[3], B=3, H=4, dk=64, dv=32, ngroups=2)
    run = Run(w, np.array([4, 8, 8, 4], np.int8))
    z = Zones()
    cur = _state_in(z, run, _random_state(run, 11), "state0")
    nxt = _state_out(z, run.ctx, "state1", w.dv)
    out = z.out((w.B, w.H, w.dv), np.float32, "out")
    run.ctx.decode_step(cur, nxt, _inputs(z, run, run.inputs(0), 0), out, 0)
    z.check()
    assert np.isfinite(host(out)).all()


def test_copy_scale_and_column_absmax_stay_inside_their_buffers():
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=3, dk=32, dv=64)
    bits = np.array([4, 8, 4], np.int8)
    q, f = Run(w, bits), Run(w, np.full(3, 32, np.int8))
    z = Zones()
    sq, sf = _random_state(q, 1), _random_state(f, 2)
    gf = _state_in(z, f, sf, "f0")
    gq = _state_in(z, q, sq, "q0")
    for t in range(2):
        inp = q.inputs(t)
        ins = _inputs(z, q, inp, t)
        gf_next = _state_out(z, f.ctx, "f%d" % (t + 1), w.dv)
        gq_next = _state_out(z, q.ctx, "q%d" % (t + 1), w.dv)
        out_f = z.out((w.B, w.H, w.dv), np.float32, "out_f@%d" % t)
        out_q = z.out((w.B, w.H, w.dv), np.float32, "out_q@%d" % t)
        absmax = z.out((w.B, w.H, w.dv), np.float32, "absmax@%d" % t)
        f.ctx.decode_step(gf, gf_next, ins, out_f, t)
        f.ctx.column_absmax(gf_next, absmax)
        q.ctx.decode_step_copy_scale(gq, gq_next, ins, absmax, out_q, t)
        z.check()
        sf, _ = f.oracle_step(sf, inp, t)
        m = np.abs(sf["f"]).max(axis=2)
        sq, o = oracle.gdn_step(sq, inp, bits, rounding=q.rounding, seed=q.seed, step=t, copy_absmax=m)
        assert np.array_equal(host(absmax), m)
        assert_state_equal(q.download(gq_next), sq, bits, what="step %d" % t)
        assert_out_equal(host(out_q), o, what="step %d" % t)
        gf, gq = gf_next, gq_next


def _window_in(z: Zones, win: dict, dv: int, name: str) -> rsq.Window:
    B, H, Wn, _ = win["b"].shape
    b = np.ascontiguousarray(win["b"].reshape(B, H, Wn, dv // 16, 16).transpose(0, 1, 3, 2, 4))
    return rsq.Window(z.put(win["a"], name + ".a"), z.put(win["as"], name + ".as"), z.put(b, name + ".b"),
                      z.put(win["bs"], name + ".bs"))


def _window_out(z: Zones, B, H, Wn, dk, dv, name: str) -> rsq.Window:
    return rsq.Window(z.out((B, H, Wn, dk), np.uint8, name + ".a"), z.out((B, H, Wn), np.float32, name + ".as"),
                      z.out((B, H, dv // 16, Wn, 16), np.uint8, name + ".b"),
                      z.out((B, H, Wn), np.float32, name + ".bs"))


def _window_host(w: rsq.Window, dv: int) -> dict:
    b = host(w.b)
    B, H, nb, Wn, _ = b.shape
    return {"a": host(w.a), "as": host(w.a_scale),
            "b": np.ascontiguousarray(b.transpose(0, 1, 3, 2, 4).reshape(B, H, Wn, dv)), "bs": host(w.b_scale)}


@pytest.mark.parametrize("Wn,dk,dv", [(4, 32, 32), (8, 64, 256), (16, 16, 64)])
def test_window_step_stays_inside_its_buffers(Wn, dk, dv):
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3, dk=dk, dv=dv)
    bits = np.array([8, 4, 8], np.int8)
    run = Run(w, bits)
    ctx = rsq.Context(rsq.RSQ_GDN, w.B, w.H, dk, dv, head_bits=bits, rounding=run.rounding,
                      in_dtype=run.in_dtype, seed=run.seed, window=Wn)
    z = Zones()
    st = _random_state(run, Wn)
    win = oracle.zero_window(w.B, w.H, Wn, dk, dv)
    cur, gwin = _state_in(z, run, st, "state0"), _window_in(z, win, dv, "win0")
    for t in range(Wn + 2):  # through the first merge
        inp = run.inputs(t)
        ins = _inputs(z, run, inp, t)
        nxt = _state_out(z, ctx, "state%d" % (t + 1), dv)
        nwin = _window_out(z, w.B, w.H, Wn, dk, dv, "win%d" % (t + 1))
        out = z.out((w.B, w.H, dv), np.float32, "out@%d" % t)
        ctx.decode_step_window(cur, nxt, gwin, nwin, ins, out, t)
        z.check()
        st, win, o = oracle.gdn_pw_step(st, win, inp, bits, rounding=run.rounding, seed=run.seed, step=t)
        assert_state_equal(run.download(nxt), st, bits, what="step %d" % t)
        assert_out_equal(host(out), o, what="step %d" % t)
        g = _window_host(nwin, dv)
        for key in ("a", "b"):
            assert np.array_equal(g[key], win[key]), "step %d window %s" % (t, key)
        for key in ("as", "bs"):
            assert np.array_equal(g[key].view(np.uint32), win[key].view(np.uint32)), "step %d window %s" % (t, key)
        cur, gwin = nxt, nwin


@pytest.mark.parametrize("dk,dv", [(32, 16), (128, 64)])
def test_key_axis_paths_stay_inside_their_buffers(dk, dv):
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=2, dk=dk, dv=dv)
    bits = np.array([4, 8], np.int8)
    run = Run(w, bits)
    ctx = rsq.Context(rsq.RSQ_GDN, w.B, w.H, dk, dv, head_bits=bits, rounding=rsq.RSQ_SR,
                      in_dtype=run.in_dtype, seed=run.seed, key_axis=1)
    z = Zones()
    rng = np.random.default_rng(dk + dv)
    S = (rng.standard_normal((w.B, w.H, dk, dv)) * 0.3).astype(np.float32)
    gS = z.put(S, "S")
    cur = _state_out(z, ctx, "state0", dk)
    ctx.quantize(gS, cur, step=4)
    z.check()
    st = oracle.quantize_ka(S, bits, rounding=oracle.SR, seed=run.seed, step=4)
    for t in range(2):
        inp = run.inputs(t)
        ins = _inputs(z, run, inp, t)
        nxt = _state_out(z, ctx, "state%d" % (t + 1), dk)
        out = z.out((w.B, w.H, dv), np.float32, "out@%d" % t)
        ctx.decode_step(cur, nxt, ins, out, t)
        z.check()
        st, o = oracle.gdn_ka_step(st, inp, bits, rounding=oracle.SR, seed=run.seed, step=t)
        got = oracle.unpack_state(host(nxt.codes), np.zeros((w.B, w.H, dv), np.float32), bits, w.B, w.H, dk, dv)
        assert np.array_equal(got["codes"], st["codes"]), "step %d codes" % t
        assert np.array_equal(host(nxt.scales).view(np.uint32), st["scales"].view(np.uint32)), "step %d scales" % t
        assert_out_equal(host(out), o, what="step %d" % t)
        cur = nxt
    D = z.out((w.B, w.H, dk, dv), np.float32, "D")
    ctx.dequantize(cur, D)
    z.check()
    assert np.array_equal(host(D).view(np.uint32), oracle.dequantize_ka(st).view(np.uint32))


@pytest.mark.parametrize("bits", [[8, 4, 8, 4, 4], [32, 32, 32, 32, 32]])
def test_quantize_dequantize_drift_stay_inside_their_buffers(bits):
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=5, dk=64, dv=32)
    bits = np.array(bits, np.int8)
    run = Run(w, bits)
    f = Run(w, np.full(5, 32, np.int8))
    z = Zones()
    rng = np.random.default_rng(int(bits[0]))
    S = (rng.standard_normal((3, 5, 64, 32)) * rng.uniform(0.01, 5, (3, 5, 1, 32))).astype(np.float32)
    s = _state_out(z, run.ctx, "q", w.dv)
    run.ctx.quantize(z.put(S, "S"), s, step=7)
    D = z.out((3, 5, 64, 32), np.float32, "D")
    run.ctx.dequantize(s, D)
    quantized = not run.f32
    if quantized:  # the drift kernel compares a quantized state with a full-precision one
        fs = oracle.zero_state(3, 5, 64, 32, fp32=True)
        fs["f"] = S * 1.01
        sums = z.out((3, 5, 2), np.float64, "sums")
        rsq.rsq_state_drift(run.ctx.ctx, s, f.ctx.ctx, _state_in(z, f, fs, "f"), sums)
    z.check()
    ref = oracle.quantize(S, bits, rounding=run.rounding, seed=run.seed, step=7)
    assert_state_equal(run.download(s), ref, bits, what="quantize")
    deq = oracle.dequantize(ref, bits)
    assert np.array_equal(host(D).view(np.uint32), deq.view(np.uint32))
    if quantized:
        e2 = ((deq.astype(np.float64) - fs["f"]) ** 2).sum(axis=(2, 3))
        assert np.allclose(host(sums)[..., 0], e2, rtol=1e-12)
