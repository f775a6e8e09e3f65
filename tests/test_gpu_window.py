"""GPU parity of the pure-write window ("Low-Bit GDN Recurrent-State
Quantization: Global Gradient-aware Allocation and Pure-Write Sliding
Windows", abstract) against the CPU oracle.

Gated DeltaNet with W window slots: both sides free-run from S_0 = 0 and an
empty window; every step the low-bit history (codes, scales), the readout and
the window itself (FP8 codes and scales of both vector sets) must agree bit for
bit -- through the first W steps (slots filling), the first merges and beyond.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal, dev, host, sample_heads

pytestmark = pytest.mark.gpu


def _upload_window(win: dict, dv: int) -> rsq.Window:
    B, H, Wn, _ = win["b"].shape
    b = np.ascontiguousarray(win["b"].reshape(B, H, Wn, dv // 16, 16).transpose(0, 1, 3, 2, 4))
    return rsq.Window(dev(win["a"]), dev(win["as"]), dev(b), dev(win["bs"]))


def _download_window(w: rsq.Window, dv: int) -> dict:
    b = host(w.b)
    B, H, nb, Wn, _ = b.shape
    return {"a": host(w.a), "as": host(w.a_scale),
            "b": np.ascontiguousarray(b.transpose(0, 1, 3, 2, 4).reshape(B, H, Wn, dv)),
            "bs": host(w.b_scale)}


def _assert_window_equal(g: dict, o: dict, heads, what):
    for b, h in heads:
        for key in ("a", "b"):
            assert np.array_equal(g[key][b, h], o[key][b, h]), "%s window %s (%d,%d)" % (what, key, b, h)
        for key in ("as", "bs"):
            assert np.array_equal(g[key][b, h].view(np.uint32), o[key][b, h].view(np.uint32)), \
                "%s window %s (%d,%d)" % (what, key, b, h)


def _run(w, bits, Wn, rounding, steps, heads=None):
    run = Run(w, bits, rounding=rounding)
    ctx = rsq.Context(rsq.RSQ_GDN, run.B, run.H, run.dk, run.dv, head_bits=bits, rounding=rounding,
                      in_dtype=run.in_dtype, seed=run.seed, window=Wn)
    st = run.zero()
    win = oracle.zero_window(run.B, run.H, Wn, run.dk, run.dv)
    g_in, g_out = run.upload(st), run.upload(st)
    wg = [_upload_window(win, run.dv), _upload_window(win, run.dv)]
    sel = heads if heads is not None else [(b, h) for b in range(run.B) for h in range(run.H)]
    for t in range(steps):
        inp = run.inputs(t)
        ins, keep = run.dev_inputs(inp)
        out = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
        ctx.decode_step_window(g_in, g_out, wg[t % 2], wg[(t + 1) % 2], ins, out, t)
        torch.cuda.synchronize()
        st, win, o = oracle.gdn_pw_step(st, win, inp, bits, rounding=rounding, seed=run.seed, step=t,
                                        heads=heads)
        assert_state_equal(run.download(g_out, heads=heads), st, bits, heads=heads, what="step %d" % t)
        assert_out_equal(host(out), o, heads=heads, what="step %d" % t)
        _assert_window_equal(_download_window(wg[(t + 1) % 2], run.dv), win, sel, "step %d" % t)
        g_in, g_out = g_out, g_in
        del keep
    ctx.close()


@pytest.mark.parametrize("Wn", [4, 8, 16])
@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_window_bit_exact(Wn, rounding):
    w = dataclasses.replace(W.WORKLOADS[1], B=3, H=4)
    _run(w, np.array([4, 8, 4, 4], np.int8), Wn, rounding, 2 * Wn + 3)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 256)])
def test_window_shapes(dk, dv):
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3, dk=dk, dv=dv)
    _run(w, np.array([4, 8, 4], np.int8), 4, rsq.RSQ_SR, 10)


def test_window_full_precision_history():
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3)
    _run(w, np.full(3, 32, np.int8), 8, rsq.RSQ_RTN, 19)


def test_window_full_size_sampled_heads():
    """The INT4 long-horizon shape at full batch with an 8-slot window, in the
    benchmark's launch configuration; the oracle computes sampled heads."""
    w = W.WORKLOADS[4]
    heads = sample_heads(w.B, w.H, 24, seed=6)
    _run(w, np.full(w.H, 4, np.int8), 8, rsq.RSQ_SR, 10, heads=heads)


def test_window_entry_points_checked():
    w = dataclasses.replace(W.WORKLOADS[1], B=1, H=2)
    run = Run(w, np.array([8, 4], np.int8))
    ctx = rsq.Context(rsq.RSQ_GDN, 1, 2, 128, 128, head_bits=[8, 4], window=4)
    st = run.upload(run.zero())
    ins, keep = run.dev_inputs(run.inputs(0))
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(rsq.RsqError) as e:
        ctx.decode_step(st, st, ins, out, 0)          # a windowed context needs the window entry
    assert e.value.status == rsq.RSQ_E_INVAL
    win = ctx.alloc_window()
    with pytest.raises(rsq.RsqError) as e:
        ctx.decode_step_window(st, st, win, win, ins, out, 0)   # in and out must differ
    assert e.value.status == rsq.RSQ_E_INVAL
    a, b, sc = rsq.rsq_window_bytes(ctx.ctx)
    assert (a, b, sc) == (1 * 2 * 4 * 128, 1 * 2 * 4 * 128, 1 * 2 * 4 * 4)
    ctx.close()


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rounding", [rsq.RSQ_SR8, rsq.RSQ_RTN])
def test_window_against_the_literal_order(bits, rounding):
    """The low-bit history of a window state against the oracle's literal order
    at the method's tolerance, teacher-forced through the first merges (8 slots):
    each step starts the GPU and both oracle orders from the canonical state,
    which the GPU matches bit for bit.  The window's own arithmetic (the slot
    propagation and its FP8 codes) is the same in both orders and must agree
    exactly; of the history's codes at most 1e-5 differ, each by one step, apart
    from nearest-rounding boundary cases (1e-3), judged against the literal
    order's full-precision history after the merge."""
    import plain_order
    Wn = 8
    w = dataclasses.replace(W.WORKLOADS[1], B=8)
    hb = np.full(w.H, bits, np.int8)
    b32 = np.full(w.H, 32, np.int8)
    run = Run(w, hb, rounding=rounding)
    ctx = rsq.Context(rsq.RSQ_GDN, run.B, run.H, run.dk, run.dv, head_bits=hb, rounding=rounding,
                      in_dtype=run.in_dtype, seed=run.seed, window=Wn)
    st = run.zero()
    win = oracle.zero_window(run.B, run.H, Wn, run.dk, run.dv)
    allh = [(b, h) for b in range(run.B) for h in range(run.H)]
    n_other = n_tie = n_tot = 0
    for t in range(Wn + 3):
        inp = run.inputs(t)
        ins, keep = run.dev_inputs(inp)
        out = torch.empty((run.B, run.H, run.dv), dtype=torch.float32, device="cuda")
        g_in, g_out = run.upload(st), run.upload(st)
        w_in, w_out = _upload_window(win, run.dv), _upload_window(win, run.dv)
        ctx.decode_step_window(g_in, g_out, w_in, w_out, ins, out, t)
        torch.cuda.synchronize()
        gpu, gwin = run.download(g_out), _download_window(w_out, run.dv)
        canon, cwin, co = oracle.gdn_pw_step(st, win, inp, hb, rounding=rounding, seed=run.seed, step=t)
        assert_state_equal(gpu, canon, hb, what="step %d" % t)
        assert_out_equal(host(out), co, what="step %d" % t)
        _assert_window_equal(gwin, cwin, allh, "step %d" % t)
        plain, pwin, po = oracle.gdn_pw_step(st, win, inp, hb, rounding=rounding, seed=run.seed, step=t,
                                             mode=oracle.PLAIN)
        _assert_window_equal(pwin, cwin, allh, "step %d (literal order)" % t)
        f = oracle.zero_state(run.B, run.H, run.dk, run.dv, fp32=True)
        f["f"] = oracle.dequantize(st, hb)
        lit, _, _ = oracle.gdn_pw_step(f, win, inp, b32, rounding=oracle.RTN, seed=0, step=t, mode=oracle.PLAIN)
        o, ti, tot = plain_order.compare_codes(gpu["codes"], plain["codes"], lit["f"], hb,
                                               nearest=rounding == rsq.RSQ_RTN)
        n_other, n_tie, n_tot = n_other + o, n_tie + ti, n_tot + tot
        assert np.allclose(gpu["scales"], plain["scales"], rtol=1e-5, atol=0)
        assert plain_order.max_rel(host(out), po) <= 1e-3
        st, win = canon, cwin
        del keep
    ctx.close()
    assert n_tot > 0
    assert n_other <= 1e-5 * n_tot, (n_other, n_tie, n_tot)
    assert n_tie <= 1e-3 * n_tot, (n_other, n_tie, n_tot)
