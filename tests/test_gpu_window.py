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
