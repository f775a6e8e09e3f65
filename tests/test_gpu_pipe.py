"""The host-buffer pipeline (rsq_pipe) against the device-buffer entry points.

Over several steps with three steps in flight, the pipe (packed pinned host
inputs copied in, the decode step, the output copied back) must leave the same
states and produce the same outputs, bit for bit, as rsq_decode_step on device
inputs -- which the other GPU tests hold to the oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, dev, host

pytestmark = pytest.mark.gpu


def _state_from(st, bits):
    return rsq.State(dev(oracle.pack_state(st, bits)), dev(np.ascontiguousarray(st["scales"], np.float32)))


def _window(win, dv):
    B, H, Wn, _ = win["b"].shape
    b = np.ascontiguousarray(win["b"].reshape(B, H, Wn, dv // 16, 16).transpose(0, 1, 3, 2, 4))
    return rsq.Window(dev(win["a"]), dev(win["as"]), dev(b), dev(win["bs"]))


CASES = {
    "gdn_mixed": dict(base=W.WORKLOADS[1], B=5, H=4, dk=128, dv=128, bits=[8, 4, 4, 8]),
    "gdn_f32_inputs": dict(base=dataclasses.replace(W.WORKLOADS[1], in_dtype="f32"), B=3, H=2, dk=64, dv=32,
                           bits=[4, 8]),
    "mamba2": dict(base=W.WORKLOADS[3], B=3, H=6, dk=64, dv=64, bits=[8, 4, 8, 4, 8, 4], ngroups=3),
    "gla": dict(base=W.BY_NAME["gla_b64_h16_d128_int8_sr"], B=2, H=3, dk=64, dv=64, bits=[8, 4, 8]),
    "kda": dict(base=W.BY_NAME["kda_b64_h16_d128_int8_sr"], B=2, H=3, dk=64, dv=64, bits=[4, 8, 4]),
    "fp32": dict(base=W.WORKLOADS[1], B=2, H=3, dk=32, dv=64, bits=[32, 32, 32]),
    "window": dict(base=W.WORKLOADS[1], B=2, H=3, dk=64, dv=64, bits=[8, 4, 8], window=4),
    "key_axis": dict(base=W.WORKLOADS[1], B=2, H=3, dk=64, dv=32, bits=[8, 4, 8], key_axis=1),
    "dk256": dict(base=W.WORKLOADS[1], B=2, H=3, dk=256, dv=64, bits=[8, 4, 8]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_pipe_matches_device_entry_points(name):
    c = CASES[name]
    w = dataclasses.replace(c["base"], B=c["B"], H=c["H"], dk=c["dk"], dv=c["dv"], ngroups=c.get("ngroups", 1))
    bits = np.array(c["bits"], np.int8)
    Wn, ka = c.get("window", 0), c.get("key_axis", 0)
    run = Run(w, bits)
    ctx = rsq.Context(run.family, w.B, w.H, w.dk, w.dv, head_bits=bits, rounding=run.rounding,
                      in_dtype=run.in_dtype, seed=run.seed, ngroups=w.ngroups, window=Wn, key_axis=ka)
    rng = np.random.default_rng(len(name))
    S = (rng.standard_normal((w.B, w.H, w.dk, w.dv)) * 0.3).astype(np.float32)
    if ka:
        st = oracle.quantize_ka(S, bits, rounding=oracle.SR, seed=1, step=0)
    elif run.f32:
        st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
        st["f"] = S
    else:
        st = oracle.quantize(S, bits, rounding=oracle.SR, seed=1, step=0)
    a = [_state_from(st, bits), _state_from(st, bits)]
    b = [_state_from(st, bits), _state_from(st, bits)]
    wa = wb = None
    if Wn:
        win = oracle.zero_window(w.B, w.H, Wn, w.dk, w.dv)
        wa = [_window(win, w.dv), _window(win, w.dv)]
        wb = [_window(win, w.dv), _window(win, w.dv)]
    torch.cuda.synchronize()        # uploads done before the pipe's own streams start
    pipe = rsq.Pipe(ctx)
    steps = 7                       # more than the 3 steps in flight: every slot reused
    host_in, host_out, want = [], [], []
    for t in range(steps):
        inp = run.inputs(t)
        # device entry point on the current stream
        ins, keep = run.dev_inputs(inp)
        out = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
        if Wn:
            ctx.decode_step_window(a[t % 2], a[(t + 1) % 2], wa[t % 2], wa[(t + 1) % 2], ins, out, t)
        else:
            ctx.decode_step(a[t % 2], a[(t + 1) % 2], ins, out, t)
        want.append(host(out))
        # the pipe, from packed pinned host buffers
        host_in.append(rsq.pack_host_inputs(ctx, inp))
        host_out.append(torch.empty((w.B, w.H, w.dv), dtype=torch.float32, pin_memory=True))
        pipe.step(b[t % 2], b[(t + 1) % 2], host_in[-1], host_out[-1], t,
                  wb[t % 2] if Wn else None, wb[(t + 1) % 2] if Wn else None)
    pipe.sync()
    torch.cuda.synchronize()
    for t in range(steps):
        assert np.array_equal(host_out[t].numpy().view(np.uint32), want[t].view(np.uint32)), "step %d output" % t
    fa, fb = a[steps % 2], b[steps % 2]
    assert np.array_equal(host(fa.codes), host(fb.codes))
    assert np.array_equal(host(fa.scales).view(np.uint32), host(fb.scales).view(np.uint32))
    if Wn:
        for x, y in zip((wa[steps % 2].a, wa[steps % 2].b), (wb[steps % 2].a, wb[steps % 2].b)):
            assert np.array_equal(host(x), host(y))
    assert ctx.check_flags() == 0
    pipe.close()


def test_pipe_layout_and_argument_checks():
    w = dataclasses.replace(W.WORKLOADS[1], B=2, H=3, dk=64, dv=32)
    ctx = rsq.Context(rsq.RSQ_GDN, 2, 3, 64, 32, head_bits=[8, 4, 8], window=4)
    off, size, total = rsq.rsq_host_input_layout(ctx.ctx)
    assert size[:5] == [2 * 3 * 64 * 2, 2 * 3 * 64 * 2, 2 * 3 * 32 * 2, 2 * 3 * 4, 2 * 3 * 4] and size[5] == 0
    assert all(o % 16 == 0 for o in off) and total >= off[4] + size[4]
    st = ctx.alloc_state()
    pipe = rsq.Pipe(ctx)
    buf = rsq.pack_host_inputs(ctx, W.inputs(w, 0))
    out = torch.empty((2, 3, 32), dtype=torch.float32, pin_memory=True)
    with pytest.raises(rsq.RsqError) as e:          # a window context needs its windows
        pipe.step(st, st, buf, out, 0)
    assert e.value.status == rsq.RSQ_E_INVAL
    with pytest.raises(ValueError):                  # host buffers only
        pipe.step(st, st, buf.cuda(), out, 0)
    pipe.close()
