"""GPU parity of the diagonal-decay mixers (GLA, KDA) and of RetNet expressed
through the scalar-decay entry, against the CPU oracle.

GLA: S_t = diag(alpha) S_{t-1} + k v^T; KDA: S_t = (I - beta k k^T) diag(alpha)
S_{t-1} + beta k v^T -- the decayed mixers of the LoReS mixer zoo (Table 1).
RetNet (a constant decay per head) is the Mamba-2 step with B = k, C = q,
x = v, dt = 1, decay = gamma, D = 0 and one B/C group per head.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import ssm_decode_02_b200 as rsq
import workloads as W
from gpu_harness import Run, assert_out_equal, assert_state_equal, dev, host, sample_heads
from test_gpu_decode import _trajectory

pytestmark = pytest.mark.gpu

GLA = W.BY_NAME["gla_b64_h16_d128_int8_sr"]
KDA = W.BY_NAME["kda_b64_h16_d128_int8_sr"]


def _start(run: Run, seed: int) -> dict:
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((run.B, run.H, run.dk, run.dv)) * 0.2).astype(np.float32)
    return oracle.quantize(S, run.head_bits, rounding=run.rounding & ~oracle.BDR, seed=run.seed, step=0)


@pytest.mark.parametrize("base", [GLA, KDA], ids=["gla", "kda"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (16, 16), (32, 64), (64, 256)])
@pytest.mark.parametrize("rounding", [rsq.RSQ_RTN, rsq.RSQ_SR, rsq.RSQ_SR8])
def test_diag_bit_exact(base, dk, dv, rounding):
    w = dataclasses.replace(base, B=3, H=4, dk=dk, dv=dv)
    run = Run(w, np.array([8, 4, 4, 8], np.int8), rounding=rounding)
    _trajectory(run, 4, init=_start(run, dk * 7 + dv))


@pytest.mark.parametrize("base", [GLA, KDA], ids=["gla", "kda"])
def test_diag_fp32_state_bit_exact(base):
    w = dataclasses.replace(base, B=3, H=4)
    run = Run(w, np.full(4, 32, np.int8))
    _trajectory(run, 4)


@pytest.mark.parametrize("base", [GLA, KDA], ids=["gla", "kda"])
@pytest.mark.parametrize("rounding", [rsq.RSQ_BDR, rsq.RSQ_SR_BDR])
def test_diag_directional_rounding_bit_exact(base, rounding):
    w = dataclasses.replace(base, B=2, H=4)
    run = Run(w, np.array([4, 8, 4, 4], np.int8), rounding=rounding)
    _trajectory(run, 3, init=_start(run, 11))


@pytest.mark.parametrize("base", [GLA, KDA], ids=["gla", "kda"])
def test_diag_full_size_sampled_heads(base):
    """B=64, H=16, d=128 INT8 SR with bf16 inputs, in the benchmark's launch
    configuration; the oracle computes sampled heads."""
    run = Run(base, np.full(base.H, 8, np.int8))
    heads = sample_heads(run.B, run.H, 48, seed=5)
    _trajectory(run, 3, heads=heads)


def test_kda_plain_order_tolerance():
    """Against the literal evaluation order: at most 1e-5 of codes differ, by one step."""
    run = Run(dataclasses.replace(KDA, B=8), np.full(KDA.H, 8, np.int8))
    nd, nt = _trajectory(run, 6, check_plain=True)
    assert nd <= 1e-5 * nt, (nd, nt)


def test_retnet_through_scalar_decay_entry():
    """RetNet on the Mamba-2 entry (B = k, C = q, x = v, dt = 1, decay = gamma, D = 0,
    one group per head) equals the oracle's GLA step with the constant decay gamma."""
    w = dataclasses.replace(GLA, B=3, H=4)
    bits = np.array([8, 4, 8, 4], np.int8)
    ctx = rsq.Context(rsq.RSQ_MAMBA2, w.B, w.H, w.dk, w.dv, head_bits=bits, rounding=rsq.RSQ_SR,
                      in_dtype=rsq.RSQ_BF16, seed=w.sr_seed, ngroups=w.H)
    ref = Run(w, bits)  # packing helpers and the oracle's format
    st = oracle.zero_state(w.B, w.H, w.dk, w.dv)
    g = ref.upload(st)
    ones = dev(np.ones((w.B, w.H), np.float32))
    zeros = dev(np.zeros(w.H, np.float32))
    for t in range(4):
        inp = W.inputs(w, t)
        gamma = np.ascontiguousarray(inp["alpha"][:, :, 0])
        inp["alpha"] = np.repeat(gamma[:, :, None], w.dk, axis=2)
        q, k, v, gm = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(gamma)
        out = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device="cuda")
        ctx.decode_step(g, g, rsq.mamba2_inputs(v, k, q, ones, zeros, zeros, gm), out, t)
        torch.cuda.synchronize()
        st, o = oracle.gla_step(st, inp, bits, rounding=oracle.SR, seed=w.sr_seed, step=t)
        assert_state_equal(ref.download(g), st, bits, what="step %d" % t)
        np.testing.assert_array_equal(host(out), o)
    ctx.close()
