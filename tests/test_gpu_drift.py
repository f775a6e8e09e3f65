"""The long-horizon drift study (bench.py --drift) against the oracle.

Every trajectory of the study -- the FP32 one (32-bit heads) and the INT4/INT8
ones with stochastic and nearest rounding -- is run free on both sides from
S_0 = 0 on the same seeded inputs; the drift ||deq(S_q) - S_fp32||_F /
||S_fp32||_F and the readout error the study reports must equal the ones
computed from the oracle's trajectories.
"""
import dataclasses
import os
import sys

import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _oracle_series(w, steps, every, variants):
    rnd = {"sr": oracle.SR8, "rtn": oracle.RTN, "bdr": oracle.BDR, "sr_bdr": oracle.SR8_BDR, "sr16": oracle.SR}
    ref = oracle.zero_state(w.B, w.H, w.dk, w.dv, fp32=True)
    qs = {lab: (oracle.zero_state_ka(w.B, w.H, w.dk, w.dv) if src == "keyaxis"
                else oracle.zero_state(w.B, w.H, w.dk, w.dv, fp32=False)) for lab, _, _, src in variants}
    wins = {lab: oracle.zero_window(w.B, w.H, int(src[1:]), w.dk, w.dv)
            for lab, _, _, src in variants if src.startswith("w")}
    out = {lab: [] for lab, _, _, _ in variants}
    f32 = np.full(w.H, 32, np.int8)
    for t in range(steps):
        inp = W.inputs(w, t)
        ref, o_ref = oracle.gdn_step(ref, inp, f32, rounding=oracle.RTN, seed=w.sr_seed, step=t)
        m = np.abs(ref["f"]).max(axis=2)
        for lab, bits, r, src in variants:
            hb = np.full(w.H, bits, np.int8)
            if lab in wins:
                qs[lab], wins[lab], o = oracle.gdn_pw_step(qs[lab], wins[lab], inp, hb, rounding=rnd[r],
                                                           seed=w.sr_seed, step=t)
            elif src == "keyaxis":
                qs[lab], o = oracle.gdn_ka_step(qs[lab], inp, hb, rounding=rnd[r], seed=w.sr_seed, step=t)
            else:
                qs[lab], o = oracle.gdn_step(qs[lab], inp, hb, rounding=rnd[r], seed=w.sr_seed, step=t,
                                             copy_absmax=m if src == "copy" else None)
            if (t + 1) % every == 0:
                F = oracle.dequantize(ref, f32).astype(np.float64)
                if lab in wins:
                    D = oracle.window_full_state(qs[lab], wins[lab], hb)
                elif src == "keyaxis":
                    D = oracle.dequantize_ka(qs[lab]).astype(np.float64)
                else:
                    D = oracle.dequantize(qs[lab], hb).astype(np.float64)
                num = ((D - F) ** 2).sum(axis=(2, 3))
                den = (F ** 2).sum(axis=(2, 3))
                o64, r64 = o.astype(np.float64), o_ref.astype(np.float64)
                out[lab].append([t + 1, np.sqrt(num.sum() / den.sum()), np.sqrt(num / den).max(),
                                 np.linalg.norm(o64 - r64) / np.linalg.norm(r64)])
    return out


def test_drift_series_matches_oracle():
    w = dataclasses.replace(W.BY_NAME["gdn_b1024_h16_d128_int4_sr_long"], B=2, H=3, dk=32, dv=32)
    steps, every = 24, 8
    got = bench.drift_series(w, steps, every)
    want = _oracle_series(w, steps, every, bench.DRIFT_VARIANTS)
    for lab, _, _, _ in bench.DRIFT_VARIANTS:
        g, e = np.array(got[lab]), np.array(want[lab])
        assert g.shape == e.shape == (steps // every, 4)
        assert np.array_equal(g[:, 0], e[:, 0])
        # the states are bit-identical; only the order of the float64 sums differs
        np.testing.assert_allclose(g[:, 1:], e[:, 1:], rtol=1e-9, atol=0)
