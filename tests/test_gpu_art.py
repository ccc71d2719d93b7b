"""GPU parity of ART early termination of the Phase-2 key walk (ART review
page; opt-in approximation).  With zero thresholds every block is visited
and the result equals exact attention; with keys whose weights underflow
the walk stops after 1 + patience blocks exactly like the oracle; on the
128K decode shape with the page's defaults the output equals the oracle's
attention over the keys the kernel reports it visited."""
import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = O_TOL[torch.bfloat16]


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def test_zero_thresholds_visit_everything(P):
    B, hq, hkv, d, T = 3, 32, 8, 128, 2000
    q = workloads.normal((B, 1, hq, d), 100, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 101, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 102, torch.bfloat16)
    o, lse, vis, ws = P.star_phase2_attend_art(q.to(DEV), kc.to(DEV), vc.to(DEV), T, 5e5, block_keys=128, tau=0.0,
                                               phi=0.0, patience=2)
    assert P.pa_workspace_status(ws) == 0
    assert (vis.cpu() == (T + 127) // 128).all()
    ro, rl, _, _ = oracle.phase2_attend(f64(q), f64(kc), f64(vc), 1, T, 5e5)
    assert_close(f64(o.cpu()), ro, TOL, "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")


def test_stops_after_patience_like_the_oracle(P):
    B, hq, hkv, d, bk, pat = 2, 8, 2, 128, 128, 3
    T = 10 * bk
    q = torch.zeros((B, 1, hq, d))
    q[..., 0] = 1.0
    kc = workloads.normal((B, T, hkv, d), 103, torch.float32) * 0.1
    kc[:, :T - bk, :, 0] = -1000.0 * d ** 0.5      # older keys: weights underflow to 0
    vc = workloads.normal((B, T, hkv, d), 104, torch.float32)
    q, kc, vc = q.bfloat16(), kc.bfloat16(), vc.bfloat16()
    o, lse, vis, _ = P.star_phase2_attend_art(q.to(DEV), kc.to(DEV), vc.to(DEV), T, 0.0, block_keys=bk, tau=1e-5,
                                              phi=1e-3, patience=pat)
    ro, rl, rv = oracle.phase2_attend_art(f64(q), f64(kc), f64(vc), T, 0.0, bk, 1e-5, 1e-3, pat)
    assert (vis.cpu().numpy() == rv).all() and (rv == 1 + pat).all()
    assert_close(f64(o.cpu()), ro, TOL, "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")


def test_decode_128k_defaults_sampled(P):
    w = workloads.DECODE_128K
    q, kc, vc = w.decode_inputs(device=DEV)
    T, g = w.decode_T, w.hq // w.hkv
    o, lse, vis, _ = P.star_phase2_attend_art(q, kc, vc, T, w.rope_theta)
    vis = vis.cpu().numpy()
    for b, kvh in ((0, 0), (7, 3), (15, 7)):
        n = min(T, int(vis[b, kvh]) * 128)
        hs = slice(kvh * g, (kvh + 1) * g)
        qs = f64(q[b:b + 1, :, hs])
        ks = f64(kc[b:b + 1, T - n:, kvh:kvh + 1])
        vs = f64(vc[b:b + 1, T - n:, kvh:kvh + 1])
        ro, rl, _, _ = oracle.phase2_attend(qs, ks, vs, 1, T, w.rope_theta)
        assert_close(f64(o[b:b + 1, :, hs].cpu()), ro, TOL, "O")
        assert_close(lse[b:b + 1, :, hs].cpu().double().numpy(), rl, LSE_TOL, "lse")
