"""GPU parity of ART early termination of the Phase-2 key walk (ART review
page; opt-in approximation).  With zero thresholds every block is visited
and the result equals exact attention; with keys whose weights underflow
the walk stops after 1 + patience blocks exactly like the oracle; on the
128K decode shape with the page's defaults and on a recency-shaped cache the
visited block counts and outputs equal the oracle's."""
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
    # N(0, 1) caches never settle: the relative change of the probe per block
    # stays near 1/t, far above tau = 1e-5, so kernel and oracle both walk
    # every block; visited counts and outputs are compared with the oracle's
    w = workloads.DECODE_128K
    q, kc, vc = w.decode_inputs(device=DEV)
    T, g = w.decode_T, w.hq // w.hkv
    o, lse, vis, ws = P.star_phase2_attend_art(q, kc, vc, T, w.rope_theta)
    assert P.pa_workspace_status(ws) == 0
    vis = vis.cpu().numpy()
    for b, kvh in ((0, 0), (7, 3), (15, 7)):
        hs = slice(kvh * g, (kvh + 1) * g)
        qs = f64(q[b:b + 1, :, hs])
        ks = f64(kc[b:b + 1, :, kvh:kvh + 1])
        vs = f64(vc[b:b + 1, :, kvh:kvh + 1])
        ro, rl, rv = oracle.phase2_attend_art(qs, ks, vs, T, w.rope_theta)
        assert int(vis[b, kvh]) == int(rv[0, 0])
        assert_close(f64(o[b:b + 1, :, hs].cpu()), ro, TOL, "O")
        assert_close(lse[b:b + 1, :, hs].cpu().double().numpy(), rl, LSE_TOL, "lse")


def test_recency_cache_stops_like_the_oracle(P):
    # keys older than the newest W move by -60 along the normalised sum of
    # their group's query vectors, so their softmax weights are about e^-30:
    # the probe changes by O(1/t) while the recent blocks come in and by
    # about e^-30 after them, both far from tau and phi.  The stop block must
    # equal the oracle's, and the output the oracle's attention over the
    # keys it visited.
    B, hq, hkv, d, T, W = 2, 32, 8, 128, 16384, 1024
    g = hq // hkv
    q = workloads.normal((B, 1, hq, d), 105, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 106, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 107, torch.bfloat16)
    u = q.float().view(B, 1, hkv, g, d).sum(3)
    u = u / u.norm(dim=-1, keepdim=True)
    for b in range(B):
        kc[b, :T - W] = (kc[b, :T - W].float() - 60.0 * u[b]).to(torch.bfloat16)
    o, lse, vis, ws = P.star_phase2_attend_art(q.to(DEV), kc.to(DEV), vc.to(DEV), T, 0.0)
    assert P.pa_workspace_status(ws) == 0
    ro, rl, rv = oracle.phase2_attend_art(f64(q), f64(kc), f64(vc), T, 0.0)
    assert (rv < T // 128).all() and (rv >= W // 128).all()
    assert (vis.cpu().numpy() == rv).all()
    assert_close(f64(o.cpu()), ro, TOL, "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
