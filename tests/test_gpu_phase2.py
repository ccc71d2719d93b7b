"""GPU parity of Phase-2 split-KV attention and the exact LSE merge against
the fp64 oracle (Pulsar Attention page §2.2; Star Attention review,
Algorithm 2 as corrected): per-shard partials and merged outputs at small
sizes, and sampled (batch, kv-head) groups of the 128K decode, the 128K
64-token query and the 1M-token decode."""
import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def _oracle_group(q, kc, vc, b, kvh, g, n_shards, q_pos0, theta):
    """Oracle for one (batch, kv head) group: its g query heads only."""
    qs = f64(q[b:b + 1, :, kvh * g:(kvh + 1) * g, :])
    ks = f64(kc[b:b + 1, :, kvh:kvh + 1, :])
    vs = f64(vc[b:b + 1, :, kvh:kvh + 1, :])
    return oracle.phase2_attend(qs, ks, vs, n_shards, q_pos0, theta)


def test_tiny_fp32_full(P):
    w = workloads.TINY
    B, T, S = 2, w.L, w.n_blocks
    q = workloads.normal((B, w.q_tokens, w.hq, w.d), 50, torch.float32)
    kc = workloads.normal((B, T, w.hkv, w.d), 51, torch.float32)
    vc = workloads.normal((B, T, w.hkv, w.d), 52, torch.float32)
    o, lse, po, pl, ws = P.star_phase2_attend(q.to(DEV), kc.to(DEV), vc.to(DEV), S, q_pos0=T,
                                              rope_theta=w.rope_theta, want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    ro, rl, ra, rs = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, w.rope_theta)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.float32], "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
    assert_close(po.cpu().double().numpy(), ra, O_TOL[torch.float32], "A_h")
    assert_close(pl.cpu().double().numpy(), rs, LSE_TOL, "s_h")


@pytest.mark.parametrize("case", [
    # (B, Tq, T, S, hq, hkv, d, theta)
    (1, 64, 3000, 5, 8, 2, 128, 500000.0),     # ragged shards, a 64-token query
    (3, 1, 999, 4, 32, 8, 128, 500000.0),      # decode rows, ragged cache
    (2, 7, 10, 16, 4, 4, 64, 0.0),             # more shards than keys: empty shards, no RoPE
    (1, 3, 0, 2, 4, 2, 64, 10000.0),           # empty cache: O = 0, lse = -inf
    (2, 20, 700, 3, 8, 2, 64, 10000.0),        # d = 64, 80 rows per kv head (tensor-core kernel)
    (1, 2, 5000, 4096, 4, 1, 128, 500000.0),   # the largest shard count: most shards of 1-2 keys
    # tensor-core query kernel (>= 64 rows per kv head, 128 % g == 0)
    (1, 48, 2000, 3, 16, 2, 128, 500000.0),    # g = 8, 384 rows: 3 row tiles, a half-empty tile pair
    (2, 100, 1500, 2, 4, 4, 64, 10000.0),      # g = 1, 100 rows, two batch elements
    (1, 80, 777, 4, 32, 2, 128, 500000.0),     # g = 16, 1280 rows: 5 tile pairs share each unit
    (1, 64, 20, 8, 8, 2, 128, 10000.0),        # 256 rows over 20 keys: 3-key shards, one empty
    (1, 64, 0, 2, 8, 2, 64, 10000.0),          # 256 rows, empty cache: O = 0, lse = -inf
    # row-split mma.sync kernel
    (1, 30, 500, 2, 6, 2, 64, 10000.0),        # g = 3 does not divide 128
    (1, 12, 900, 3, 8, 2, 128, 500000.0),      # 48 rows per kv head
])
def test_bf16_small_full(P, case):
    B, Tq, T, S, hq, hkv, d, theta = case
    q = workloads.normal((B, Tq, hq, d), 60, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 61, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 62, torch.bfloat16)
    o, lse, po, pl, ws = P.star_phase2_attend(q.to(DEV), kc.to(DEV), vc.to(DEV), S, q_pos0=T,
                                              rope_theta=theta, want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    ro, rl, ra, rs = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, theta)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.bfloat16], "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
    assert_close(po.cpu().double().numpy(), ra, O_TOL[torch.bfloat16], "A_h")
    assert_close(pl.cpu().double().numpy(), rs, LSE_TOL, "s_h")


def test_query_kernel_running_max_jumps(P):
    # A 64-token query with g = 4 (256 rows per kv head: the tensor-core
    # kernel) over two 512-key shards, one unit each.  For the odd query heads
    # the first 128 keys of each shard score about 7 nat lower, so those rows'
    # running max jumps by more than 2^8 at the unit's second key tile (the
    # lazy-rescale branch), while the even heads' rows, in the same warps, keep
    # theirs.  No RoPE, so the shifted dimensions stay as written.
    B, Tq, T, S, hq, hkv, d = 1, 64, 1024, 2, 8, 2, 128
    q = workloads.normal((B, Tq, hq, d), 63, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 64, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 65, torch.bfloat16)
    rng = np.random.default_rng(6)
    idx = torch.arange(96, 128)
    t = np.arange(T)
    kx = ((t % 512) < 128)[None, :, None, None] * -2.5 * (1.0 + 0.25 * rng.standard_normal((B, T, hkv, 32)))
    qx = (np.arange(hq) % 2 == 1)[None, None, :, None] * (1.0 + 0.25 * rng.standard_normal((B, Tq, hq, 32)))
    kc[..., idx] = torch.from_numpy(kx).to(torch.bfloat16)
    q[..., idx] = torch.from_numpy(qx).to(torch.bfloat16)
    o, lse, po, pl, ws = P.star_phase2_attend(q.to(DEV), kc.to(DEV), vc.to(DEV), S, q_pos0=T, rope_theta=0.0,
                                              want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    ro, rl, ra, rs = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, 0.0)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.bfloat16], "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
    assert_close(po.cpu().double().numpy(), ra, O_TOL[torch.bfloat16], "A_h")
    assert_close(pl.cpu().double().numpy(), rs, LSE_TOL, "s_h")


@pytest.mark.parametrize("wname,groups", [
    ("decode_128k_b16", [(0, 0), (9, 5), (15, 7)]),
    ("scale_1m", [(0, 3), (3, 7)]),
])
def test_decode_sampled_groups(P, wname, groups):
    w = workloads.WORKLOADS[wname]
    q, kc, vc = w.decode_inputs(device=DEV)
    T, S, g = w.decode_T, w.decode_shards, w.hq // w.hkv
    o, lse, po, pl, ws = P.star_phase2_attend(q, kc, vc, S, q_pos0=T, rope_theta=w.rope_theta,
                                              want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    for b, kvh in groups:
        ro, rl, ra, rs = _oracle_group(q, kc, vc, b, kvh, g, S, T, w.rope_theta)
        hs = slice(kvh * g, (kvh + 1) * g)
        assert_close(f64(o[b:b + 1, :, hs].cpu()), ro, O_TOL[torch.bfloat16], "O")
        assert_close(lse[b:b + 1, :, hs].cpu().double().numpy(), rl, LSE_TOL, "lse")
        assert_close(pl[b:b + 1, :, :, hs].cpu().double().numpy(), rs, LSE_TOL, "s_h")
        assert_close(f64(po[b:b + 1, :, :, hs].cpu()), ra, O_TOL[torch.bfloat16], "A_h")


def test_query_128k_sampled_groups(P):
    w = workloads.LLAMA_128K
    q = w.query(device=DEV)
    kc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_KC, w.dtype, DEV)
    vc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_VC, w.dtype, DEV)
    o, lse, _, _, ws = P.star_phase2_attend(q, kc, vc, w.n_blocks, q_pos0=w.L, rope_theta=w.rope_theta)
    assert P.pa_workspace_status(ws) == 0
    g = w.hq // w.hkv
    for kvh in (0, 6):
        ro, rl, _, _ = _oracle_group(q, kc, vc, 0, kvh, g, w.n_blocks, w.L, w.rope_theta)
        hs = slice(kvh * g, (kvh + 1) * g)
        assert_close(f64(o[:, :, hs].cpu()), ro, O_TOL[torch.bfloat16], "O")
        assert_close(lse[:, :, hs].cpu().double().numpy(), rl, LSE_TOL, "lse")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_lse_merge_entry_point(P, dtype):
    # pa_lse_merge fed partials the oracle computed (fp64 -> fp32), with whole
    # shards empty (s_h = -inf, A_h garbage that must be ignored) next to
    # finite ones, and rows whose shards are all empty, against the oracle's
    # merge of the same partials
    B, S, Tq, hq, hkv, d, T = 2, 6, 3, 8, 2, 128, 900
    q = workloads.normal((B, Tq, hq, d), 70, torch.float32)
    kc = workloads.normal((B, T, hkv, d), 71, torch.float32)
    vc = workloads.normal((B, T, hkv, d), 72, torch.float32)
    A, s = oracle.phase2_partials(f64(q), f64(kc), f64(vc), S)
    s[0, 2] = -np.inf                    # shard 2 of batch 0 empty for every row
    s[1, :, 1, 3] = -np.inf              # batch 1, token 1, head 3: every shard empty
    s[1, 4, 2, :] = -np.inf              # batch 1, shard 4, token 2: empty for every head
    s[0, 1] += 3.0                       # shards of very different weight
    s[1, 0, 0] -= 40.0
    A_in = A.copy()
    A_in[np.isneginf(s)] = 1.0e30        # values of empty shards are ignored
    po = torch.from_numpy(A_in).float().to(DEV)
    pl = torch.from_numpy(s).float().to(DEV)
    o, lse = P.pa_lse_merge(po, pl, dtype=dtype)
    ro, rl = oracle.lse_merge(A, s)
    assert_close(f64(o.cpu()), ro, O_TOL[dtype], "O")
    fin = np.isfinite(rl)
    assert (~fin).sum() == 1 and torch.isneginf(lse.cpu()[torch.from_numpy(~fin)]).all()
    assert (o.cpu().float()[torch.from_numpy(~fin)] == 0).all()
    assert np.abs(lse.cpu().double().numpy()[fin] - rl[fin]).max() <= LSE_TOL


@pytest.mark.parametrize("where,d", [("key", 128), ("query", 128), ("key", 64), ("both", 128)])
def test_query_kernel_values_beyond_fp16(P, where, d):
    # the tensor-core query kernel carries the query and the keys in fp16; a
    # unit that meets a key beyond fp16 range (any unit, when the scaled
    # rotated query is) is recomputed in fp32, so bf16 inputs of any size give
    # the right result (status PA_OK).  Scores here reach ~10^5 nat, and fp32
    # sums of d products of that size carry a rounding of about
    # |s| * 2^-24 * sqrt(d): the lse tolerance grows as 2^-20 |lse| beyond the
    # stated 1e-3 (below 1e-3 for every score of normal-range inputs).
    B, Tq, hq, hkv, T, S = 1, 64, 8, 2, 700, 3    # 256 rows per kv head: the tensor-core kernel
    q = workloads.normal((B, Tq, hq, d), 90, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 91, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 92, torch.bfloat16)
    if where in ("key", "both"):
        kc[0, 321, 1, 7] = 7.0e4      # beyond 65504: its unit is recomputed
        kc[0, 650, 0, 3] = -9.0e4
    if where in ("query", "both"):
        q[0, 5, 3, 9] = 6.0e5         # x log2(e)/sqrt(d) is beyond 65504: every unit is recomputed
    o, lse, po, pl, ws = P.star_phase2_attend(q.to(DEV), kc.to(DEV), vc.to(DEV), S, q_pos0=T, rope_theta=0.0,
                                              want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    ro, rl, ra, rs = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, 0.0)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.bfloat16], "O")
    assert_close(f64(po.cpu()), ra, O_TOL[torch.bfloat16], "A_h")
    for got, want, what in ((lse.cpu().double().numpy(), rl, "lse"), (pl.cpu().double().numpy(), rs, "s_h")):
        fin = np.isfinite(want)
        err = np.abs(got[fin] - want[fin])
        assert (err <= LSE_TOL + 2.0 ** -20 * np.abs(want[fin])).all(), (what, float(err.max()))
    # the same inputs within range still run the tensor-core path alone
    kc[0, 321, 1, 7], kc[0, 650, 0, 3], q[0, 5, 3, 9] = 1.0, -1.0, 1.0
    o2, lse2, _, _, ws = P.star_phase2_attend(q.to(DEV), kc.to(DEV), vc.to(DEV), S, q_pos0=T, rope_theta=0.0)
    assert P.pa_workspace_status(ws) == 0
    ro2, rl2, _, _ = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, 0.0)
    assert_close(f64(o2.cpu()), ro2, O_TOL[torch.bfloat16], "O in range")
    assert_close(lse2.cpu().double().numpy(), rl2, LSE_TOL, "lse in range")


def test_query_step_own_key_beyond_fp16(P):
    # a generated token's key beyond fp16 range lands in the query host's own
    # cache; the own-cache unit is recomputed exactly like a shard's
    B, Tq, hq, hkv, d, T, S, cap = 1, 64, 8, 2, 128, 500, 2, 80
    dt = torch.bfloat16
    q = workloads.normal((B, Tq, hq, d), 93, dt)
    kn = workloads.normal((B, Tq, hkv, d), 94, dt)
    vn = workloads.normal((B, Tq, hkv, d), 95, dt)
    kc = workloads.normal((B, T, hkv, d), 96, dt)
    vc = workloads.normal((B, T, hkv, d), 97, dt)
    kn[0, 10, 1, 4] = 8.0e4
    ks = torch.zeros((B, cap, hkv, d), dtype=dt, device=DEV)
    vs = torch.zeros_like(ks)
    o, lse, ws = P.star_phase2_query_step(q.to(DEV), kn.to(DEV), vn.to(DEV), kc.to(DEV), vc.to(DEV), S, ks, vs, 0,
                                          T, 0.0)
    assert P.pa_workspace_status(ws) == 0
    ro, rl = oracle.phase2_attend_with_self(f64(q), f64(kc), f64(vc), S, f64(kn), f64(vn), 0, T, 0.0)
    assert_close(f64(o.cpu()), ro, O_TOL[dt], "O")
    err = np.abs(lse.cpu().double().numpy() - rl)
    assert (err <= LSE_TOL + 2.0 ** -20 * np.abs(rl)).all(), float(err.max())


def test_query_32k_sampled_groups(P):
    # the 32K workload's 64-token query over its 4 retained blocks (the
    # tensor-core query kernel: 256 rows per kv head, 4 splits per shard)
    w = workloads.LLAMA_32K
    q = w.query(device=DEV)
    kc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_KC, w.dtype, DEV)
    vc = workloads.normal((1, w.L, w.hkv, w.d), workloads.SEED_VC, w.dtype, DEV)
    o, lse, po, pl, ws = P.star_phase2_attend(q, kc, vc, w.n_blocks, q_pos0=w.L, rope_theta=w.rope_theta,
                                              want_partials=True)
    assert P.pa_workspace_status(ws) == 0
    g = w.hq // w.hkv
    for kvh in (1, 7):
        ro, rl, ra, rs = _oracle_group(q, kc, vc, 0, kvh, g, w.n_blocks, w.L, w.rope_theta)
        hs = slice(kvh * g, (kvh + 1) * g)
        assert_close(f64(o[:, :, hs].cpu()), ro, O_TOL[torch.bfloat16], "O")
        assert_close(lse[:, :, hs].cpu().double().numpy(), rl, LSE_TOL, "lse")
        assert_close(f64(po[:, :, :, hs].cpu()), ra, O_TOL[torch.bfloat16], "A_h")
        assert_close(pl[:, :, :, hs].cpu().double().numpy(), rs, LSE_TOL, "s_h")
