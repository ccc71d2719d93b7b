"""Pins for the oracle's Phase-1 and Phase-2 attention.

Against: torch's scaled_dot_product_attention in float64 (a library routine,
independent of the oracle), RoPE written as complex multiplication, closed
forms (uniform scores, single-key rows), the dense-attention identity of the
shard merge (Star Attention review: Phase 2 is exact), and the Pulsar page's
prefix and FLOP arithmetic.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rope_complex(x, pos, theta):
    """Rotary embedding as complex multiplication: z_m = x_m + i x_{m+d/2},
    z_m * exp(i p theta^(-2m/d))."""
    d = x.shape[-1]
    half = d // 2
    z = x[..., :half] + 1j * x[..., half:]
    w = np.exp(1j * np.outer(pos, theta ** (-np.arange(half) * 2.0 / d)))
    z = z * w[:, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


def _sdpa(q, k, v, causal):
    """Library attention in fp64: q [n][Hq][d], k/v [m][Hkv][d] -> [n][Hq][d]."""
    hq, hkv = q.shape[1], k.shape[1]
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).repeat_interleave(hq // hkv, dim=1).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).repeat_interleave(hq // hkv, dim=1).permute(1, 0, 2)[None]
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_rope_matches_complex_form():
    x = _rand((37, 3, 16), 1)
    pos = np.arange(37) * 7 + 3
    np.testing.assert_allclose(oracle.rope(x, pos, 10000.0), _rope_complex(x, pos, 10000.0),
                               rtol=0, atol=1e-13)


def test_rope_relative_position_invariance_and_norm():
    q, k = _rand((1, 1, 64), 2), _rand((1, 1, 64), 3)
    base = None
    for shift in (0, 1000, 131000):
        qq = oracle.rope(q, np.array([5 + shift]), 500000.0)
        kk = oracle.rope(k, np.array([2 + shift]), 500000.0)
        dot = float((qq * kk).sum())
        base = dot if base is None else base
        assert dot == pytest.approx(base, abs=1e-10)
        assert np.linalg.norm(qq) == pytest.approx(np.linalg.norm(q), rel=1e-14)


def test_causal_attention_vs_library():
    q, k, v = _rand((50, 4, 32), 4), _rand((50, 2, 32), 5), _rand((50, 2, 32), 6)
    o, lse = oracle.causal_attention(q, k, v)
    np.testing.assert_allclose(o, _sdpa(q, k, v, True), rtol=0, atol=1e-12)
    # row 0 sees one key: lse_0 = q_0 . k_0 / sqrt(d)
    for h in range(4):
        assert lse[0, h] == pytest.approx(float(q[0, h] @ k[0, h // 2]) / math.sqrt(32), abs=1e-12)
    # row subset gives the same rows
    rows = np.array([0, 7, 49, 13])
    o2, lse2 = oracle.causal_attention(q, k, v, rows)
    np.testing.assert_allclose(o2, o[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse2, lse[rows], rtol=0, atol=1e-14)


def test_uniform_scores_closed_form():
    # q = 0: every visible key scores 0, so lse_r = ln(r + 1) and o_r is the
    # mean of v_0..v_r.
    n = 40
    q = np.zeros((n, 2, 8))
    k, v = _rand((n, 1, 8), 7), _rand((n, 1, 8), 8)
    o, lse = oracle.causal_attention(q, k, v)
    r = np.arange(n)
    np.testing.assert_allclose(lse, np.log(r + 1.0)[:, None].repeat(2, 1), rtol=0, atol=1e-13)
    mean = np.cumsum(v[:, 0, :], axis=0) / (r + 1.0)[:, None]
    np.testing.assert_allclose(o[:, 0, :], mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o[:, 1, :], mean, rtol=0, atol=1e-13)


def test_single_block_reduces_to_causal_attention_with_rope():
    L, hq, hkv, d, theta = 64, 4, 2, 16, 10000.0
    q, k, v = _rand((L, hq, d), 9), _rand((L, hkv, d), 10), _rand((L, hkv, d), 11)
    pos = oracle.host_positions(L, L, 0, 8, np.zeros((1, 0), dtype=np.int64))
    assert len(pos) == 1 and pos[0].tolist() == list(range(L))
    (o, lse), = oracle.phase1_encode(q, k, v, pos, theta)
    p = np.arange(L)
    want = _sdpa(_rope_complex(q, p, theta), _rope_complex(k, p, theta), v, True)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("star", [False, True])
def test_full_context_hosts_equal_dense_rows(star):
    # Pulsar with sink 0 and a 100 % budget (every chunk of every earlier
    # block), or Star with two blocks: host i sees exactly tokens 0..(i+1)b-1
    # in order, so its B_i rows equal the dense causal rows.
    n_blocks = 2 if star else 3
    b, chunk, hq, hkv, d, theta = 32, 8, 4, 2, 16, 500000.0
    L = n_blocks * b
    q, k, v = _rand((L, hq, d), 12), _rand((L, hkv, d), 13), _rand((L, hkv, d), 14)
    sel = np.tile(np.arange(b // chunk), (n_blocks, 1))
    pos = oracle.host_positions(L, b, 0, chunk, sel, star=star)
    out = oracle.phase1_encode(q, k, v, pos, theta)
    p = np.arange(L)
    dense = _sdpa(_rope_complex(q, p, theta), _rope_complex(k, p, theta), v, True)
    for i, (o, _) in enumerate(out):
        np.testing.assert_allclose(o[-b:], dense[i * b:(i + 1) * b], rtol=0, atol=1e-12)


def test_star_and_pulsar_host_layouts():
    L, b, sink, chunk = 4 * 64, 64, 16, 8
    sel = np.array([[1, 5], [0, 7], [2, 3], [4, 6]])
    pul = oracle.host_positions(L, b, sink, chunk, sel)
    star = oracle.host_positions(L, b, sink, chunk, sel, star=True)
    assert pul[0].tolist() == list(range(64))
    assert pul[2].tolist() == (list(range(16)) + list(range(8, 16)) + list(range(40, 48))
                               + list(range(64, 72)) + list(range(120, 128)) + list(range(128, 192)))
    assert star[3].tolist() == list(range(64)) + list(range(192, 256))
    off = oracle.host_row_offsets(pul)
    assert off.tolist() == [0, 64, 64 + 96, 64 + 96 + 112, 64 + 96 + 112 + 128]


def test_flop_ratio_matches_pages():
    # Pulsar page abstract: up to 3.3x fewer Phase-1 FLOPs than Star on the
    # critical (last) host, b = 16384, four blocks, sigma = 512, 64-token sink.
    b, n = 16384, 4
    sel = np.tile(np.arange(16), (n, 1))
    pul = oracle.host_positions(n * b, b, 64, 32, sel)
    star = oracle.host_positions(n * b, b, 64, 32, sel, star=True)
    r = oracle.phase1_flops([star[-1]], 32, 128) / oracle.phase1_flops([pul[-1]], 32, 128)
    assert round(r, 1) == 3.3


def test_phase2_merge_equals_dense_attention():
    B, Tq, hq, hkv, d, T = 2, 5, 4, 2, 16, 97
    q = _rand((B, Tq, hq, d), 20)
    kc, vc = _rand((B, T, hkv, d), 21), _rand((B, T, hkv, d), 22)
    for S in (1, 3, 4, 8):
        o, lse, A, s = oracle.phase2_attend(q, kc, vc, S, q_pos0=0, theta=0.0)
        for b in range(B):
            np.testing.assert_allclose(o[b], _sdpa(q[b], kc[b], vc[b], False), rtol=0, atol=1e-12)
            sc = np.einsum("thd,nhd->thn", q[b], kc[b].repeat(2, axis=1)) / math.sqrt(d)
            ref = torch.logsumexp(torch.from_numpy(sc), dim=-1).numpy()
            np.testing.assert_allclose(lse[b], ref, rtol=0, atol=1e-12)
        if S == 1:
            np.testing.assert_allclose(A[:, 0], o, rtol=0, atol=0)
            np.testing.assert_allclose(s[:, 0], lse, rtol=0, atol=0)


def test_phase2_empty_shards_and_empty_cache():
    B, Tq, hq, hkv, d = 1, 2, 2, 1, 8
    q = _rand((B, Tq, hq, d), 30)
    kc, vc = _rand((B, 3, hkv, d), 31), _rand((B, 3, hkv, d), 32)
    o, lse, A, s = oracle.phase2_attend(q, kc, vc, 5, 0, 0.0)   # shards of 1,1,1,0,0
    assert np.isneginf(s[0, 3]).all() and np.isneginf(s[0, 4]).all()
    np.testing.assert_allclose(o[0], _sdpa(q[0], kc[0], vc[0], False), rtol=0, atol=1e-12)
    o0, lse0, _, _ = oracle.phase2_attend(q, kc[:, :0], vc[:, :0], 2, 0, 0.0)
    assert (o0 == 0).all() and np.isneginf(lse0).all()


def test_phase2_query_rotation_position():
    # The query is rotated at q_pos0 + j; against the complex form over a
    # cache rotated at 0..T-1 this is plain dense attention.
    T, hq, hkv, d, theta, p0 = 40, 2, 1, 16, 10000.0, 40
    q = _rand((1, 3, hq, d), 40)
    k, v = _rand((T, hkv, d), 41), _rand((T, hkv, d), 42)
    kr, vr = oracle.retained_kv(k, v, theta)
    np.testing.assert_allclose(kr, _rope_complex(k, np.arange(T), theta), rtol=0, atol=1e-13)
    o, _, _, _ = oracle.phase2_attend(q, kr[None], vr[None], 4, p0, theta)
    want = _sdpa(_rope_complex(q[0], p0 + np.arange(3), theta), kr, v, False)
    np.testing.assert_allclose(o[0], want, rtol=0, atol=1e-12)


def test_query_step_equals_dense_masked_attention():
    # row j sees the whole context plus own keys 0..self_off+j: compare with
    # library attention over the concatenated keys under an explicit mask
    B, Tq, hq, hkv, d, T, S, off = 2, 5, 4, 2, 16, 37, 3, 4
    q = _rand((B, Tq, hq, d), 60)
    kc, vc = _rand((B, T, hkv, d), 61), _rand((B, T, hkv, d), 62)
    ks, vs = _rand((B, off + Tq + 2, hkv, d), 63), _rand((B, off + Tq + 2, hkv, d), 64)
    o, lse = oracle.phase2_attend_with_self(q, kc, vc, S, ks, vs, off, 0, 0.0)
    for b in range(B):
        keys = np.concatenate([kc[b], ks[b, :off + Tq]])
        vals = np.concatenate([vc[b], vs[b, :off + Tq]])
        mask = np.ones((Tq, T + off + Tq), dtype=bool)
        for j in range(Tq):
            mask[j, T + off + j + 1:] = False
        tq = torch.from_numpy(q[b]).permute(1, 0, 2)[None]
        tk = torch.from_numpy(keys).repeat_interleave(2, dim=1).permute(1, 0, 2)[None]
        tv = torch.from_numpy(vals).repeat_interleave(2, dim=1).permute(1, 0, 2)[None]
        want = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask))[0].permute(1, 0, 2)
        np.testing.assert_allclose(o[b], want.numpy(), rtol=0, atol=1e-12)


def test_query_step_without_context_is_causal_attention():
    B, Tq, hq, hkv, d = 1, 9, 2, 1, 8
    q = _rand((B, Tq, hq, d), 70)
    ks, vs = _rand((B, Tq, hkv, d), 71), _rand((B, Tq, hkv, d), 72)
    o, _ = oracle.phase2_attend_with_self(q, np.zeros((B, 0, hkv, d)), np.zeros((B, 0, hkv, d)), 2, ks, vs, 0,
                                          0, 0.0)
    np.testing.assert_allclose(o[0], _sdpa(q[0], ks[0], vs[0], True), rtol=0, atol=1e-12)


def test_art_never_stable_equals_exact_attention():
    # thresholds of zero: no step is stable, every block is visited, and the
    # result is exact attention over the whole cache
    B, Tq, hq, hkv, d, T = 2, 1, 4, 2, 16, 300
    q = _rand((B, Tq, hq, d), 90)
    kc, vc = _rand((B, T, hkv, d), 91), _rand((B, T, hkv, d), 92)
    o, lse, visited = oracle.phase2_attend_art(q, kc, vc, 0, 0.0, block_keys=64, tau=0.0, phi=0.0, patience=3)
    assert (visited == 5).all()
    for b in range(B):
        np.testing.assert_allclose(o[b], _sdpa(q[b], kc[b], vc[b], False), rtol=0, atol=1e-12)


def test_art_stops_after_patience_when_old_keys_carry_no_weight():
    # keys older than the newest block score -1000 below it: their weights
    # underflow to exactly 0, every later step is exactly stable, so the walk
    # stops after 1 + patience blocks and equals attention over the newest block
    B, Tq, hq, hkv, d, T, bk, pat = 1, 2, 2, 1, 8, 64 * 10, 64, 3
    q = np.zeros((B, Tq, hq, d))
    q[..., 0] = 1.0
    kc = _rand((B, T, hkv, d), 93) * 0.1
    kc[0, :T - bk, 0, 0] = -1000.0 * np.sqrt(d)      # q.k / sqrt(d) = -1000 for old keys
    vc = _rand((B, T, hkv, d), 94)
    o, lse, visited = oracle.phase2_attend_art(q, kc, vc, 0, 0.0, block_keys=bk, tau=1e-5, phi=1e-3, patience=pat)
    assert visited[0, 0] == 1 + pat
    want = _sdpa(q[0], kc[0, T - bk:], vc[0, T - bk:], False)
    np.testing.assert_allclose(o[0], want, rtol=0, atol=1e-12)
