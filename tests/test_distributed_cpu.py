"""The multi-GPU layout across ranks, on CPU with the gloo backend: Phase 1
with the hosts spread over ranks (Pulsar page §2.1: no communication), and
the Phase-2 exchange (§2.2: partials are all-gathered, then merged exactly).
The per-rank compute steps come from the oracle, so these tests check the
host and shard partitions, packing, gather order and padding of
long_context_blockwise_max_b200.distributed against the oracle run on one
process."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_partials(q, k, v, n_local, q_pos0, theta):
    import oracle
    qn = q.double().numpy()
    if theta > 0:
        pos = q_pos0 + np.arange(qn.shape[1])
        qn = np.stack([oracle.rope(qn[b], pos, theta) for b in range(qn.shape[0])])
    A, s = oracle.phase2_partials(qn, k.double().numpy(), v.double().numpy(), n_local)
    return torch.from_numpy(A).float(), torch.from_numpy(s).float()


def _oracle_merge(part_o, part_lse, dtype):
    import oracle
    o, lse = oracle.lse_merge(part_o.double().numpy(), part_lse.double().numpy())
    return torch.from_numpy(o), torch.from_numpy(lse)


def _worker(rank, world, port, n_shards, out):
    sys.path.insert(0, ROOT)
    from long_context_blockwise_max_b200 import distributed as D
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(5)
        B, Tq, hq, hkv, d, shard = 2, 3, 4, 2, 16, 10
        q = torch.randn(B, Tq, hq, d, generator=g)
        kc = torch.randn(B, n_shards * shard, hkv, d, generator=g)
        vc = torch.randn(B, n_shards * shard, hkv, d, generator=g)
        lo, hi = D.shard_ranges(n_shards, world)[rank]
        o, lse = D.phase2_attend_distributed(q, kc[:, lo * shard:hi * shard], vc[:, lo * shard:hi * shard], hi - lo,
                                             n_shards, 100, 10000.0, partials_fn=_oracle_partials,
                                             merge_fn=_oracle_merge)
        out[rank] = (o.numpy(), lse.numpy(), q.numpy(), kc.numpy(), vc.numpy())
    finally:
        dist.destroy_process_group()


def _run(n_shards):
    import oracle
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, n_shards, out), nprocs=world, join=True)
        res = dict(out)
    o0, l0, q, kc, vc = res[0]
    o1, l1 = res[1][0], res[1][1]
    np.testing.assert_array_equal(o0, o1)
    ro, rl, _, _ = oracle.phase2_attend(q.astype(np.float64), kc.astype(np.float64), vc.astype(np.float64), n_shards,
                                        100, 10000.0)
    np.testing.assert_allclose(o0, ro, rtol=0, atol=1e-5)
    np.testing.assert_allclose(l0, rl, rtol=0, atol=1e-5)


def test_exchange_even_shards():
    _run(4)


def test_exchange_uneven_shards_pads_empty():
    _run(3)      # rank 0 holds 2 shards, rank 1 holds 1 and pads one empty shard


def test_balanced_host_ranges_are_optimal():
    # every contiguous split of the hosts into `world` ranges, by brute force:
    # none has a smaller largest range work (sum of n (n + 1) / 2)
    import itertools
    from long_context_blockwise_max_b200.distributed import balanced_host_ranges, host_rows
    cost = lambda rows, rg: max(sum(x * (x + 1) // 2 for x in rows[a:b]) for a, b in rg)
    for rows in (host_rows(8, 16384, 64, 2048, False), host_rows(8, 16384, 0, 0, True),
                 host_rows(7, 256, 16, 32, False), [5, 100, 3, 3, 90, 1]):
        n = len(rows)
        for world in range(1, n + 1):
            got = balanced_host_ranges(rows, world)
            assert len(got) == world and got[0][0] == 0 and got[-1][1] == n
            assert all(a[1] == b[0] and a[0] < a[1] for a, b in zip(got, got[1:]))
            best = min(cost(rows, [(0, c[0])] + list(zip(c, c[1:])) + [(c[-1], n)] if c else [(0, n)])
                       for c in itertools.combinations(range(1, n), world - 1))
            assert cost(rows, got) == best, (rows, world)
    assert balanced_host_ranges([10, 20], 4) == [(0, 1), (1, 2), (2, 2), (2, 2)]


def test_shard_ranges():
    from long_context_blockwise_max_b200.distributed import shard_ranges
    assert shard_ranges(8, 4) == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert shard_ranges(3, 2) == [(0, 2), (2, 3)]
    assert shard_ranges(1, 3) == [(0, 1), (1, 1), (1, 1)]


# --------------------------------------------------------------------------
# Phase 1 spread over ranks, then the Phase-2 exchange over the ranks' blocks
# --------------------------------------------------------------------------
L1, BLK1, SINK1, CH1, K1, HQ1, HKV1, D1, TH1 = 256, 64, 16, 16, 1, 4, 2, 16, 10000.0


def _pipeline_inputs():
    g = torch.Generator().manual_seed(11)
    q = torch.randn(L1, HQ1, D1, generator=g, dtype=torch.float64)
    k = torch.randn(L1, HKV1, D1, generator=g, dtype=torch.float64)
    v = torch.randn(L1, HKV1, D1, generator=g, dtype=torch.float64)
    sel = torch.tensor([[2], [0], [3], [1]], dtype=torch.int64)
    qq = torch.randn(1, 3, HQ1, D1, generator=g, dtype=torch.float64)
    return q, k, v, sel, qq


def _oracle_encode_hosts(q, k, v, theta, block, sink, chunk, k_chunks, sel, star, h0, h1):
    import oracle
    pos = oracle.host_positions(q.shape[0], block, sink, chunk, sel.numpy(), star=star)
    outs = oracle.phase1_encode(q.numpy(), k.numpy(), v.numpy(), pos, theta)[h0:h1]
    kr, vr = oracle.retained_kv(k.numpy(), v.numpy(), theta)
    o = np.concatenate([x[0] for x in outs]) if outs else np.zeros((0, q.shape[1], q.shape[2]))
    lse = np.concatenate([x[1] for x in outs]) if outs else np.zeros((0, q.shape[1]))
    return (torch.from_numpy(o), torch.from_numpy(lse), torch.from_numpy(kr[h0 * block:h1 * block]),
            torch.from_numpy(vr[h0 * block:h1 * block]))


def _pipeline_worker(rank, world, port, star, out):
    sys.path.insert(0, ROOT)
    from long_context_blockwise_max_b200 import distributed as D
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, sel, qq = _pipeline_inputs()
        o, lse, kr, vr, (h0, h1) = D.phase1_encode_distributed(q, k, v, TH1, BLK1, SINK1, CH1, K1, sel, star,
                                                               encode_fn=_oracle_encode_hosts)
        ranges = D.phase1_host_ranges(L1, BLK1, SINK1, CH1, K1, star, world)
        og, lg = D.phase2_attend_distributed(qq, kr[None], vr[None], h1 - h0, L1 // BLK1, L1, TH1,
                                             partials_fn=_oracle_partials, merge_fn=_oracle_merge,
                                             max_local=max(b - a for a, b in ranges))
        out[rank] = (h0, h1, o.numpy(), lse.numpy(), og.numpy(), lg.numpy())
    finally:
        dist.destroy_process_group()


def _pipeline(world, star):
    import oracle
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_pipeline_worker, args=(world, port, star, out), nprocs=world, join=True)
        res = [out[r] for r in range(world)]
    q, k, v, sel, qq = _pipeline_inputs()
    n = L1 // BLK1
    # the ranks' host ranges tile [0, n) in order
    from long_context_blockwise_max_b200 import distributed as D
    ranges = D.phase1_host_ranges(L1, BLK1, SINK1, CH1, K1, star, world)
    assert [(r[0], r[1]) for r in res] == ranges
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    # Phase 1: the ranks' rows, in rank order, are the one-process encoding
    pos = oracle.host_positions(L1, BLK1, SINK1, CH1, sel.numpy(), star=star)
    full = oracle.phase1_encode(q.numpy(), k.numpy(), v.numpy(), pos, TH1)
    np.testing.assert_array_equal(np.concatenate([r[2] for r in res]), np.concatenate([x[0] for x in full]))
    np.testing.assert_array_equal(np.concatenate([r[3] for r in res]), np.concatenate([x[1] for x in full]))
    # Phase 2 over the ranks' retained blocks equals one-process attention
    kr, vr = oracle.retained_kv(k.numpy(), v.numpy(), TH1)
    ro, rl, _, _ = oracle.phase2_attend(qq.numpy(), kr[None], vr[None], n, L1, TH1)
    for r in res:
        np.testing.assert_allclose(r[4], ro, rtol=0, atol=1e-6)
        np.testing.assert_allclose(r[5], rl, rtol=0, atol=1e-6)


def test_phase1_hosts_over_two_ranks_then_exchange():
    _pipeline(2, False)


def test_star_hosts_over_three_ranks_one_empty():
    _pipeline(3, True)   # 4 hosts over 3 ranks: (0, 2), (2, 4), (4, 4)
