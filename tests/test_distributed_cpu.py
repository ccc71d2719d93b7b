"""The Phase-2 exchange across ranks (Pulsar page §2.2: partials are
all-gathered, then merged exactly), on CPU with the gloo backend and world
size 2: per-rank partials and the merge come from the oracle, so this
checks the shard partition, packing, gather order and padding of
long_context_blockwise_max_b200.distributed against dense attention."""
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
    with mp.Manager() as m:
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


def test_shard_ranges():
    from long_context_blockwise_max_b200.distributed import shard_ranges
    assert shard_ranges(8, 4) == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert shard_ranges(3, 2) == [(0, 2), (2, 3)]
    assert shard_ranges(1, 3) == [(0, 1), (1, 1), (1, 1)]
