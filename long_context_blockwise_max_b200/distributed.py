"""The multi-GPU layout of the method: one host (block) per GPU.

The Pulsar Attention page (§2.1, §2.2) and the Star Attention review
(key_machinery) spread the hosts of one sequence over devices.

Phase 1 needs no communication: every host encodes its own input (sink,
summaries of the earlier blocks, its own block) from the whole sequence's
ids and Q / K / V, and keeps its own block's KV.  ``phase1_encode_distributed``
gives each rank a contiguous range of hosts, balanced by attention work, and
runs ``pulsar_phase1_encode_hosts`` (or the Star variant) on it.

Phase 2 has the method's one exchange step:

1. The query is broadcast.
2. Each host attends over the retained cache it holds.
3. The partial results (one vector and one scalar per query token and head)
   are all-gathered.
4. An exact online-softmax merge follows.

``phase2_attend_distributed`` computes a rank's shard partials with
``star_phase2_attend``, all-gathers the packed partials with
``torch.distributed`` (NCCL on GPUs), and merges all of them with
``pa_lse_merge`` on every rank.  The per-rank steps can be replaced by other
functions of the same contract, which the CPU tests use with the gloo
backend.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_ranges(n_shards: int, world: int) -> list[tuple[int, int]]:
    """Contiguous shard ranges of the ranks: ceil(n_shards / world) each, the
    last ranks possibly shorter or empty."""
    per = -(-n_shards // world)
    return [(min(r * per, n_shards), min((r + 1) * per, n_shards)) for r in range(world)]


def host_rows(n_hosts: int, block: int, sink: int, summary_tokens: int, star: bool) -> list[int]:
    """Phase-1 rows of every host: block for host 0; 2 * block (Star) or
    sink + i * summary_tokens + block (Pulsar) for host i >= 1."""
    return [block if i == 0 else (2 * block if star else sink + i * summary_tokens + block)
            for i in range(n_hosts)]


def balanced_host_ranges(rows: list[int], world: int) -> list[tuple[int, int]]:
    """Contiguous host ranges of the ranks that minimise the largest rank's
    causal attention work, sum over its hosts of n (n + 1) / 2.  Later hosts
    carry longer prefixes, so equal host counts would leave the last rank
    the most work.  Ranks past the hosts get empty ranges."""
    n = len(rows)
    work = [r * (r + 1) // 2 for r in rows]
    pre = [0]
    for w in work:
        pre.append(pre[-1] + w)
    k = max(1, min(world, n))
    INF = float("inf")
    # best[m][i]: the least achievable maximum over m ranks covering hosts [0, i)
    best = [[INF] * (n + 1) for _ in range(k + 1)]
    cut = [[0] * (n + 1) for _ in range(k + 1)]
    best[0][0] = 0
    for m in range(1, k + 1):
        for i in range(m, n + 1):
            for t in range(m - 1, i):
                c = max(best[m - 1][t], pre[i] - pre[t])
                if c < best[m][i]:
                    best[m][i], cut[m][i] = c, t
    bounds, i = [], n
    for m in range(k, 0, -1):
        bounds.append((cut[m][i], i))
        i = cut[m][i]
    bounds.reverse()
    return bounds + [(n, n)] * (world - k)


def _gpu_encode_hosts(q, k, v, rope_theta, block, sink, chunk, k_chunks, sel, star, h0, h1):
    from . import pulsar
    if star:
        o, lse, k_ret, v_ret, _, _ = pulsar.star_phase1_encode_hosts(q, k, v, rope_theta, block, h0, h1)
    else:
        o, lse, k_ret, v_ret, _, _ = pulsar.pulsar_phase1_encode_hosts(q, k, v, rope_theta, block, sink, chunk,
                                                                       k_chunks, sel, h0, h1)
    return o, lse, k_ret, v_ret


def phase1_host_ranges(L: int, block: int, sink: int, chunk: int, k_chunks: int, star: bool,
                       world: int) -> list[tuple[int, int]]:
    """The ranks' host ranges of one sequence (balanced_host_ranges)."""
    return balanced_host_ranges(host_rows(L // block, block, 0 if star else sink,
                                          0 if star else k_chunks * chunk, star), world)


def phase1_encode_distributed(q, k, v, rope_theta: float, block: int, sink: int = 64, chunk: int = 32,
                              k_chunks: int = 0, sel=None, star: bool = False, group=None, encode_fn=None):
    """Phase 1 of one sequence with its N = L / block hosts spread over the
    ranks: rank r encodes the contiguous host range phase1_host_ranges(...)[r],
    balanced by attention work (no collective).

    q [L][hq][d], k, v [L][hkv][d] and sel [N][k_chunks] are the whole
    sequence's, the same on every rank.  Returns (o, lse, k_ret, v_ret,
    (host_begin, host_end)): the range's Phase-1 rows and retained blocks,
    which are this rank's shards for ``phase2_attend_distributed``."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = phase1_host_ranges(q.shape[0], block, sink, chunk, k_chunks, star, world)[rank]
    fn = encode_fn or _gpu_encode_hosts
    o, lse, k_ret, v_ret = fn(q, k, v, rope_theta, block, sink, chunk, k_chunks, sel, star, h0, h1)
    return o, lse, k_ret, v_ret, (h0, h1)


def _gpu_partials(q, k_local, v_local, n_local, q_pos0, rope_theta):
    from . import pulsar
    _, _, part_o, part_lse, _ = pulsar.star_phase2_attend(q, k_local, v_local, n_local, q_pos0=q_pos0,
                                                          rope_theta=rope_theta, want_partials=True)
    return part_o, part_lse


def _gpu_merge(part_o, part_lse, dtype):
    from . import pulsar
    return pulsar.pa_lse_merge(part_o, part_lse, dtype=dtype)


def phase2_attend_distributed(q, k_local, v_local, n_local: int, n_shards_total: int, q_pos0: int,
                              rope_theta: float, group=None, partials_fn=None, merge_fn=None,
                              max_local: int | None = None):
    """Exact global query attention over shards spread across ranks.

    q: [B][Tq][hq][d], the same on every rank.
    k_local, v_local: [B][T_local][hkv][d], this rank's n_local shards in
    order (K rotated). The ranks' shards, concatenated in rank order, are
    the n_shards_total shards of the whole cache.  max_local: the most
    shards any rank holds, the same on every rank (default
    ceil(n_shards_total / world)); ranks with fewer pad with empty shards.
    Returns (O [B][Tq][hq][d], lse [B][Tq][hq]) on every rank.
    """
    partials_fn = partials_fn or _gpu_partials
    merge_fn = merge_fn or _gpu_merge
    world = dist.get_world_size(group)
    per = max_local if max_local is not None else -(-n_shards_total // world)
    if n_local > per:
        raise ValueError(f"{n_local} local shards exceed max_local = {per}")
    B, Tq, hq, d = q.shape
    if n_local > 0:
        part_o, part_lse = partials_fn(q, k_local, v_local, n_local, q_pos0, rope_theta)
    else:
        part_o = q.new_zeros((B, 0, Tq, hq, d), dtype=torch.float32)
        part_lse = q.new_zeros((B, 0, Tq, hq), dtype=torch.float32)
    # pack [per][B][Tq][hq][d + 1]; ranks with fewer shards pad with empty ones (lse -inf)
    packed = torch.zeros((per, B, Tq, hq, d + 1), dtype=torch.float32, device=q.device)
    packed[..., d] = float("-inf")
    if n_local:
        packed[:n_local, ..., :d] = part_o.permute(1, 0, 2, 3, 4)
        packed[:n_local, ..., d] = part_lse.permute(1, 0, 2, 3)
    gathered = torch.empty((world * per,) + tuple(packed.shape[1:]), dtype=torch.float32, device=q.device)
    dist.all_gather_into_tensor(gathered, packed, group=group)
    all_o = gathered[..., :d].permute(1, 0, 2, 3, 4).contiguous()      # [B][world*per][Tq][hq][d]
    all_lse = gathered[..., d].permute(1, 0, 2, 3).contiguous()        # [B][world*per][Tq][hq]
    return merge_fn(all_o, all_lse, q.dtype)
