"""Plain fp64 restatement of the Star / Pulsar attention path (test oracle).

TEST INFRASTRUCTURE ONLY -- never imported by the product path.

Sources (web pages, cited by title and section):

* [P]  "Dropping the Anchor: Statistical Context Summarization for Distributed
       Systems via Pulsar Attention", project page: §1 (the anchor problem),
       §2 (method), §2.1 (selecting summaries with Max-IDF), Figure 2 (toy
       example), §2.2 (query phase), §4 (efficiency), §5 (code / CLI flags).
* [PS] "Technische Samenvatting: Pulsar Attention" (Dutch technical summary),
       sections "Fase 1" and "Fase 2".
* [S]  Star Attention review (machine review of arXiv 2411.17116): summary,
       key_machinery, and the referee's minor comments on the online-softmax
       update of Algorithm 2 and on c'_1 = c_1.

Everything is computed in float64 from the inputs exactly as stored (bf16 and
fp32 inputs are widened to fp64 by the caller).  Library primitives used as
single steps: ``np.unique`` (set of ids in a block), ``np.matmul`` (dot
products), ``np.exp`` / ``np.log``.  No blocking, fusion or reordering beyond
the definitions below; computing a subset of attention rows evaluates each
requested row by its own definition.

Readings of points the pages leave open (each also listed in the design notes):

* IDF(t) = ln(N / df(t)) with N blocks as documents, no smoothing ([P] §2.1;
  Figure 2 gives IDF 0 for a token present in every block).
* Ties in chunk score: lower chunk index first.
* Budget: k = floor(0.125 * block / chunk) chunks per block ([P] §2.1).
* Host 0 has no prefix (c'_1 = c_1, [S] minor comment); hosts i >= 1 see
  [sink || Sigma_0 || ... || Sigma_{i-1} || B_i] ([PS] Fase 1; [P] §2).
* Summary chunks of block 0 that overlap the sink are not removed.
* The causal mask is over the concatenated host row index, not position id.
* Every host row produces an output (a layer's output for all of its rows).
* RoPE: rotate-half convention, omega_m = theta^(-2m/d), no frequency scaling.
* Phase-2 query attends to every retained key (no mask); shard h covers keys
  [h*ceil(T/S), min((h+1)*ceil(T/S), T)); an empty shard has lse = -inf and
  weight 0; if every shard is empty, O = 0 and lse = -inf.

Parity pins (tests/test_oracle_*.py): brute-force top-k and a Figure-2
analogue (selection); N = 1 reduces to library causal attention, full-budget
/ zero-sink hosts equal dense causal attention rows, the uniform-score closed
form lse = ln(r+1), and complex-multiplication RoPE (Phase 1); the shard merge
equals library dense attention over the concatenated cache (Phase 2).  Added
rows: mean-IDF against hand-worked Figure-2 means, a hand-worked tie at
N = 16 and brute force over a high-precision evaluation of the real mean
IDF; evenly spaced chunks against their closed form; entropy against its
closed forms (all distinct, all equal), a hand-worked tie between tf
multisets {4, 1, 1, 1, 1} and {2, 2, 2, 2}, and brute force over a
high-precision evaluation; BM25 against hand-worked values (the formulas of
entropy and BM25 are not on the pages: parity unpinned beyond these); the query-host step against masked
library attention; ART with zero thresholds against library attention and
its stop block against a closed form where the weights underflow.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# Max-IDF summary selection  ([P] §2.1; [PS] Fase 1, "Heuristiek" / "Selectie")
# ----------------------------------------------------------------------------


def _blocks(ids: np.ndarray, block: int) -> list[np.ndarray]:
    """Contiguous blocks of ``block`` tokens ([P] §1: the context is split into
    contiguous blocks, one per host)."""
    ids = np.asarray(ids)
    if ids.size % block:
        raise ValueError("sequence length must be a multiple of the block size")
    return [ids[j * block:(j + 1) * block] for j in range(ids.size // block)]


def document_frequency(ids: np.ndarray, block: int, vocab: int) -> np.ndarray:
    """df(t) = number of blocks that contain token t, blocks being the documents
    ([P] §2.1).  Returns int64 [vocab]."""
    df = np.zeros(vocab, dtype=np.int64)
    for blk in _blocks(ids, block):
        present = np.unique(blk)            # the set of ids in this document
        df[present] += 1
    return df


def idf_table(df: np.ndarray, n_blocks: int) -> np.ndarray:
    """IDF(t) = ln(N / df(t)) for every token present in the sequence; NaN for
    tokens that never occur (they are never looked up)."""
    out = np.full(df.shape, np.nan, dtype=np.float64)
    m = df > 0
    out[m] = np.log(float(n_blocks) / df[m].astype(np.float64))
    return out


def chunk_scores(ids: np.ndarray, block: int, chunk: int, idf: np.ndarray) -> np.ndarray:
    """Score of every non-overlapping ``chunk``-token chunk of every block: the
    maximum IDF over its tokens, i.e. the IDF of its rarest token ([P] §2.1).
    Returns float64 [N][block // chunk]."""
    if block % chunk:
        raise ValueError("block must be a multiple of the chunk size")
    blocks = _blocks(ids, block)
    C = block // chunk
    out = np.empty((len(blocks), C), dtype=np.float64)
    for j, blk in enumerate(blocks):
        for c in range(C):
            out[j, c] = max(idf[t] for t in blk[c * chunk:(c + 1) * chunk].tolist())
    return out


def chunk_min_df(ids: np.ndarray, block: int, chunk: int, df: np.ndarray) -> np.ndarray:
    """Smallest df over the tokens of each chunk, int64 [N * (block // chunk)]
    in sequence order (the integer twin of ``chunk_scores``: ln(N/df) is
    strictly decreasing in df, so the chunk's max IDF is the IDF of its min df)."""
    blocks = _blocks(ids, block)
    C = block // chunk
    out = np.empty(len(blocks) * C, dtype=np.int64)
    for j, blk in enumerate(blocks):
        for c in range(C):
            out[j * C + c] = min(int(df[t]) for t in blk[c * chunk:(c + 1) * chunk].tolist())
    return out


def select_summaries(ids: np.ndarray, block: int, chunk: int, k: int, vocab: int,
                     return_scores: bool = False):
    """Top-k chunks per block by Max-IDF score, kept in original order
    ([P] §2.1: the summary is the k best chunks in their original order).
    Equal scores: the lower chunk index wins.

    Returns int64 [N][k] local chunk indices, ascending within each block
    (and the [N][C] score table when ``return_scores``)."""
    n_blocks = len(ids) // block
    C = block // chunk
    if not 0 <= k <= C:
        raise ValueError("k must be in [0, block/chunk]")
    df = document_frequency(ids, block, vocab)
    idf = idf_table(df, n_blocks)
    scores = chunk_scores(ids, block, chunk, idf)
    sel = np.empty((n_blocks, k), dtype=np.int64)
    for j in range(n_blocks):
        order = sorted(range(C), key=lambda c: (-scores[j, c], c))
        sel[j] = sorted(order[:k])
    return (sel, scores) if return_scores else sel


# ----------------------------------------------------------------------------
# Alternative summary scorers ([P] §3.1 and Table 1: the other statistical
# scores and the non-statistical baselines; [P] §2.1 contrasts max with mean)
# ----------------------------------------------------------------------------

def chunk_mean_idf(ids: np.ndarray, block: int, chunk: int, idf: np.ndarray) -> np.ndarray:
    """Mean IDF over each chunk's tokens (exactly rounded sum / chunk),
    float64 [N][C].  Reported score only: the ranking below is exact."""
    blocks = _blocks(ids, block)
    C = block // chunk
    out = np.empty((len(blocks), C), dtype=np.float64)
    for j, blk in enumerate(blocks):
        for c in range(C):
            out[j, c] = math.fsum(idf[t] for t in blk[c * chunk:(c + 1) * chunk].tolist()) / chunk
    return out


def chunk_df_product(ids: np.ndarray, block: int, chunk: int, df: np.ndarray) -> list:
    """Product of df(t) over each chunk's tokens, as exact Python integers
    [N * C] in sequence order.

    With every chunk holding the same number c of tokens,
        mean IDF = (1/c) sum_t ln(N / df(t)) = ln N - (1/c) ln prod_t df(t),
    so a higher mean IDF is exactly a smaller product, and equal means are
    exactly equal products: the real-valued order of the definition, with
    its ties, and no rounding anywhere."""
    blocks = _blocks(ids, block)
    C = block // chunk
    out = []
    for blk in blocks:
        for c in range(C):
            prod = 1
            for t in blk[c * chunk:(c + 1) * chunk].tolist():
                prod *= int(df[t])
            out.append(prod)
    return out


def select_evenly_spaced(n_blocks: int, block: int, chunk: int, k: int) -> np.ndarray:
    """Evenly spaced chunks, the same in every block: chunk floor(m * C / k)
    for m = 0..k-1 (the non-statistical baseline of [P] §3.1)."""
    C = block // chunk
    row = [(m * C) // k for m in range(k)]
    return np.tile(np.array(row, dtype=np.int64), (n_blocks, 1)).reshape(n_blocks, k)


def select_summaries_mean_idf(ids: np.ndarray, block: int, chunk: int, k: int, vocab: int,
                              return_rank: bool = False):
    """Top-k chunks per block by mean IDF ([P] §3.1, Table 1; §2.1 contrasts
    the maximum with the mean), kept in original order; equal means go to the
    lower chunk index.  The order is the exact real-valued one: ascending
    product of df over the chunk (chunk_df_product).

    Returns int64 [N][k] local chunk indices, ascending (and, when
    ``return_rank``, int64 [N * C]: each chunk's 0-based position in its
    block's order, best first)."""
    n_blocks = len(ids) // block
    C = block // chunk
    if not 0 <= k <= C:
        raise ValueError("k must be in [0, block/chunk]")
    df = document_frequency(ids, block, vocab)
    prod = chunk_df_product(ids, block, chunk, df)
    sel = np.empty((n_blocks, k), dtype=np.int64)
    rank = np.empty(n_blocks * C, dtype=np.int64)
    for j in range(n_blocks):
        order = sorted(range(C), key=lambda c: (prod[j * C + c], c))
        for r, c in enumerate(order):
            rank[j * C + c] = r
        sel[j] = sorted(order[:k])
    return (sel, rank) if return_rank else sel


def chunk_entropy(ids: np.ndarray, block: int, chunk: int) -> np.ndarray:
    """Shannon entropy (natural log) of each chunk's token distribution,
    H(c) = -sum_t p_t ln p_t with p_t = tf(t, c) / |c|, float64 [N][C].
    Reading: the pages list entropy among the statistical scorers of §3.1 /
    Table 1 without a formula; this is the textbook Shannon entropy of the
    chunk's empirical token frequencies, and chunks of higher entropy are
    kept.  Parity unpinned beyond the closed forms and hand-worked values in
    the tests."""
    blocks = _blocks(ids, block)
    C = block // chunk
    out = np.empty((len(blocks), C), dtype=np.float64)
    for j, blk in enumerate(blocks):
        for c in range(C):
            toks = blk[c * chunk:(c + 1) * chunk].tolist()
            tf = {}
            for t in toks:
                tf[t] = tf.get(t, 0) + 1
            out[j, c] = -math.fsum((n / chunk) * math.log(n / chunk) for n in tf.values())
    return out


def chunk_tf_power_product(ids: np.ndarray, block: int, chunk: int) -> list:
    """prod_t tf(t, c)^tf(t, c) over the distinct tokens of each chunk, as
    exact Python integers [N * C].  With a fixed chunk length,
    H(c) = ln |c| - (1/|c|) ln prod_t tf^tf, so a higher entropy is exactly a
    smaller product and equal entropies are exactly equal products."""
    blocks = _blocks(ids, block)
    C = block // chunk
    out = []
    for blk in blocks:
        for c in range(C):
            tf = {}
            for t in blk[c * chunk:(c + 1) * chunk].tolist():
                tf[t] = tf.get(t, 0) + 1
            prod = 1
            for n in tf.values():
                prod *= n ** n
            out.append(prod)
    return out


def select_summaries_entropy(ids: np.ndarray, block: int, chunk: int, k: int, return_rank: bool = False):
    """Top-k chunks per block by entropy (chunk_entropy), exact order
    (ascending chunk_tf_power_product), equal entropies to the lower index,
    kept in original order.  Returns int64 [N][k] (and the int64 [N * C]
    ranks, best first, when ``return_rank``)."""
    n_blocks = len(ids) // block
    C = block // chunk
    if not 0 <= k <= C:
        raise ValueError("k must be in [0, block/chunk]")
    prod = chunk_tf_power_product(ids, block, chunk)
    sel = np.empty((n_blocks, k), dtype=np.int64)
    rank = np.empty(n_blocks * C, dtype=np.int64)
    for j in range(n_blocks):
        order = sorted(range(C), key=lambda c: (prod[j * C + c], c))
        for r, c in enumerate(order):
            rank[j * C + c] = r
        sel[j] = sorted(order[:k])
    return (sel, rank) if return_rank else sel


BM25_K1 = 1.2
BM25_B = 0.75


def chunk_bm25(ids: np.ndarray, block: int, chunk: int, vocab: int) -> np.ndarray:
    """BM25 weight of each chunk over its own tokens, float64 [N * C] in
    sequence order: sum over the distinct tokens t of the chunk, in order of
    their first occurrence, of
        idf(t) * tf (k1 + 1) / (tf + k1 (1 - b + b |c| / avgdl)),
        idf(t) = ln(1 + (N - df(t) + 0.5) / (df(t) + 0.5)),
    with blocks as the documents for df (as for Max-IDF), k1 = 1.2, b = 0.75,
    and |c| = avgdl = chunk (every chunk has the chunk length).
    Reading: the pages list BM25 among the statistical scorers of §3.1 /
    Table 1 without a formula; this is the standard Okapi BM25 term weight
    (Robertson-Sparck Jones idf with +1 inside the log) summed over the
    chunk's own terms.  Parity unpinned beyond the hand-worked values in the
    tests."""
    n = len(ids) // block
    df = document_frequency(ids, block, vocab)
    blocks = _blocks(ids, block)
    C = block // chunk
    norm = BM25_K1 * (1.0 - BM25_B + BM25_B * chunk / chunk)
    out = np.empty(n * C, dtype=np.float64)
    for j, blk in enumerate(blocks):
        for c in range(C):
            tf, order = {}, []
            for t in blk[c * chunk:(c + 1) * chunk].tolist():
                if t not in tf:
                    order.append(t)
                tf[t] = tf.get(t, 0) + 1
            total = 0.0
            for t in order:
                d = float(df[t])
                idf = math.log(1.0 + (n - d + 0.5) / (d + 0.5))
                total += idf * (tf[t] * (BM25_K1 + 1.0)) / (tf[t] + norm)
            out[j * C + c] = total
    return out


def select_summaries_bm25(ids: np.ndarray, block: int, chunk: int, k: int, vocab: int):
    """Top-k chunks per block by chunk_bm25 (descending, ties to the lower
    index), kept in original order.  Returns int64 [N][k]."""
    n_blocks = len(ids) // block
    C = block // chunk
    if not 0 <= k <= C:
        raise ValueError("k must be in [0, block/chunk]")
    sc = chunk_bm25(ids, block, chunk, vocab).reshape(n_blocks, C)
    sel = np.empty((n_blocks, k), dtype=np.int64)
    for j in range(n_blocks):
        order = sorted(range(C), key=lambda c: (-sc[j, c], c))
        sel[j] = sorted(order[:k])
    return sel


# ----------------------------------------------------------------------------
# Phase 1: host inputs  ([PS] Fase 1; [P] §2, Figure 1; [S] key_machinery)
# ----------------------------------------------------------------------------


def host_positions(L: int, block: int, sink: int, chunk: int, sel, star: bool = False):
    """Original position ids of every row of every host's Phase-1 input.

    Pulsar ([PS] Fase 1): host i >= 1 encodes [S_sink || Sigma_0 || ... ||
    Sigma_{i-1} || B_i]; S_sink is the first ``sink`` tokens of the sequence,
    Sigma_j the selected chunks of block j in original order.
    Star ([S] key_machinery): host i >= 1 encodes [B_0 || B_i].
    Host 0 encodes B_0 alone in both (c'_1 = c_1, [S] minor comment)."""
    n = L // block
    hosts = [np.arange(0, block, dtype=np.int64)]
    for i in range(1, n):
        parts = []
        if star:
            parts.append(np.arange(0, block, dtype=np.int64))
        else:
            parts.append(np.arange(0, sink, dtype=np.int64))
            for j in range(i):
                for c in sel[j]:
                    start = j * block + int(c) * chunk
                    parts.append(np.arange(start, start + chunk, dtype=np.int64))
        parts.append(np.arange(i * block, (i + 1) * block, dtype=np.int64))
        hosts.append(np.concatenate(parts))
    return hosts


def host_row_offsets(positions) -> np.ndarray:
    """Row offsets of the hosts in the packed output: [N + 1] int64."""
    off = np.zeros(len(positions) + 1, dtype=np.int64)
    off[1:] = np.cumsum([len(p) for p in positions])
    return off


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding, rotate-half convention, at position ids ``pos``
    ([P] §2.1: every host encodes its tokens at their original position ids).

    x: [n][H][d] float64.  For m < d/2, with omega_m = theta^(-2m/d) and
    a = p * omega_m:  x'[m] = x[m] cos a - x[m + d/2] sin a,
                      x'[m + d/2] = x[m + d/2] cos a + x[m] sin a."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    m = np.arange(half, dtype=np.float64)
    omega = theta ** (-2.0 * m / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * omega[None, :]  # [n][d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows=None):
    """Causal softmax attention over one host's concatenated rows.

    q: [n][Hq][d], k/v: [n][Hkv][d] (already rotated), fp64.  Query head h
    reads kv head h // (Hq / Hkv).  Row r attends to rows c <= r:
    s_rc = q_r . k_c / sqrt(d);  o_r = sum_c softmax(s_r)_c v_c;
    lse_r = ln sum_{c <= r} exp(s_rc).
    Returns (o [len(rows)][Hq][d], lse [len(rows)][Hq])."""
    n, hq, d = q.shape
    hkv = k.shape[1]
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = hq // hkv
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.zeros((rows.size, hq, d), dtype=np.float64)
    lse = np.zeros((rows.size, hq), dtype=np.float64)
    if rows.size == 0:
        return o, lse
    ncols = int(rows.max()) + 1
    scale = 1.0 / math.sqrt(d)
    mask = np.arange(ncols)[None, :] > rows[:, None]          # True where c > r
    for h in range(hq):
        kh = k[:ncols, h // g, :]
        vh = v[:ncols, h // g, :]
        s = (q[rows, h, :] @ kh.T) * scale
        s[mask] = -np.inf
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        z = e.sum(axis=1, keepdims=True)
        o[:, h, :] = (e @ vh) / z
        lse[:, h] = (mx + np.log(z))[:, 0]
    return o, lse


def phase1_encode(q, k, v, positions, theta: float, rows_per_host=None):
    """Phase-1 encoding of every host: RoPE at the original positions, then
    causal attention over the host's rows ([S] summary; [PS] Fase 1).

    q: [L][Hq][d], k/v: [L][Hkv][d] fp64 (unrotated).  ``positions`` from
    ``host_positions``.  ``rows_per_host``: optional list of row subsets.
    Returns a list of (o, lse) per host."""
    out = []
    for i, pos in enumerate(positions):
        rows = None if rows_per_host is None else rows_per_host[i]
        upto = len(pos) if rows is None or len(rows) == 0 else int(np.max(rows)) + 1
        p = pos[:upto]
        qh = rope(q[p], p, theta)
        kh = rope(k[p], p, theta)
        vh = np.asarray(v[p], dtype=np.float64)
        out.append(causal_attention(qh, kh, vh, rows))
    return out


def retained_kv(k, v, theta: float):
    """KV kept after Phase 1: only each host's own block B_i survives, so the
    retained cache over all hosts is the whole sequence's K (rotated at its
    original positions) and V ([P] §2.1: the KV of the sink and of the
    summaries is dropped; §2.2: a host keeps the KV cache of its own block
    alone).  Layout [L][Hkv][d] ==
    [N][block][Hkv][d]."""
    L = k.shape[0]
    return rope(k, np.arange(L), theta), np.asarray(v, dtype=np.float64)


def phase1_flops(positions, hq: int, d: int) -> float:
    """Algorithmic Phase-1 FLOPs: QK^T and PV over the causal pairs (diagonal
    included), 4 * d * Hq * n(n+1)/2 per host."""
    return float(sum(4.0 * d * hq * len(p) * (len(p) + 1) / 2.0 for p in positions))


# ----------------------------------------------------------------------------
# Phase 2: split-KV query attention and exact merge
# ([P] §2.2; [PS] Fase 2; [S] key_machinery and Algorithm 2 minor comment)
# ----------------------------------------------------------------------------


def shard_bounds(T: int, n_shards: int):
    """[start, end) of each shard: equal contiguous shards of ceil(T/S) keys,
    the last ones shorter or empty."""
    step = -(-T // n_shards) if n_shards else 0
    return [(min(h * step, T), min((h + 1) * step, T)) for h in range(n_shards)]


def phase2_partials(q, k_cache, v_cache, n_shards: int):
    """Local attention of the (already rotated) query over each shard.

    q: [B][Tq][Hq][d]; k_cache, v_cache: [B][T][Hkv][d] (K rotated), fp64.
    For shard h: A_h = softmax(q K_h^T / sqrt(d)) V_h and s_h = ln sum exp
    (every key of the shard visible).  Returns A [B][S][Tq][Hq][d] and
    s [B][S][Tq][Hq]; an empty shard gives A_h = 0, s_h = -inf."""
    B, Tq, hq, d = q.shape
    T, hkv = k_cache.shape[1], k_cache.shape[2]
    g = hq // hkv
    scale = 1.0 / math.sqrt(d)
    A = np.zeros((B, n_shards, Tq, hq, d), dtype=np.float64)
    s = np.full((B, n_shards, Tq, hq), -np.inf, dtype=np.float64)
    for b in range(B):
        for h, (lo, hi) in enumerate(shard_bounds(T, n_shards)):
            if hi <= lo:
                continue
            for head in range(hq):
                kk = k_cache[b, lo:hi, head // g, :]
                vv = v_cache[b, lo:hi, head // g, :]
                sc = (q[b, :, head, :] @ kk.T) * scale               # [Tq][n]
                mx = sc.max(axis=1, keepdims=True)
                e = np.exp(sc - mx)
                z = e.sum(axis=1, keepdims=True)
                A[b, h, :, head, :] = (e @ vv) / z
                s[b, h, :, head] = (mx + np.log(z))[:, 0]
    return A, s


def lse_merge(A, s):
    """Exact merge of shard partials ([S] Algorithm 2 as corrected in the
    referee's minor comment): s_global = ln sum_h exp(s_h);
    A = sum_h exp(s_h - s_global) * A_h.  Shard axis is axis 1.
    All shards empty: A = 0, s_global = -inf."""
    B, S = s.shape[0], s.shape[1]
    m = np.max(s, axis=1)                                 # [B][Tq][Hq]
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(s - m_safe[:, None])                       # exp(-inf) = 0
    z = w.sum(axis=1)
    s_global = np.where(finite, m_safe + np.log(np.where(finite, z, 1.0)), -np.inf)
    coef = np.where(finite[:, None], np.exp(s - np.where(finite, s_global, 0.0)[:, None]), 0.0)
    out = (coef[..., None] * A).sum(axis=1)
    return out, s_global


def phase2_attend(q, k_cache, v_cache, n_shards: int, q_pos0: int, theta: float):
    """Phase-2 global query attention: rotate the query at positions
    q_pos0 + j (if theta > 0), attend to every shard, merge exactly.
    q: [B][Tq][Hq][d] pre-RoPE; caches [B][T][Hkv][d] with K rotated.
    Returns (O [B][Tq][Hq][d], lse [B][Tq][Hq], A, s)."""
    q = np.asarray(q, dtype=np.float64)
    if theta > 0:
        B, Tq = q.shape[:2]
        pos = q_pos0 + np.arange(Tq)
        q = np.stack([rope(q[b], pos, theta) for b in range(B)])
    A, s = phase2_partials(q, np.asarray(k_cache, np.float64), np.asarray(v_cache, np.float64),
                           n_shards)
    o, lse = lse_merge(A, s)
    return o, lse, A, s


def phase2_attend_with_self(q, k_cache, v_cache, n_shards: int, k_self, v_self, self_off: int,
                            q_pos0: int, theta: float):
    """Query-host step: the query and generated tokens attend globally ([S]
    summary: global attention is reserved for the query and the generated
    tokens; [P] §5
    --tokens_to_generate).  Row j of q (rotated at q_pos0 + j) attends to
    every retained key of the shards and, causally, to the query host's own
    keys 0 .. self_off + j; the own keys form one more partial, merged with
    the shards' by the same exact LSE merge.

    q: [B][Tq][Hq][d] pre-RoPE; caches [B][T][Hkv][d]; k_self/v_self
    [B][S][Hkv][d] with K already rotated, S >= self_off + Tq.
    Returns (O [B][Tq][Hq][d], lse [B][Tq][Hq])."""
    q = np.asarray(q, dtype=np.float64)
    B, Tq, hq, d = q.shape
    if theta > 0:
        pos = q_pos0 + np.arange(Tq)
        q = np.stack([rope(q[b], pos, theta) for b in range(B)])
    A, s = phase2_partials(q, np.asarray(k_cache, np.float64), np.asarray(v_cache, np.float64), n_shards)
    hkv = k_self.shape[2]
    g = hq // hkv
    scale = 1.0 / math.sqrt(d)
    A_self = np.zeros((B, 1, Tq, hq, d), dtype=np.float64)
    s_self = np.full((B, 1, Tq, hq), -np.inf, dtype=np.float64)
    ks = np.asarray(k_self, np.float64)
    vs = np.asarray(v_self, np.float64)
    for b in range(B):
        for j in range(Tq):
            n = self_off + j + 1                       # own keys 0 .. self_off + j
            for head in range(hq):
                sc = (ks[b, :n, head // g, :] @ q[b, j, head, :]) * scale
                mx = sc.max()
                e = np.exp(sc - mx)
                A_self[b, 0, j, head] = (e @ vs[b, :n, head // g, :]) / e.sum()
                s_self[b, 0, j, head] = mx + np.log(e.sum())
    return lse_merge(np.concatenate([A, A_self], axis=1), np.concatenate([s, s_self], axis=1))


def phase2_attend_art(q, k_cache, v_cache, q_pos0: int, theta: float, block_keys: int = 128,
                      tau: float = 1e-5, phi: float = 1e-3, patience: int = 5):
    """Run-time early termination of the key traversal (ART review page:
    "Attention Run-time Termination" -- stop walking the KV cache once a
    probe of the running attention output has been stable in magnitude and
    direction for `patience` consecutive blocks; defaults tau = 1e-5,
    phi = 1e-3, p = 5; reverse-temporal traversal).

    Readings: blocks of `block_keys` keys from the newest backwards
    (block 1 = keys [T - block_keys, T)); the probe x_t is the full
    normalised running output after block t; step t >= 2 is stable when
    | |x_t| - |x_{t-1}| | <= tau |x_{t-1}| and 1 - cos(x_t, x_{t-1}) <= phi;
    a (batch, kv head) group stops after block t when its last `patience`
    steps were stable for every query row of the group (Tq tokens x the
    group's query heads); otherwise every block is visited.

    q: [B][Tq][Hq][d] pre-RoPE (rotated at q_pos0 + j when theta > 0);
    caches [B][T][Hkv][d] with K rotated.  Returns (O, lse over the visited
    keys, visited block counts [B][Hkv])."""
    q = np.asarray(q, dtype=np.float64)
    B, Tq, hq, d = q.shape
    if theta > 0:
        pos = q_pos0 + np.arange(Tq)
        q = np.stack([rope(q[b], pos, theta) for b in range(B)])
    kc = np.asarray(k_cache, np.float64)
    vc = np.asarray(v_cache, np.float64)
    T, hkv = kc.shape[1], kc.shape[2]
    g = hq // hkv
    scale = 1.0 / math.sqrt(d)
    n_blocks = -(-T // block_keys) if T else 0
    O = np.zeros((B, Tq, hq, d))
    lse = np.full((B, Tq, hq), -np.inf)
    visited = np.zeros((B, hkv), dtype=np.int64)
    for b in range(B):
        for kvh in range(hkv):
            heads = list(range(kvh * g, (kvh + 1) * g))
            m = np.full((Tq, g), -np.inf)
            l = np.zeros((Tq, g))
            acc = np.zeros((Tq, g, d))
            prev = None
            run = 0
            t = 0
            while t < n_blocks:
                t += 1
                lo, hi = max(T - t * block_keys, 0), T - (t - 1) * block_keys
                for jj in range(Tq):
                    for hh, head in enumerate(heads):
                        sc = (kc[b, lo:hi, kvh, :] @ q[b, jj, head, :]) * scale
                        mn = max(m[jj, hh], sc.max())
                        c_old = math.exp(m[jj, hh] - mn) if m[jj, hh] > -np.inf else 0.0
                        e = np.exp(sc - mn)
                        l[jj, hh] = l[jj, hh] * c_old + e.sum()
                        acc[jj, hh] = acc[jj, hh] * c_old + e @ vc[b, lo:hi, kvh, :]
                        m[jj, hh] = mn
                x = acc / l[..., None]
                if prev is not None:
                    nx = np.linalg.norm(x, axis=-1)
                    npv = np.linalg.norm(prev, axis=-1)
                    cos = (x * prev).sum(-1) / (nx * npv)
                    stable = (np.abs(nx - npv) <= tau * npv) & (1.0 - cos <= phi)
                    run = run + 1 if stable.all() else 0
                prev = x
                if run >= patience:
                    break
            visited[b, kvh] = t
            for hh, head in enumerate(heads):
                O[b, :, head, :] = acc[:, hh, :] / l[:, hh, None] if t else 0.0
                lse[b, :, head] = (m[:, hh] + np.log(l[:, hh])) if t else -np.inf
    return O, lse, visited
