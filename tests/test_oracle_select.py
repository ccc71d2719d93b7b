"""Pins for the oracle's Max-IDF selection (Pulsar Attention page, §2.1).

Each test checks the oracle against something other than itself: the
hand-worked Figure-2 analogue, document frequencies known by construction,
brute force over every k-subset, and the planted-singleton property.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from long_context_blockwise_max_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(tok):
    return {"0": 0.0, "log2": math.log(2.0), "log4": math.log(4.0)}[tok]


def test_figure2_toy_scores_and_selection():
    g = json.load(open(os.path.join(GOLDEN, "figure2_toy.json")))
    ids = np.array(g["ids"], dtype=np.int64)
    df = oracle.document_frequency(ids, g["block"], g["vocab"])
    for t, want in g["expected_df"].items():
        assert df[int(t)] == want
    idf = oracle.idf_table(df, len(ids) // g["block"])
    sc = oracle.chunk_scores(ids, g["block"], g["chunk"], idf)
    want = np.array([[_val(t) for t in row] for row in g["expected_scores"]])
    np.testing.assert_allclose(sc, want, rtol=0, atol=1e-15)
    sel = oracle.select_summaries(ids, g["block"], g["chunk"], g["k"], g["vocab"])
    assert sel.tolist() == g["expected_selection"]
    mdf = oracle.chunk_min_df(ids, g["block"], g["chunk"], df)
    assert mdf.tolist() == g["expected_min_df"]


def test_figure2_max_beats_mean():
    # The page's argument for max over mean: averaging divides a single rare
    # token's signal by the chunk length.  In block 2 of the analogue the mean
    # picks the distractor chunk, the max picks the answer chunk.
    g = json.load(open(os.path.join(GOLDEN, "figure2_toy.json")))
    ids = np.array(g["ids"], dtype=np.int64)
    df = oracle.document_frequency(ids, g["block"], g["vocab"])
    idf = oracle.idf_table(df, 4)
    blk2 = ids[32:48].reshape(4, 4)
    means = [float(np.mean(idf[c])) for c in blk2]
    assert int(np.argmax(means)) == g["mean_idf_would_select_in_block2"]
    assert oracle.select_summaries(ids, 16, 4, 1, 32)[2, 0] == 3


def test_df_known_by_construction():
    # Block j (of 5) holds tokens 100+t for t < j+1 repeated, plus its own
    # private token 200+j: token 100+t occurs in blocks t..4, df = 5 - t.
    blocks = []
    for j in range(5):
        toks = [100 + t for t in range(j + 1)] * 2 + [200 + j]
        toks += [150] * (16 - len(toks))     # 150 is in every block
        blocks.append(toks[:16])
    ids = np.array(sum(blocks, []), dtype=np.int64)
    df = oracle.document_frequency(ids, 16, 256)
    for t in range(5):
        assert df[100 + t] == 5 - t
    for j in range(5):
        assert df[200 + j] == 1
    assert df[150] == 5
    assert df[0] == 0
    idf = oracle.idf_table(df, 5)
    assert idf[150] == 0.0
    assert idf[204] == pytest.approx(math.log(5.0), abs=0)
    assert np.isnan(idf[0])


def _brute_force_topk(scores_row, k):
    """The unique k-subset S with: for a in S, b not in S, score_a > score_b
    or (score_a == score_b and a < b)."""
    C = len(scores_row)
    found = []
    for S in itertools.combinations(range(C), k):
        inside = set(S)
        ok = all(scores_row[a] > scores_row[b] or (scores_row[a] == scores_row[b] and a < b)
                 for a in inside for b in range(C) if b not in inside)
        if ok:
            found.append(list(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    block, chunk, n = 32, 4, 4
    vocab = 12 if seed % 2 else 40          # small vocab -> many ties
    ids = rng.integers(0, vocab, size=block * n)
    C = block // chunk
    for k in (0, 1, 3, C):
        sel, scores = oracle.select_summaries(ids, block, chunk, k, vocab, return_scores=True)
        for j in range(n):
            assert sel[j].tolist() == _brute_force_topk(scores[j].tolist(), k)


def test_scores_are_ln_n_over_min_df():
    w = workloads.TINY
    ids = w.token_ids()
    df = oracle.document_frequency(ids, w.block, w.vocab)
    idf = oracle.idf_table(df, w.n_blocks)
    sc = oracle.chunk_scores(ids, w.block, w.chunk, idf).reshape(-1)
    mdf = oracle.chunk_min_df(ids, w.block, w.chunk, df)
    np.testing.assert_allclose(sc, np.log(w.n_blocks / mdf.astype(np.float64)), rtol=0, atol=0)
    # strict monotonicity of ln(N/df) in df over 1..N, so ordering by score
    # equals ordering by integer min-df with the same ties
    vals = [math.log(w.n_blocks / x) for x in range(1, w.n_blocks + 1)]
    assert all(a > b for a, b in zip(vals, vals[1:]))


def test_planted_singletons_selected():
    # Zipf ids over a small vocabulary (no natural singletons) with 24 new ids
    # written once each: every block with <= k chunks holding a df = 1 token
    # selects all of them, and nothing else outranks them.
    block, chunk, k, n = 2048, 32, 8, 4
    ids = workloads.zipf_token_ids(n * block, 120, 1.1, seed=11).astype(np.int64)
    rng = np.random.default_rng(12)
    pos = rng.choice(ids.size, size=24, replace=False)
    ids[pos] = 120 + np.arange(24)
    df = oracle.document_frequency(ids, block, 144)
    assert sorted(np.nonzero(df == 1)[0].tolist()) == list(range(120, 144))
    sel = oracle.select_summaries(ids, block, chunk, k, 144)
    for j in range(n):
        planted_chunks = sorted({int(p % block) // chunk for p in pos if p // block == j})
        assert 0 < len(planted_chunks) <= k
        assert set(planted_chunks) <= set(sel[j].tolist())
        assert list(sel[j]) == sorted(sel[j])


def test_budget_and_prefix_arithmetic():
    # §5 of the Pulsar page: 4K blocks with 16 chunks of 32 tokens = 12.5 %.
    assert int(0.125 * 4096) // 32 == 16
    # §4: each later host adds 64 sink tokens + three 512-token summaries = 1600.
    L, b = 4 * 4096, 4096
    sel = np.tile(np.arange(16), (4, 1))
    pos = oracle.host_positions(L, b, 64, 32, sel)
    assert len(pos[3]) - b == 1600
    assert [len(p) for p in pos] == [4096, 4096 + 64 + 512, 4096 + 64 + 1024, 4096 + 1600]


def test_mean_idf_figure2():
    g = json.load(open(os.path.join(GOLDEN, "figure2_toy.json")))
    ids = np.array(g["ids"], dtype=np.int64)
    df = oracle.document_frequency(ids, g["block"], g["vocab"])
    idf = oracle.idf_table(df, 4)
    vals = {"0": 0.0, "log2": math.log(2.0), "log4/4": math.log(4.0) / 4}
    want = np.array([[vals[t] for t in row] for row in g["expected_mean_scores"]])
    np.testing.assert_allclose(oracle.chunk_mean_idf(ids, g["block"], g["chunk"], idf), want, rtol=0, atol=1e-15)
    assert oracle.select_summaries_mean_idf(ids, g["block"], g["chunk"], 1, g["vocab"]).tolist() == \
        g["expected_mean_idf_selection"]


def _tie_case(swap: bool):
    """N = 16 blocks of four 4-token chunks, worked by hand.  Token 0 is in
    every block (df 16, IDF 0), token 1 in block 0 only (df 1), token 2 in
    blocks 0..8 (df 9), tokens 3 and 4 in blocks 0..2 (df 3).  In block 0 the
    chunks {3, 4, 0, 0} and {1, 2, 0, 0} have the same mean IDF:
    (2 ln(16/3)) / 4 = (ln 16 + ln(16/9)) / 4, since ln 9 = 2 ln 3; the two
    all-filler chunks have mean 0."""
    F = 0
    blocks = []
    pair_a, pair_b = [3, 4, F, F], [1, 2, F, F]
    if swap:
        pair_a, pair_b = pair_b, pair_a
    blocks.append([F] * 4 + pair_a + pair_b + [F] * 4)
    for j in range(1, 16):
        head = [2 if j <= 8 else F, 3 if j <= 2 else F, 4 if j <= 2 else F, F]
        blocks.append(head + [F] * 12)
    ids = np.array(sum(blocks, []), dtype=np.int64)
    df = oracle.document_frequency(ids, 16, 5)
    assert df.tolist() == [16, 1, 9, 3, 3]
    return ids


@pytest.mark.parametrize("swap", [False, True])
def test_mean_idf_hand_worked_tie_at_n16(swap):
    ids = _tie_case(swap)
    idf = oracle.idf_table(oracle.document_frequency(ids, 16, 5), 16)
    m = oracle.chunk_mean_idf(ids, 16, 4, idf)[0]
    assert abs(m[1] - m[2]) < 1e-15 and abs(m[1] - 2 * math.log(16 / 3) / 4) < 1e-15
    # equal real means: the lower chunk index wins, whichever multiset it holds
    assert oracle.select_summaries_mean_idf(ids, 16, 4, 1, 5)[0].tolist() == [1]
    assert oracle.select_summaries_mean_idf(ids, 16, 4, 2, 5)[0].tolist() == [1, 2]
    _, rank = oracle.select_summaries_mean_idf(ids, 16, 4, 1, 5, return_rank=True)
    assert rank[:4].tolist() == [2, 0, 1, 3]


def _real_mean_idf_resolved(ids, block, chunk, vocab):
    """The definition evaluated to 60 significant digits: mean over each
    chunk's tokens of ln(N / df(t)), df counted by brute force over the
    blocks.  Means of c-token chunks with N <= 64 that differ at all differ
    by at least ln(1 + 64^-c) / c, above 1e-16 for c <= 8, so values closer
    than 1e-40 are the same real number; each value is replaced by the
    smallest value of its group of equals."""
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    n = len(ids) // block
    sets = [set(ids[j * block:(j + 1) * block].tolist()) for j in range(n)]
    C = block // chunk
    rows = []
    for j in range(n):
        vals = []
        for c in range(C):
            toks = ids[j * block + c * chunk:j * block + (c + 1) * chunk].tolist()
            tot = sum((Decimal(n) / Decimal(sum(t in s for s in sets))).ln() for t in toks)
            vals.append(tot / Decimal(chunk))
        srt = sorted(vals)
        rep = {}
        for v in srt:
            rep[v] = next(w for w in srt if abs(w - v) < Decimal("1e-40"))
        rows.append([rep[v] for v in vals])
    return rows


def _brute_force_real_order(n_blocks):
    """Brute force over every k-subset against the real-valued mean IDF
    (not the oracle's integer products).  Returns the number of exact real
    ties between chunks with different df multisets."""
    rng = np.random.default_rng(900 + n_blocks)
    block, chunk, vocab = 16, 2, 40
    # every id confined to a random set of blocks whose size is a power of
    # two, 3 or 9 (so that different df multisets often have equal products,
    # e.g. {1, 4} and {2, 2}, {1, 9} and {3, 3}); others of any size
    sizes = [z for z in (1, 2, 3, 4, 8, 9, 16, 32, 64) if z <= n_blocks]
    home = [rng.choice(n_blocks, size=int(rng.choice(sizes)) if t % 4 else int(rng.integers(1, n_blocks + 1)),
                       replace=False) for t in range(vocab)]
    ids = np.empty(n_blocks * block, dtype=np.int64)
    for j in range(n_blocks):
        allowed = [t for t in range(vocab) if j in home[t]] or [0]
        ids[j * block:(j + 1) * block] = rng.choice(allowed, size=block)
    real = _real_mean_idf_resolved(ids, block, chunk, vocab)
    df = oracle.document_frequency(ids, block, vocab)
    prods = oracle.chunk_df_product(ids, block, chunk, df)
    C = block // chunk
    cross_ties = 0
    for j in range(n_blocks):
        for a in range(C):
            for b in range(a + 1, C):
                ma = sorted(int(df[t]) for t in ids[j * block + a * chunk:j * block + (a + 1) * chunk])
                mb = sorted(int(df[t]) for t in ids[j * block + b * chunk:j * block + (b + 1) * chunk])
                cross_ties += real[j][a] == real[j][b] and ma != mb
    for k in (1, 3, 5):
        sel, rank = oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab, return_rank=True)
        for j in range(n_blocks):
            assert sel[j].tolist() == _brute_force_topk(real[j], k)
            order = sorted(range(C), key=lambda c: (-real[j][c], c))
            assert [int(rank[j * C + c]) for c in order] == list(range(C))
    assert len(prods) == n_blocks * C
    return cross_ties


@pytest.mark.parametrize("n_blocks", [16, 32, 64])
def test_mean_idf_brute_force_real_order(n_blocks):
    _brute_force_real_order(n_blocks)


@pytest.mark.parametrize("n_blocks", [16, 32, 64])
def test_mean_idf_planted_ties_real_order(n_blocks):
    """Ids whose df values are fixed by construction (1, 2, 3, 4, 8, 9, 16 and
    the filler's N), paired into 2-token chunks: many chunks with different
    df multisets have equal real means ({1, 4} and {2, 2}, {1, 9} and {3, 3},
    {2, 8} and {4, 4}, ...).  The oracle's full order must be the real-valued
    order, ties to the lower index."""
    block, chunk = 64, 2
    ids = workloads.windowed_token_ids(n_blocks, block, seed=40 + n_blocks).astype(np.int64)
    vocab = 1 + 7 * n_blocks
    real = _real_mean_idf_resolved(ids, block, chunk, vocab)
    df = oracle.document_frequency(ids, block, vocab)
    C = block // chunk
    cross = 0
    for j in range(n_blocks):
        ms = [sorted(int(df[t]) for t in ids[j * block + c * chunk:j * block + (c + 1) * chunk]) for c in range(C)]
        cross += sum(real[j][a] == real[j][b] and ms[a] != ms[b] for a in range(C) for b in range(a + 1, C))
    assert cross >= n_blocks, cross
    for k in (1, 4, 11):
        sel, rank = oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab, return_rank=True)
        for j in range(n_blocks):
            order = sorted(range(C), key=lambda c: (-real[j][c], c))
            assert sel[j].tolist() == sorted(order[:k])
            assert [int(rank[j * C + c]) for c in order] == list(range(C))


def test_mean_idf_brute_force_has_cross_multiset_ties():
    # the brute-force cases must include equal real means reached by
    # different df multisets (the case a rounded score can get wrong)
    ties = [_brute_force_real_order(n) for n in (16, 32, 64)]
    assert sum(ties) > 0, ties


def test_evenly_spaced_closed_form():
    sel = oracle.select_evenly_spaced(3, 4096, 32, 16)      # 128 chunks, 16 kept: every 8th
    assert sel.shape == (3, 16) and sel[1].tolist() == list(range(0, 128, 8))
    assert oracle.select_evenly_spaced(1, 96, 32, 3).tolist() == [[0, 1, 2]]
    assert oracle.select_evenly_spaced(2, 320, 32, 3).tolist() == [[0, 3, 6]] * 2


# --------------------------------------------------------------------------
# entropy and BM25 scorers (named on the Pulsar page, §3.1 / Table 1, without
# formulas: the textbook definitions, pinned by closed forms and hand-worked
# values)
# --------------------------------------------------------------------------
def test_entropy_closed_forms():
    ids = np.array(list(range(8)) + [5] * 8 + [1, 1, 2, 2, 3, 3, 4, 4] + [9, 9, 9, 9, 1, 2, 3, 4], dtype=np.int64)
    h = oracle.chunk_entropy(ids, 32, 8)[0]
    assert abs(h[0] - math.log(8)) < 1e-15           # all distinct: ln |c|
    assert h[1] == 0.0                               # one token repeated
    # tf multisets {2, 2, 2, 2} and {4, 1, 1, 1, 1}: ln 8 - (1/8) 4 (2 ln 2)
    # = ln 8 - (1/8) 4 ln 4 = ln 4, the same real number
    assert abs(h[2] - math.log(4)) < 1e-15 and abs(h[3] - math.log(4)) < 1e-15
    prod = oracle.chunk_tf_power_product(ids, 32, 8)
    assert prod == [1, 8 ** 8, 256, 256]


@pytest.mark.parametrize("swap", [False, True])
def test_entropy_hand_worked_tie_goes_to_the_lower_index(swap):
    a = [1, 1, 2, 2, 3, 3, 4, 4]
    b = [9, 9, 9, 9, 1, 2, 3, 4]
    if swap:
        a, b = b, a
    ids = np.array([5] * 8 + a + b + [6, 6, 7, 7, 7, 7, 7, 7], dtype=np.int64)
    sel, rank = oracle.select_summaries_entropy(ids, 32, 8, 1, return_rank=True)
    assert sel.tolist() == [[1]]
    assert rank.tolist() == [3, 0, 1, 2]


def _real_entropy_resolved(ids, block, chunk):
    """-sum p ln p of every chunk to 60 digits; entropies of different tf
    multisets with c <= 8 tokens differ by more than 1e-16, so values closer
    than 1e-40 are the same real number (each replaced by the smallest of its
    group)."""
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    n, C = len(ids) // block, block // chunk
    rows = []
    for j in range(n):
        vals = []
        for c in range(C):
            toks = ids[j * block + c * chunk:j * block + (c + 1) * chunk].tolist()
            tot = Decimal(0)
            for t in set(toks):
                p = Decimal(toks.count(t)) / Decimal(chunk)
                tot -= p * p.ln()
            vals.append(tot)
        srt = sorted(vals)
        rows.append([next(w for w in srt if abs(w - v) < Decimal("1e-40")) for v in vals])
    return rows


@pytest.mark.parametrize("seed", range(3))
def test_entropy_brute_force_real_order(seed):
    rng = np.random.default_rng(70 + seed)
    block, chunk = 64, 8
    ids = rng.integers(0, 6, size=block * 3)        # few distinct ids: many equal entropies
    real = _real_entropy_resolved(ids, block, chunk)
    C = block // chunk
    for k in (1, 3, 6):
        sel = oracle.select_summaries_entropy(ids, block, chunk, k)
        for j in range(3):
            assert sel[j].tolist() == _brute_force_topk(real[j], k)


def test_bm25_hand_worked():
    # N = 2 blocks of 4 ids, 2-token chunks: df(1) = df(3) = df(4) = 1,
    # df(2) = 2; idf = ln(1 + (N - df + 0.5)/(df + 0.5)): ln 2 for df 1,
    # ln 1.2 for df 2; tf weight tf (k1 + 1)/(tf + k1) with k1 = 1.2: 1 for
    # tf 1, 4.4 / 3.2 = 1.375 for tf 2.
    ids = np.array([1, 1, 2, 3, 2, 4, 4, 4], dtype=np.int64)
    got = oracle.chunk_bm25(ids, 4, 2, 5)
    l2, l12 = math.log(2.0), math.log(1.2)
    want = [1.375 * l2, l12 + l2, l12 + l2, 1.375 * l2]
    assert np.allclose(got, want, rtol=0, atol=1e-15)
    assert oracle.select_summaries_bm25(ids, 4, 2, 1, 5).tolist() == [[0], [1]]
