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


def test_mean_idf_figure2_and_fixed_scale():
    g = json.load(open(os.path.join(GOLDEN, "figure2_toy.json")))
    ids = np.array(g["ids"], dtype=np.int64)
    df = oracle.document_frequency(ids, g["block"], g["vocab"])
    idf = oracle.idf_table(df, 4)
    vals = {"0": 0.0, "log2": math.log(2.0), "log4/4": math.log(4.0) / 4}
    want = np.array([[vals[t] for t in row] for row in g["expected_mean_scores"]])
    np.testing.assert_allclose(oracle.chunk_mean_idf(ids, g["block"], g["chunk"], idf), want, rtol=0, atol=1e-15)
    assert oracle.select_summaries_mean_idf(ids, g["block"], g["chunk"], 1, g["vocab"]).tolist() == \
        g["expected_mean_idf_selection"]
    # the fixed-point table: q[df] ~ ln(N/df) * 2^24, q[N] = 0
    q = oracle.idf_fixed_table(4)
    assert q[4] == 0 and abs(q[1] - math.log(4.0) * 2 ** 24) <= 0.5 and abs(q[2] - math.log(2.0) * 2 ** 24) <= 0.5
    fx = oracle.chunk_mean_idf_fixed(ids, g["block"], g["chunk"], df).reshape(4, 4)
    assert (np.abs(fx / 2.0 ** 24 / g["chunk"] - want) <= 4 * 0.5 / 2 ** 24 / g["chunk"] + 1e-15).all()


@pytest.mark.parametrize("seed", range(4))
def test_mean_idf_brute_force(seed):
    rng = np.random.default_rng(500 + seed)
    block, chunk, n, vocab = 32, 4, 4, 14
    ids = rng.integers(0, vocab, size=block * n)
    df = oracle.document_frequency(ids, block, vocab)
    sc = oracle.chunk_mean_idf_fixed(ids, block, chunk, df).reshape(n, block // chunk)
    for k in (1, 3, 8):
        sel = oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab)
        for j in range(n):
            assert sel[j].tolist() == _brute_force_topk(sc[j].tolist(), k)


def test_evenly_spaced_closed_form():
    sel = oracle.select_evenly_spaced(3, 4096, 32, 16)      # 128 chunks, 16 kept: every 8th
    assert sel.shape == (3, 16) and sel[1].tolist() == list(range(0, 128, 8))
    assert oracle.select_evenly_spaced(1, 96, 32, 3).tolist() == [[0, 1, 2]]
    assert oracle.select_evenly_spaced(2, 320, 32, 3).tolist() == [[0, 3, 6]] * 2
