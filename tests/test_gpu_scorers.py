"""GPU parity of the alternative summary scorers (Pulsar Attention page
§3.1, Table 1): mean-IDF and entropy (exact orders, ties to the lower index)
and evenly spaced sampling, bit-exact against the oracle -- the selection and
every chunk's rank; BM25 (fp64) against the oracle's order except among
scores equal to fp64 rounding; Max-IDF through the scored entry point
against the oracle's selection and min df."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def _cases():
    g = json.load(open(os.path.join(GOLDEN, "figure2_toy.json")))
    yield np.array(g["ids"]), g["vocab"], g["block"], g["chunk"], 1
    yield workloads.zipf_token_ids(4096, 50, 1.1, seed=9), 50, 1024, 32, 5
    yield workloads.zipf_token_ids(64 * 16, 30, 0.5, seed=8), 30, 16, 16, 1
    yield workloads.zipf_token_ids(8 * 4096, 700, 1.1, seed=7), 700, 4096, 32, 16
    w = workloads.LLAMA_32K
    yield w.token_ids(), w.vocab, w.block, w.chunk, w.k_chunks
    # df fixed by construction (1, 2, 3, 4, 8, 9, 16 and N): many equal real
    # means from different df multisets ({1, 9} and {3, 3}, {2, 8} and {4, 4})
    # at N = 16, 32 and 64, in 2-token and 32-token chunks
    for n in (16, 32, 64):
        yield workloads.windowed_token_ids(n, 64, seed=40 + n), 1 + 7 * n, 64, 2, 11
    yield workloads.windowed_token_ids(64, 1024, seed=5), 1 + 7 * 64, 1024, 32, 4   # products up to 2^192


N_CASES = 9


def _check_bm25(P, dev_ids, ids, vocab, block, chunk, k):
    """BM25 is an fp64 score (the kernel's and the oracle's logarithms may
    differ in the last bit): every chunk's rank must equal the oracle's
    unless its score is within 1e-12 (relative) of another chunk's of the
    same block, where only the order among those near-equal chunks may
    differ; the selection must be the oracle's unless the k-th and (k+1)-th
    best scores are within 1e-12."""
    sel, rank, ws = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_BM25,
                                                    want_scores=True)
    assert P.pa_workspace_status(ws) == 0
    n, C = ids.size // block, block // chunk
    sc = oracle.chunk_bm25(ids, block, chunk, vocab).reshape(n, C)
    want_sel = oracle.select_summaries_bm25(ids, block, chunk, k, vocab)
    got_rank = rank.cpu().numpy().reshape(n, C)
    got_sel = sel.cpu().numpy()
    for j in range(n):
        order = sorted(range(C), key=lambda c: (-sc[j, c], c))
        near = lambda a, b: abs(a - b) <= 1e-12 * max(abs(a), abs(b), 1.0)
        for r, c in enumerate(order):
            if got_rank[j, c] != r:   # allowed only inside a group of near-equal scores
                assert near(sc[j, c], sc[j, order[got_rank[j, c]]]), (j, c, r, got_rank[j, c])
        if 0 < k < C and near(sc[j, order[k - 1]], sc[j, order[k]]):
            continue
        assert got_sel[j].tolist() == want_sel[j].tolist(), j


@pytest.mark.parametrize("idx", range(N_CASES))
def test_mean_idf_and_evenly_spaced(P, idx):
    ids, vocab, block, chunk, k = list(_cases())[idx]
    ids = ids.astype(np.int32)
    dev_ids = torch.from_numpy(ids).to(DEV)
    sel, rank, ws = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_MEAN_IDF,
                                                    want_scores=True)
    assert P.pa_workspace_status(ws) == 0
    want_sel, want_rank = oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab, return_rank=True)
    assert np.array_equal(rank.cpu().numpy(), want_rank)
    assert np.array_equal(sel.cpu().numpy(), want_sel)
    sel_nr, none, _ = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_MEAN_IDF)
    assert none is None and np.array_equal(sel_nr.cpu().numpy(), want_sel)
    sel2, _, _ = P.pulsar_select_summaries_scored(None, vocab, block, chunk, k, P.PA_SCORE_EVENLY_SPACED,
                                                 L=ids.size)
    assert np.array_equal(sel2.cpu().numpy(), oracle.select_evenly_spaced(ids.size // block, block, chunk, k))
    # entropy: exact order (integer prod tf^tf), bit-exact selection and ranks
    sel_e, rank_e, ws = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_ENTROPY,
                                                        want_scores=True)
    assert P.pa_workspace_status(ws) == 0
    want_e, want_re = oracle.select_summaries_entropy(ids, block, chunk, k, return_rank=True)
    assert np.array_equal(rank_e.cpu().numpy(), want_re)
    assert np.array_equal(sel_e.cpu().numpy(), want_e)
    _check_bm25(P, dev_ids, ids, vocab, block, chunk, k)
    sel3, sc3, _ = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_MAX_IDF,
                                                   want_scores=True)
    df = oracle.document_frequency(ids, block, vocab)
    assert np.array_equal(sel3.cpu().numpy(), oracle.select_summaries(ids, block, chunk, k, vocab))
    assert np.array_equal(sc3.cpu().numpy(), oracle.chunk_min_df(ids, block, chunk, df))


def test_mean_idf_hand_worked_tie(P):
    """N = 16, chunks with df {3, 3, 16, 16} and {1, 9, 16, 16}: equal real
    means, so the lower index wins whichever of the two it holds."""
    for swap in (False, True):
        F = 0
        a, b = [3, 4, F, F], [1, 2, F, F]
        if swap:
            a, b = b, a
        blocks = [[F] * 4 + a + b + [F] * 4]
        for j in range(1, 16):
            blocks.append([2 if j <= 8 else F, 3 if j <= 2 else F, 4 if j <= 2 else F, F] + [F] * 12)
        ids = torch.tensor(sum(blocks, []), dtype=torch.int32, device=DEV)
        sel, rank, _ = P.pulsar_select_summaries_scored(ids, 5, 16, 4, 1, P.PA_SCORE_MEAN_IDF, want_scores=True)
        assert sel[0].tolist() == [1]
        assert rank[:4].tolist() == [2, 0, 1, 3]


def test_scorers_at_the_1m_scale_shape(P):
    # 1M Zipf ids, 32 blocks of 32768, 1024 chunks per block, 128 kept: mean
    # IDF and entropy bit-exact (selection and ranks), BM25 by order
    w = workloads.SCALE_1M
    ids = w.token_ids()
    dev_ids = torch.from_numpy(ids).to(DEV)
    for method, ref in ((P.PA_SCORE_MEAN_IDF,
                         lambda: oracle.select_summaries_mean_idf(ids, w.block, w.chunk, w.k_chunks, w.vocab,
                                                                  return_rank=True)),
                        (P.PA_SCORE_ENTROPY,
                         lambda: oracle.select_summaries_entropy(ids, w.block, w.chunk, w.k_chunks,
                                                                 return_rank=True))):
        sel, rank, ws = P.pulsar_select_summaries_scored(dev_ids, w.vocab, w.block, w.chunk, w.k_chunks, method,
                                                        want_scores=True)
        assert P.pa_workspace_status(ws) == 0
        want_sel, want_rank = ref()
        assert np.array_equal(sel.cpu().numpy(), want_sel), method
        assert np.array_equal(rank.cpu().numpy(), want_rank), method
    _check_bm25(P, dev_ids, ids, w.vocab, w.block, w.chunk, w.k_chunks)


@pytest.mark.parametrize("case", [
    # (L, vocab, block, chunk, k, what)
    (512, 40, 512, 32, 3, "one block: every df is 1, all means equal"),
    (2048, 40, 512, 32, 0, "k = 0"),
    (2048, 40, 512, 32, 16, "k = C: every chunk kept"),
    (1024, 30, 256, 1, 5, "one-token chunks"),
    (2048, 1, 512, 32, 4, "a one-id vocabulary: every score equal"),
    (64 * 64, 50, 64, 32, 1, "64 blocks, two chunks each"),
])
def test_scorer_edge_cases(P, case):
    L, vocab, block, chunk, k, _ = case
    ids = workloads.zipf_token_ids(L, vocab, 1.0, seed=L + vocab)
    dev_ids = torch.from_numpy(ids).to(DEV)
    for method in (P.PA_SCORE_MEAN_IDF, P.PA_SCORE_ENTROPY):
        sel, rank, ws = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, method, want_scores=True)
        assert P.pa_workspace_status(ws) == 0
        if method == P.PA_SCORE_MEAN_IDF:
            want_sel, want_rank = oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab, return_rank=True)
        else:
            want_sel, want_rank = oracle.select_summaries_entropy(ids, block, chunk, k, return_rank=True)
        assert np.array_equal(sel.cpu().numpy().reshape(want_sel.shape), want_sel), (case, method)
        assert np.array_equal(rank.cpu().numpy(), want_rank), (case, method)
    _check_bm25(P, dev_ids, ids, vocab, block, chunk, k)
