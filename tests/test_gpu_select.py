"""GPU parity of Max-IDF selection against the oracle: bit-exact selected
chunk indices, document frequencies and chunk min-df (Pulsar Attention page,
§2.1)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def _check(P, ids, vocab, block, chunk, k):
    dev = torch.device("cuda:0")
    sel, df, mdf, ws = P.pulsar_select_summaries(torch.from_numpy(ids.astype(np.int32)).to(dev), vocab, block,
                                                 chunk, k, want_df=True, want_mindf=True)
    assert P.pa_workspace_status(ws) == 0
    df_ref = oracle.document_frequency(ids, block, vocab)
    assert np.array_equal(df.cpu().numpy(), df_ref)
    assert np.array_equal(mdf.cpu().numpy(), oracle.chunk_min_df(ids, block, chunk, df_ref))
    assert np.array_equal(sel.cpu().numpy(), oracle.select_summaries(ids, block, chunk, k, vocab))


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_select_workloads(P, name):
    w = workloads.WORKLOADS[name]
    _check(P, w.token_ids(), w.vocab, w.block, w.chunk, w.k_chunks)


CASES = [
    # (L, vocab, block, chunk, k, zipf_s)  -- small vocabularies spread df over 1..N
    (4096, 50, 1024, 32, 5, 1.1),
    (64 * 16, 30, 16, 16, 1, 0.5),          # N = 64 blocks, the maximum
    (3 * 480, 200, 480, 48, 3, 1.1),        # chunk 48: lanes loop over a chunk
    (2048, 1000, 2048, 4, 0, 1.1),          # N = 1, k = 0
    (2048, 100, 512, 8, 64, 1.1),           # k = all chunks
    (1024, 64, 256, 1, 17, 0.8),            # one-token chunks
    (24 * 1000, 300, 1000, 40, 7, 1.3),     # blocks not a multiple of 32
    (8 * 32768, 2000, 32768, 32, 512, 1.1), # 1024 chunks per block, several tiles of the compaction
    (4 * 8192, 1 << 20, 8192, 32, 16, 1.1), # vocabulary of 2^20 ids: the largest shared-memory bitmap
    (4 * 1024, 1500000, 1024, 32, 4, 1.1),  # vocabulary above 2^20 ids: the per-warp dedupe kernel
    (7 * 640, 500, 640, 32, 3, 0.3),        # tiles end at block ends inside the per-tile kernel
]


@pytest.mark.parametrize("case", CASES)
def test_select_edge_cases(P, case):
    L, vocab, block, chunk, k, s = case
    ids = workloads.zipf_token_ids(L, vocab, s, seed=L + vocab)
    _check(P, ids, vocab, block, chunk, k)


def test_select_invalid_id_sets_status(P):
    ids = workloads.zipf_token_ids(2048, 100, 1.1, seed=3)
    ids[777] = 100          # == vocab: out of range
    dev = torch.device("cuda:0")
    _, _, _, ws = P.pulsar_select_summaries(torch.from_numpy(ids).to(dev), 100, 512, 32, 2)
    assert P.pa_workspace_status(ws) == -1   # PA_ERR_INVALID recorded on the device
