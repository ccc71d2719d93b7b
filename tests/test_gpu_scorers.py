"""GPU parity of the alternative summary scorers (Pulsar Attention page
§3.1, Table 1): mean-IDF on the fixed-point scale and evenly spaced
sampling, bit-exact against the oracle; Max-IDF through the scored entry
point equals pulsar_select_summaries."""
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


@pytest.mark.parametrize("idx", range(5))
def test_mean_idf_and_evenly_spaced(P, idx):
    ids, vocab, block, chunk, k = list(_cases())[idx]
    ids = ids.astype(np.int32)
    dev_ids = torch.from_numpy(ids).to(DEV)
    sel, sc, ws = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_MEAN_IDF,
                                                  want_scores=True)
    assert P.pa_workspace_status(ws) == 0
    df = oracle.document_frequency(ids, block, vocab)
    assert np.array_equal(sc.cpu().numpy(), oracle.chunk_mean_idf_fixed(ids, block, chunk, df))
    assert np.array_equal(sel.cpu().numpy(), oracle.select_summaries_mean_idf(ids, block, chunk, k, vocab))
    sel2, _, _ = P.pulsar_select_summaries_scored(None, vocab, block, chunk, k, P.PA_SCORE_EVENLY_SPACED,
                                                 L=ids.size)
    assert np.array_equal(sel2.cpu().numpy(), oracle.select_evenly_spaced(ids.size // block, block, chunk, k))
    sel3, sc3, _ = P.pulsar_select_summaries_scored(dev_ids, vocab, block, chunk, k, P.PA_SCORE_MAX_IDF,
                                                   want_scores=True)
    ref, _, mdf, _ = P.pulsar_select_summaries(dev_ids, vocab, block, chunk, k, want_mindf=True)
    assert torch.equal(sel3, ref)
    assert torch.equal(sc3, mdf.to(torch.int64))
