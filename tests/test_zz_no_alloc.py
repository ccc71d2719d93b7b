"""The allocation-free selection entry point, for callers that cannot
allocate device memory (a plugin inside an application that owns all device
allocations, or a serving thread that must never call cudaMalloc).

Calls pulsar_select_summaries_noalloc through the C ABI twice in a row, on
two different inputs, and checks each result against the workspace-based
pulsar_select_summaries and against the fp64 oracle (selection is integer
work: the comparisons are exact).  The second call would differ if the
shared scratch array kept stale block masks from the first.  A third case
passes no df / min-df outputs, so the min df goes to the array's own region,
at the largest chunk count it holds.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    from long_context_blockwise_max_b200 import pulsar as P
    dev = torch.device("cuda:0")
    cases = [
        (workloads.LLAMA_32K.token_ids(), 128256, 8192, 32, 32),
        (workloads.zipf_token_ids(8 * 2048, 300, 1.1, seed=77), 300, 2048, 32, 8),
    ]
    for ids_np, vocab, block, chunk, k in cases:
        ids = torch.from_numpy(ids_np.astype(np.int32)).to(dev)
        n = ids.numel() // block
        sel = torch.full((n, k), -7, dtype=torch.int32, device=dev)
        df = torch.full((vocab,), -7, dtype=torch.int32, device=dev)
        mdf = torch.full((ids.numel() // chunk,), -7, dtype=torch.int32, device=dev)
        P.pulsar_select_summaries_noalloc(ids, vocab, block, chunk, k, sel, df, mdf)
        ref_sel, ref_df, ref_mdf, ws = P.pulsar_select_summaries(ids, vocab, block, chunk, k, want_df=True,
                                                                 want_mindf=True)
        assert P.pa_workspace_status(ws) == 0
        torch.cuda.synchronize()
        assert torch.equal(sel, ref_sel)
        assert torch.equal(df, ref_df)
        assert torch.equal(mdf, ref_mdf)
        odf = oracle.document_frequency(ids_np, block, vocab)
        assert np.array_equal(sel.cpu().numpy(), oracle.select_summaries(ids_np, block, chunk, k, vocab))
        assert np.array_equal(df.cpu().numpy(), odf)
        assert np.array_equal(mdf.cpu().numpy(), oracle.chunk_min_df(ids_np, block, chunk, odf))


def test_noalloc_without_df_outputs_at_the_chunk_limit():
    # 2^21 ids in 32 blocks of 65536: 65536 chunks, the most the scratch array
    # holds; df and min df not requested (min df in the array's own region)
    from long_context_blockwise_max_b200 import pulsar as P
    dev = torch.device("cuda:0")
    L, vocab, block, chunk, k = 1 << 21, 128256, 65536, 32, 256
    ids_np = workloads.zipf_token_ids(L, vocab, 1.1, seed=78, planted=500)
    ids = torch.from_numpy(ids_np).to(dev)
    for _ in range(2):
        sel = torch.full((L // block, k), -7, dtype=torch.int32, device=dev)
        P.pulsar_select_summaries_noalloc(ids, vocab, block, chunk, k, sel)
        torch.cuda.synchronize()
        assert np.array_equal(sel.cpu().numpy(), oracle.select_summaries(ids_np, block, chunk, k, vocab))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from long_context_blockwise_max_b200 import pulsar as P
    dev = torch.device("cuda:0")
    ids = torch.zeros(4096, dtype=torch.int32, device=dev)
    sel = torch.empty((4, 1), dtype=torch.int32, device=dev)
    with pytest.raises(P.PulsarError) as e:
        P.pulsar_select_summaries_noalloc(ids, 262145, 1024, 32, 1, sel)
    assert e.value.code == -2
