"""The allocation-free selection entry point, for callers that cannot
allocate device memory (a plugin inside an application that owns all device
allocations, or a serving thread that must never call cudaMalloc).

Calls pulsar_select_summaries_noalloc through the C ABI twice in a row, on
two different inputs, and checks each result against the workspace-based
pulsar_select_summaries (selection is integer work: the comparison is
exact).  The second call would differ if the shared scratch array kept
stale block masks from the first.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

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


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from long_context_blockwise_max_b200 import pulsar as P
    dev = torch.device("cuda:0")
    ids = torch.zeros(4096, dtype=torch.int32, device=dev)
    sel = torch.empty((4, 1), dtype=torch.int32, device=dev)
    with pytest.raises(P.PulsarError) as e:
        P.pulsar_select_summaries_noalloc(ids, 262145, 1024, 32, 1, sel)
    assert e.value.code == -2
