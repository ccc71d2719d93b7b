"""The multi-GPU layout's GPU functions, run on the one GPU a test gets: a
process group of world size 1 over NCCL executes phase1_encode_distributed
(pulsar_phase1_encode_hosts / star_phase1_encode_hosts on the rank's host
range) and phase2_attend_distributed (star_phase2_attend partials, packed,
NCCL all_gather_into_tensor, pa_lse_merge) with their default GPU steps,
and both are compared with the fp64 oracle (Pulsar Attention page §2.1 and
§2.2: Phase 1 without communication, then the all-gather of the hosts'
partials and the online-softmax merge).  The host ranges, padding and
gather order across several ranks are covered on CPU with gloo."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    import datetime
    torch.cuda.set_device(DEV)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=DEV)
    try:
        yield dist.group.WORLD
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("star", [False, True])
def test_phase1_encode_distributed_on_nccl(nccl_group, star):
    from long_context_blockwise_max_b200 import distributed as D
    L, block, hq, hkv, d, sink, chunk, kc, theta = 4 * 640, 640, 8, 2, 128, 64, 32, 3, 500000.0
    ids = workloads.zipf_token_ids(L, 300, 1.1, seed=31)
    sel = oracle.select_summaries(ids, block, chunk, kc, 300)
    q = workloads.normal((L, hq, d), 32, torch.bfloat16)
    k = workloads.normal((L, hkv, d), 33, torch.bfloat16)
    v = workloads.normal((L, hkv, d), 34, torch.bfloat16)
    o, lse, kr, vr, (h0, h1) = D.phase1_encode_distributed(
        q.to(DEV), k.to(DEV), v.to(DEV), theta, block, sink, chunk, kc,
        torch.from_numpy(sel.astype(np.int32)).to(DEV), star, group=nccl_group)
    assert (h0, h1) == (0, L // block)
    pos = oracle.host_positions(L, block, sink, chunk, sel, star=star)
    off = oracle.host_row_offsets(pos)
    ref = oracle.phase1_encode(f64(q), f64(k), f64(v), pos, theta)
    for i, (ro, rl) in enumerate(ref):
        assert_close(f64(o[off[i]:off[i + 1]].cpu()), ro, O_TOL[torch.bfloat16], f"host {i} O")
        assert_close(lse[off[i]:off[i + 1]].cpu().double().numpy(), rl, LSE_TOL, f"host {i} lse")
    assert torch.equal(vr.cpu(), v)
    kref, _ = oracle.retained_kv(f64(k), f64(v), theta)
    tol = 2.0 ** -8 * np.abs(kref) + 1e-5 * np.linalg.norm(f64(k), axis=-1, keepdims=True)
    assert (np.abs(f64(kr.cpu()) - kref) <= tol).all()


@pytest.mark.parametrize("case", [
    # (B, Tq, T, shards, hq, hkv, d, theta)
    (1, 64, 3000, 5, 8, 2, 128, 500000.0),   # 256 rows per kv head: the tensor-core query kernel
    (2, 1, 1111, 4, 32, 8, 128, 500000.0),   # decode rows: the mma.sync kernel, ragged shards
    (1, 3, 10, 16, 4, 4, 64, 0.0),           # more shards than keys: empty shards in the exchange
])
def test_phase2_attend_distributed_on_nccl(nccl_group, case):
    from long_context_blockwise_max_b200 import distributed as D
    B, Tq, T, S, hq, hkv, d, theta = case
    q = workloads.normal((B, Tq, hq, d), 35, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 36, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 37, torch.bfloat16)
    o, lse = D.phase2_attend_distributed(q.to(DEV), kc.to(DEV), vc.to(DEV), S, S, T, theta, group=nccl_group)
    ro, rl, _, _ = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, theta)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.bfloat16], "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
