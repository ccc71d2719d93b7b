"""Failure detection on the GPU without a fault: a barrier that can never
complete makes every bounded wait of a tensor-core kernel (Phase 1, and the
Phase-2 query kernel) run out; the kernel records PA_ERR_TIMEOUT, frees its
resources and returns, and the next call on the same context computes
correct results."""
import time

import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def test_stalled_barrier_times_out_and_context_survives():
    from long_context_blockwise_max_b200 import pulsar as P
    L, block, hq, hkv, d = 256, 128, 4, 2, 128
    q = workloads.normal((L, hq, d), 90, torch.bfloat16)
    k = workloads.normal((L, hkv, d), 91, torch.bfloat16)
    v = workloads.normal((L, hkv, d), 92, torch.bfloat16)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    t0 = time.time()
    ws = P.pa_testing_phase1_stall(qd, kd, vd, block, wait_limit_us=20000)
    assert P.pa_workspace_status(ws) == -5          # PA_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    # the same context still runs a normal call correctly
    o, lse, _, _, off, ws2 = P.star_phase1_encode(qd, kd, vd, 10000.0, block)
    assert P.pa_workspace_status(ws2) == 0
    pos = oracle.host_positions(L, block, 0, 16, np.zeros((2, 0), dtype=np.int64), star=True)
    for i, (ro, rl) in enumerate(oracle.phase1_encode(f64(q), f64(k), f64(v), pos, 10000.0)):
        assert_close(f64(o[off[i]:off[i + 1]].cpu()), ro, O_TOL[torch.bfloat16], "O")
        assert_close(lse[off[i]:off[i + 1]].cpu().double().numpy(), rl, LSE_TOL, "lse")



def test_stalled_query_kernel_times_out_and_context_survives():
    from long_context_blockwise_max_b200 import pulsar as P
    B, Tq, hq, hkv, d, T, S = 1, 64, 8, 2, 128, 1000, 3   # 256 query rows per kv head
    q = workloads.normal((B, Tq, hq, d), 93, torch.bfloat16)
    kc = workloads.normal((B, T, hkv, d), 94, torch.bfloat16)
    vc = workloads.normal((B, T, hkv, d), 95, torch.bfloat16)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    t0 = time.time()
    ws = P.pa_testing_phase2_stall(qd, kd, vd, S, wait_limit_us=20000)
    assert P.pa_workspace_status(ws) == -5          # PA_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    o, lse, _, _, ws2 = P.star_phase2_attend(qd, kd, vd, S, q_pos0=T, rope_theta=0.0)
    assert P.pa_workspace_status(ws2) == 0
    ro, rl, _, _ = oracle.phase2_attend(f64(q), f64(kc), f64(vc), S, T, 0.0)
    assert_close(f64(o.cpu()), ro, O_TOL[torch.bfloat16], "O")
    assert_close(lse.cpu().double().numpy(), rl, LSE_TOL, "lse")
