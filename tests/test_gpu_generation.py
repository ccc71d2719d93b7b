"""GPU parity of the query-host step and the generation loop: a query of Tq
tokens, then tokens generated one at a time, each appending its own K/V and
attending to the retained shards plus its own earlier tokens (causal).
Every step's rows must equal the oracle's one-shot result for the same
rows; all steps' rows together must equal a single batched call."""
import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


@pytest.mark.parametrize("dtype,B,Tq0,gen,T,S,hq,hkv,d,theta", [
    (torch.bfloat16, 2, 16, 12, 3000, 4, 32, 8, 128, 500000.0),
    (torch.bfloat16, 1, 64, 4, 4096, 8, 32, 8, 128, 500000.0),    # 256 rows per kv head: row-split kernel
    (torch.float32, 1, 5, 7, 700, 3, 4, 2, 64, 10000.0),
])
def test_query_then_generate(P, dtype, B, Tq0, gen, T, S, hq, hkv, d, theta):
    n_tok = Tq0 + gen
    q = workloads.normal((B, n_tok, hq, d), 80, dtype)
    kn = workloads.normal((B, n_tok, hkv, d), 81, dtype)
    vn = workloads.normal((B, n_tok, hkv, d), 82, dtype)
    kc = workloads.normal((B, T, hkv, d), 83, dtype)
    vc = workloads.normal((B, T, hkv, d), 84, dtype)
    qd, knd, vnd, kcd, vcd = (t.to(DEV) for t in (q, kn, vn, kc, vc))
    cap = n_tok + 3
    k_self = torch.zeros((B, cap, hkv, d), dtype=dtype, device=DEV)
    v_self = torch.zeros((B, cap, hkv, d), dtype=dtype, device=DEV)
    outs, lses = [], []
    # the query, then one token at a time
    steps = [(0, Tq0)] + [(Tq0 + i, 1) for i in range(gen)]
    for start, n in steps:
        o, lse, ws = P.star_phase2_query_step(qd[:, start:start + n].contiguous(), knd[:, start:start + n].contiguous(),
                                              vnd[:, start:start + n].contiguous(), kcd, vcd, S, k_self, v_self,
                                              start, T + start, theta)
        assert P.pa_workspace_status(ws) == 0
        outs.append(o.cpu())
        lses.append(lse.cpu())
    o_all = torch.cat(outs, dim=1)
    lse_all = torch.cat(lses, dim=1)
    # oracle: own keys are the new tokens' K rotated at T + j
    ks_ref = np.stack([oracle.rope(f64(kn[b]), T + np.arange(n_tok), theta) for b in range(B)])
    ro, rl = oracle.phase2_attend_with_self(f64(q), f64(kc), f64(vc), S, ks_ref, f64(vn), 0, T, theta)
    assert_close(f64(o_all), ro, O_TOL[dtype], "O")
    assert_close(lse_all.double().numpy(), rl, LSE_TOL, "lse")
    # the own cache holds the rotated K (input dtype) and V of every token
    assert torch.equal(v_self[:, :n_tok].cpu(), vn)
    tol = 1e-5 if dtype == torch.float32 else 2.0 ** -8 * np.abs(ks_ref) + 1e-5
    assert (np.abs(f64(k_self[:, :n_tok].cpu()) - ks_ref) <= tol).all()
