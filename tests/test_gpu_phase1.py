"""GPU parity of Phase-1 encoding (Pulsar and the Star anchor variant)
against the fp64 oracle: every row at small sizes (several 128-row tiles and
ragged tails), sampled rows of every host at the 32K and 128K Llama-3.1-8B
attention shapes, and the retained cache layout."""
import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_TOL, O_TOL, assert_close, f64, sample_rows
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def _inputs(L, hq, hkv, d, dtype, seed):
    q = workloads.normal((L, hq, d), seed, dtype)
    k = workloads.normal((L, hkv, d), seed + 1, dtype)
    v = workloads.normal((L, hkv, d), seed + 2, dtype)
    return q, k, v


def _run(P, q, k, v, theta, block, sink, chunk, kc, sel, star):
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    if star:
        o, lse, kr, vr, off, ws = P.star_phase1_encode(qd, kd, vd, theta, block)
    else:
        o, lse, kr, vr, off, ws = P.pulsar_phase1_encode(qd, kd, vd, theta, block, sink, chunk, kc,
                                                         torch.from_numpy(sel.astype(np.int32)).to(DEV))
    assert P.pa_workspace_status(ws) == 0
    return o, lse, kr, vr, off


def _parity(P, q, k, v, theta, block, sink, chunk, kc, sel, star, rows_fn=None):
    L = q.shape[0]
    o, lse, kr, vr, off = _run(P, q, k, v, theta, block, sink, chunk, kc, sel, star)
    pos = oracle.host_positions(L, block, sink, chunk, sel, star=star)
    assert off == oracle.host_row_offsets(pos).tolist()
    rows = None if rows_fn is None else [rows_fn(i, len(p)) for i, p in enumerate(pos)]
    ref = oracle.phase1_encode(f64(q), f64(k), f64(v), pos, theta, rows)
    tol = O_TOL[q.dtype]
    o_c, lse_c = o.cpu(), lse.cpu()
    worst = (0.0, 0.0)
    for i, (ro, rl) in enumerate(ref):
        r = np.arange(len(pos[i])) if rows is None else rows[i]
        eo = assert_close(f64(o_c[off[i] + r]), ro, tol, f"host {i} O")
        el = assert_close(lse_c[off[i] + r].double().numpy(), rl, LSE_TOL, f"host {i} lse")
        worst = (max(worst[0], eo), max(worst[1], el))
    # retained cache: V unchanged (bit-exact), K rotated at original positions
    assert torch.equal(vr.cpu(), v)
    kref, _ = oracle.retained_kv(f64(k), f64(v), theta)
    if q.dtype == torch.float32:
        assert_close(f64(kr.cpu()), kref, 1e-6, "k_ret")
    else:
        # the fp64 rotation rounded to bf16: within half a bf16 step of the
        # exact value, plus the fp32 rotation's own rounding
        tol = 2.0 ** -8 * np.abs(kref) + 1e-5 * np.linalg.norm(f64(k), axis=-1, keepdims=True)
        assert (np.abs(f64(kr.cpu()) - kref) <= tol).all()
    return worst


@pytest.mark.parametrize("star", [False, True])
def test_tiny_fp32_all_rows(P, star):
    w = workloads.TINY
    ids = w.token_ids()
    sel = oracle.select_summaries(ids, w.block, w.chunk, w.k_chunks, w.vocab)
    q, k, v = w.qkv()
    _parity(P, q, k, v, w.rope_theta, w.block, w.sink, w.chunk, w.k_chunks, sel, star)


BF16_CASES = [
    # (L, block, hq, hkv, d, sink, chunk, k, theta)
    (4 * 640, 640, 8, 2, 128, 64, 32, 3, 500000.0),     # ragged host lengths 640/800/896/992
    (3 * 384, 384, 4, 4, 64, 32, 16, 5, 10000.0),       # d = 64, MHA (g = 1: SIMT kernel), 16-token chunks
    (3 * 384, 384, 8, 2, 64, 32, 16, 5, 10000.0),       # d = 64, g = 4: tensor-core kernel
    (1024, 1024, 8, 1, 128, 64, 32, 4, 10000.0),        # N = 1: plain causal attention
]


@pytest.mark.parametrize("case", BF16_CASES)
@pytest.mark.parametrize("star", [False, True])
def test_bf16_small_all_rows(P, case, star):
    L, block, hq, hkv, d, sink, chunk, kc, theta = case
    q, k, v = _inputs(L, hq, hkv, d, torch.bfloat16, seed=L + d)
    n = L // block
    rng = np.random.default_rng(L)
    sel = np.sort(np.stack([rng.choice(block // chunk, kc, replace=False) for _ in range(n)]), axis=1)
    _parity(P, q, k, v, theta, block, sink, chunk, kc, sel, star)


def test_bf16_sixty_four_hosts_and_full_sink(P):
    # the largest host count (64 blocks of 128) with a 16-token sink, and a
    # sink as long as a block
    for L, block, sink, chunk, kc in ((64 * 128, 128, 16, 16, 1), (3 * 128, 128, 128, 16, 2)):
        q, k, v = _inputs(L, 4, 2, 64, torch.bfloat16, seed=L + sink)
        n = L // block
        rng = np.random.default_rng(n)
        sel = np.sort(np.stack([rng.choice(block // chunk, kc, replace=False) for _ in range(n)]), axis=1)
        _parity(P, q, k, v, 10000.0, block, sink, chunk, kc, sel, False)


def test_star_single_block(P):
    q, k, v = _inputs(384, 8, 2, 128, torch.bfloat16, seed=31)
    _parity(P, q, k, v, 500000.0, 384, 0, 16, 0, np.zeros((1, 0), dtype=np.int64), True)


def test_bf16_zero_sink_zero_budget(P):
    L, block = 3 * 256, 256
    q, k, v = _inputs(L, 4, 2, 128, torch.bfloat16, seed=5)
    sel = np.zeros((3, 0), dtype=np.int64)
    _parity(P, q, k, v, 10000.0, block, 0, 32, 0, sel, False)


@pytest.mark.parametrize("star", [False, True])
def test_bf16_running_max_jumps_mid_sequence(P, star):
    # Rows at positions >= 128 with p = 1 (mod 4), and rows at positions >= 256
    # with p = 3 (mod 4), score the keys before that point about 7 nat lower
    # through sixteen of the slowest-turning RoPE dimensions.  Their running
    # max therefore jumps by more than 2^8 at key tile 1 or 2, which takes the
    # lazy-rescale branch (the running max moves and O in TMEM is rescaled
    # before the next PV) for some rows of every warp while the others keep
    # their max.  The jump comes from pushing
    # early keys down, so the dominant scores stay small and the fp16 operand
    # rounding stays well inside the lse tolerance.
    L, block, theta, a = 2 * 512, 512, 500000.0, 5.0
    q, k, v = _inputs(L, 4, 2, 128, torch.bfloat16, seed=77)
    pos = np.arange(L)
    rng = np.random.default_rng(5)
    for dims, start, rem in ((np.r_[48:56, 112:120], 128, 1), (np.r_[56:64, 120:128], 256, 3)):
        idx = torch.from_numpy(dims)
        kx = (pos < start)[:, None, None] * -a * (1.0 + 0.25 * rng.standard_normal((L, 2, 16)))
        qx = ((pos % 4 == rem) & (pos >= start))[:, None, None] * (1.0 + 0.25 * rng.standard_normal((L, 4, 16)))
        k[:, :, idx] = torch.from_numpy(kx).to(torch.bfloat16)
        q[:, :, idx] = torch.from_numpy(qx).to(torch.bfloat16)
    sel = np.array([[1, 9], [3, 14]])
    _parity(P, q, k, v, theta, block, 64, 32, 2, sel, star)


@pytest.mark.parametrize("wname", ["llama3.1-8b_attn_32k", "llama3.1-8b_attn_128k"])
@pytest.mark.parametrize("star", [False, True])
def test_llama_shapes_sampled_rows(P, wname, star):
    w = workloads.WORKLOADS[wname]
    ids = w.token_ids()
    sel = oracle.select_summaries(ids, w.block, w.chunk, w.k_chunks, w.vocab)
    q, k, v = w.qkv()
    summ = w.k_chunks * w.chunk

    def rows(i, n):
        bounds = [w.sink, w.sink + summ, n - w.block] if i else []
        return sample_rows(n, bounds, count=6, seed=i)

    _parity(P, q, k, v, w.rope_theta, w.block, w.sink, w.chunk, w.k_chunks, sel, star, rows)


def test_range_status_for_values_beyond_fp16(P):
    L, block = 256, 128
    q, k, v = _inputs(L, 4, 2, 64, torch.bfloat16, seed=9)
    k[5, 1, 3] = 1.0e6
    sel = np.zeros((2, 1), dtype=np.int64)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    *_, ws = P.pulsar_phase1_encode(qd, kd, vd, 1e4, block, 0, 16, 1, torch.zeros((2, 1), dtype=torch.int32,
                                                                                   device=DEV))
    assert P.pa_workspace_status(ws) == -6   # PA_ERR_RANGE
    # Phase 1 carries rotated Q and K in fp16 for bf16 inputs and refuses
    # values beyond its range through the device status; with the binding's
    # status checks on, the call itself raises
    prev = P.set_status_checks(True)
    try:
        with pytest.raises(P.PulsarError) as e:
            P.pulsar_phase1_encode(qd, kd, vd, 1e4, block, 0, 16, 1, torch.zeros((2, 1), dtype=torch.int32,
                                                                              device=DEV))
        assert e.value.code == -6
        k[5, 1, 3] = 1.0
        P.pulsar_phase1_encode(qd, k.to(DEV), vd, 1e4, block, 0, 16, 1,
                               torch.zeros((2, 1), dtype=torch.int32, device=DEV))   # in range: no error
    finally:
        P.set_status_checks(prev)


def test_bad_summary_index_sets_status(P):
    L, block = 256, 128
    q, k, v = _inputs(L, 4, 2, 64, torch.bfloat16, seed=10)
    bad = torch.tensor([[9], [0]], dtype=torch.int32, device=DEV)   # 128/16 = 8 chunks: 9 is out of range
    *_, ws = P.pulsar_phase1_encode(q.to(DEV), k.to(DEV), v.to(DEV), 1e4, block, 16, 16, 1, bad)
    assert P.pa_workspace_status(ws) == -1


@pytest.mark.parametrize("star,dtype,splits", [
    (False, torch.bfloat16, [(0, 2), (2, 5), (5, 6), (3, 3)]),   # tensor-core kernel; an empty range
    (True, torch.bfloat16, [(0, 1), (1, 6), (4, 6)]),            # (4, 6) rotates B_0 and its blocks only
    (False, torch.float32, [(0, 4), (4, 6)]),                    # SIMT kernel
])
def test_host_ranges_equal_full_encode(P, star, dtype, splits):
    # one GPU's share of a sequence's hosts (the multi-GPU layout of the
    # Pulsar page §2.1 / §2.2): the rows and retained blocks of every range
    # are bit-identical to the same rows of the all-host call.  Ranges that
    # read few positions ((2, 5), (5, 6), (4, 6)) rotate only those, in the
    # compact row order, with a smaller workspace.
    L, block, sink, chunk, kc = 6 * 256, 256, 64, 32, 2
    hq, hkv, d = (8, 2, 128) if dtype == torch.bfloat16 else (4, 2, 64)
    q, k, v = _inputs(L, hq, hkv, d, dtype, seed=30)
    sel = np.array([[1, 5], [0, 7], [2, 3], [4, 6], [1, 2], [0, 3]], dtype=np.int32)
    o, lse, kr, vr, off = _run(P, q, k, v, 5e5, block, sink, chunk, kc, sel, star)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    seld = torch.from_numpy(sel).to(DEV)
    for h0, h1 in splits:
        if star:
            o2, lse2, kr2, vr2, off2, ws = P.star_phase1_encode_hosts(qd, kd, vd, 5e5, block, h0, h1)
        else:
            o2, lse2, kr2, vr2, off2, ws = P.pulsar_phase1_encode_hosts(qd, kd, vd, 5e5, block, sink, chunk, kc,
                                                                        seld, h0, h1)
        assert P.pa_workspace_status(ws) == 0
        assert off2 == [r - off[h0] for r in off[h0:h1 + 1]]
        rows = slice(off[h0], off[h1])
        assert torch.equal(o2, o[rows]), (h0, h1)
        assert torch.equal(lse2, lse[rows]), (h0, h1)
        assert torch.equal(kr2, kr[h0 * block:h1 * block]), (h0, h1)
        assert torch.equal(vr2, vr[h0 * block:h1 * block]), (h0, h1)
