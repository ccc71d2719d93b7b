"""Out-of-bounds write checks for every kernel path, in place of a memory
checker: each output is passed as a view into a larger buffer filled with a
sentinel bit pattern, with guard regions of 64 KiB before and after it, and
after the call every guard element must still hold the sentinel.  Outputs
that are only partly written by design (the query host's own cache beyond
the new rows) keep their sentinel there too.  Small, ragged shapes cover
every kernel: the selection kernels and scorers, Phase 1 on the tensor cores
(Pulsar, Star, a compact host range) and in fp32, the Phase-2 tensor-core
query, the mma.sync decode and row-group kernels, the fp32 kernel, the
merge, the query-host step and ART."""
import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_max_b200 import workloads

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
GUARD_BYTES = 65536
# sentinel bit patterns (NaN payloads for the float types)
SENT = {torch.bfloat16: 0x7FA5, torch.float32: 0x7FC0A5A5, torch.int32: -0x5A5A5A5B, torch.int64: -0x5A5A5A5A5A5A5A5B}
BITS = {torch.bfloat16: torch.int16, torch.float32: torch.int32, torch.int32: torch.int32, torch.int64: torch.int64}


@pytest.fixture(scope="module")
def P():
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


class Guarded:
    """A sentinel-filled buffer [guard | out | guard]; ``out`` is a
    contiguous view of ``shape`` (16-byte aligned)."""

    def __init__(self, shape, dtype):
        self.dtype = dtype
        esz = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // esz
        self.n = int(np.prod(shape)) if len(shape) else 1
        self.raw = torch.empty(self.g * 2 + self.n, dtype=BITS[dtype], device=DEV)
        self.raw.fill_(SENT[dtype])
        self.out = self.raw[self.g:self.g + self.n].view(dtype).view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.raw[:self.g]
        tail = self.raw[self.g + self.n:]
        s = SENT[self.dtype]
        bad_h = int((head != s).sum().item())
        bad_t = int((tail != s).sum().item())
        assert bad_h == 0 and bad_t == 0, f"{what}: {bad_h} guard elements before and {bad_t} after were written"

    def bits(self):
        return self.raw[self.g:self.g + self.n]


def _status_ok(P, ws):
    assert P.pa_workspace_status(ws) == 0


def test_selection_kernels(P):
    # 5 blocks of 480 ids (15 chunks of 32), vocabulary of 700 (not a multiple of 32)
    L, vocab, block, chunk, k = 5 * 480, 700, 480, 32, 3
    ids = torch.from_numpy(workloads.zipf_token_ids(L, vocab, 1.0, seed=3)).to(DEV)
    sel, df, mdf = Guarded((5, k), torch.int32), Guarded((vocab,), torch.int32), Guarded((L // chunk,), torch.int32)
    _, _, _, ws = P.pulsar_select_summaries(ids, vocab, block, chunk, k, sel=sel.out, df=df.out,
                                            chunk_mindf=mdf.out)
    _status_ok(P, ws)
    for g, name in ((sel, "sel"), (df, "df"), (mdf, "chunk_mindf")):
        g.check(name)
    assert np.array_equal(sel.out.cpu().numpy(), oracle.select_summaries(ids.cpu().numpy(), block, chunk, k, vocab))
    for method in (P.PA_SCORE_MEAN_IDF, P.PA_SCORE_MAX_IDF, P.PA_SCORE_EVENLY_SPACED):
        sel2 = Guarded((5, k), torch.int32)
        _, _, ws = P.pulsar_select_summaries_scored(ids, vocab, block, chunk, k, method, sel=sel2.out)
        _status_ok(P, ws)
        sel2.check(f"scored sel, method {method}")
    sel3, df3, mdf3 = Guarded((5, k), torch.int32), Guarded((vocab,), torch.int32), Guarded((L // chunk,), torch.int32)
    P.pulsar_select_summaries_noalloc(ids, vocab, block, chunk, k, sel3.out, df3.out, mdf3.out)
    for g, name in ((sel3, "noalloc sel"), (df3, "noalloc df"), (mdf3, "noalloc chunk_mindf")):
        g.check(name)


def test_scored_rank_output(P):
    # the int64 chunk-score output of the scored entry point (ranks / min df)
    L, vocab, block, chunk, k = 3 * 352, 90, 352, 32, 2      # 11 chunks per block
    ids = torch.from_numpy(workloads.zipf_token_ids(L, vocab, 0.8, seed=4)).to(DEV)
    for method in (P.PA_SCORE_MEAN_IDF, P.PA_SCORE_MAX_IDF):
        sel, sc = Guarded((3, k), torch.int32), Guarded((L // chunk,), torch.int64)
        ws = torch.empty(P.pa_select_workspace_size(L, vocab, block, chunk), dtype=torch.uint8, device=DEV)
        rc = P._lib.pulsar_select_summaries_scored(P._ptr(ids), L, vocab, block, chunk, k, method, P._ptr(sel.out),
                                                   P._ptr(sc.out), P._ptr(ws), ws.numel(), P._stream())
        assert rc == 0
        _status_ok(P, ws)
        sel.check("scored sel")
        sc.check("chunk scores")


@pytest.mark.parametrize("star,dtype,hosts", [
    (False, torch.bfloat16, None),      # tensor-core kernel, ragged host lengths
    (True, torch.bfloat16, None),
    (False, torch.float32, None),       # SIMT kernel
    (False, torch.bfloat16, (3, 4)),    # compact host range
    (True, torch.bfloat16, (2, 4)),
])
def test_phase1(P, star, dtype, hosts):
    L, block, sink, chunk, kc = 4 * 640, 640, 64, 32, 3
    hq, hkv, d = (8, 2, 128) if dtype == torch.bfloat16 else (4, 2, 64)
    q = workloads.normal((L, hq, d), 40, dtype).to(DEV)
    k = workloads.normal((L, hkv, d), 41, dtype).to(DEV)
    v = workloads.normal((L, hkv, d), 42, dtype).to(DEV)
    sel = torch.tensor([[0, 5, 19], [2, 3, 4], [1, 7, 11], [6, 8, 9]], dtype=torch.int32, device=DEV)
    full = P.pa_phase1_layout(L, block, 0 if star else sink, 0 if star else kc * chunk, star)
    h0, h1 = hosts or (0, L // block)
    R = full[h1] - full[h0]
    o, lse = Guarded((R, hq, d), dtype), Guarded((R, hq), torch.float32)
    kr, vr = Guarded(((h1 - h0) * block, hkv, d), dtype), Guarded(((h1 - h0) * block, hkv, d), dtype)
    kw = dict(o=o.out, lse=lse.out, k_ret=kr.out, v_ret=vr.out)
    if hosts is None and star:
        *_, ws = P.star_phase1_encode(q, k, v, 5e5, block, **kw)
    elif hosts is None:
        *_, ws = P.pulsar_phase1_encode(q, k, v, 5e5, block, sink, chunk, kc, sel, **kw)
    elif star:
        *_, ws = P.star_phase1_encode_hosts(q, k, v, 5e5, block, h0, h1, **kw)
    else:
        *_, ws = P.pulsar_phase1_encode_hosts(q, k, v, 5e5, block, sink, chunk, kc, sel, h0, h1, **kw)
    _status_ok(P, ws)
    for g, name in ((o, "o"), (lse, "lse"), (kr, "k_ret"), (vr, "v_ret")):
        g.check(name)
        assert not torch.isnan(g.out.float()).any(), f"{name}: an element was not written"


@pytest.mark.parametrize("case", [
    # (B, Tq, T, S, hq, hkv, d, dtype)
    (1, 64, 1000, 3, 8, 2, 128, torch.bfloat16),   # tensor-core query kernel, ragged shards
    (1, 48, 777, 4, 16, 2, 128, torch.bfloat16),   # g = 8: a half-empty tile pair
    (3, 1, 999, 4, 32, 8, 128, torch.bfloat16),    # mma.sync decode
    (1, 30, 500, 2, 6, 2, 64, torch.bfloat16),     # row-group kernel (g = 3)
    (2, 5, 300, 3, 4, 2, 64, torch.float32),       # fp32 kernel
    (2, 7, 10, 16, 4, 4, 64, torch.bfloat16),      # empty shards
])
def test_phase2_and_merge(P, case):
    B, Tq, T, S, hq, hkv, d, dtype = case
    q = workloads.normal((B, Tq, hq, d), 43, dtype).to(DEV)
    kc = workloads.normal((B, T, hkv, d), 44, dtype).to(DEV)
    vc = workloads.normal((B, T, hkv, d), 45, dtype).to(DEV)
    o, lse = Guarded((B, Tq, hq, d), dtype), Guarded((B, Tq, hq), torch.float32)
    po, pl = Guarded((B, S, Tq, hq, d), torch.float32), Guarded((B, S, Tq, hq), torch.float32)
    *_, ws = P.star_phase2_attend(q, kc, vc, S, q_pos0=T, rope_theta=5e5, o=o.out, lse=lse.out,
                                  want_partials=True, part_o=po.out, part_lse=pl.out)
    _status_ok(P, ws)
    for g, name in ((o, "o"), (lse, "lse"), (po, "part_o"), (pl, "part_lse")):
        g.check(name)
    o2, lse2 = Guarded((B, Tq, hq, d), dtype), Guarded((B, Tq, hq), torch.float32)
    P.pa_lse_merge(po.out, pl.out, dtype=dtype, o=o2.out, lse=lse2.out)
    o2.check("merge o")
    lse2.check("merge lse")


def test_query_step_writes_only_its_rows(P):
    B, Tq, T, S, hq, hkv, d, cap, self_len = 2, 3, 600, 3, 8, 2, 128, 16, 5
    dt = torch.bfloat16
    q = workloads.normal((B, Tq, hq, d), 46, dt).to(DEV)
    kn = workloads.normal((B, Tq, hkv, d), 47, dt).to(DEV)
    vn = workloads.normal((B, Tq, hkv, d), 48, dt).to(DEV)
    kc = workloads.normal((B, T, hkv, d), 49, dt).to(DEV)
    vc = workloads.normal((B, T, hkv, d), 50, dt).to(DEV)
    ks, vs = Guarded((B, cap, hkv, d), dt), Guarded((B, cap, hkv, d), dt)
    # rows already in the own cache hold data; rows past the new ones keep the sentinel
    ks.out[:, :self_len] = workloads.normal((B, self_len, hkv, d), 51, dt).to(DEV)
    vs.out[:, :self_len] = workloads.normal((B, self_len, hkv, d), 52, dt).to(DEV)
    o, lse = Guarded((B, Tq, hq, d), dt), Guarded((B, Tq, hq), torch.float32)
    *_, ws = P.star_phase2_query_step(q, kn, vn, kc, vc, S, ks.out, vs.out, self_len, T + self_len, 5e5,
                                      o=o.out, lse=lse.out)
    _status_ok(P, ws)
    for g, name in ((ks, "k_self"), (vs, "v_self"), (o, "o"), (lse, "lse")):
        g.check(name)
    for g, name in ((ks, "k_self"), (vs, "v_self")):
        rows = g.bits().view(B, cap, hkv, d)[:, self_len + Tq:]
        assert (rows == SENT[dt]).all(), f"{name}: rows past self_len + Tq were written"


def test_art(P):
    B, Tq, T, hq, hkv, d = 2, 1, 1000, 32, 8, 128
    dt = torch.bfloat16
    q = workloads.normal((B, Tq, hq, d), 53, dt).to(DEV)
    kc = workloads.normal((B, T, hkv, d), 54, dt).to(DEV)
    vc = workloads.normal((B, T, hkv, d), 55, dt).to(DEV)
    o, lse, vis = Guarded((B, Tq, hq, d), dt), Guarded((B, Tq, hq), torch.float32), Guarded((B, hkv), torch.int32)
    ws = torch.empty(P.pa_phase2_workspace_size(B, Tq, T, 1, hq, hkv, d), dtype=torch.uint8, device=DEV)
    rc = P._lib.star_phase2_attend_art(P._ptr(q), 1, B, Tq, T, 5e5, P._ptr(kc), P._ptr(vc), T, hq, hkv, d, 128,
                                       1e-5, 1e-3, 5, P._ptr(o.out), P._ptr(lse.out), P._ptr(vis.out), P._ptr(ws),
                                       ws.numel(), P._stream())
    assert rc == 0
    _status_ok(P, ws)
    for g, name in ((o, "o"), (lse, "lse"), (vis, "visited")):
        g.check(name)
