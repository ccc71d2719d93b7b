"""Host-side checks of the C ABI (no GPU needed): the shared library loads,
exports every function include/pulsar.h declares, and rejects invalid
arguments on the host before any launch."""
import ctypes
import os
import re

import numpy as np
import torch
import pytest

import oracle
from long_context_blockwise_max_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    from long_context_blockwise_max_b200 import pulsar
    return pulsar


def _header_functions():
    src = open(os.path.join(ROOT, "include", "pulsar.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol(lib):
    names = _header_functions()
    assert len(names) == 20
    assert sorted(lib.ABI_SYMBOLS) == names
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(so, n), n
    assert lib.pa_abi_version() == 1
    assert lib.status_string(-3).startswith("workspace")


def test_phase1_layout_matches_oracle(lib):
    L, b, sink, chunk, k = 8 * 16384, 16384, 64, 32, 64
    sel = np.zeros((8, k), dtype=np.int64)
    for star in (False, True):
        want = oracle.host_row_offsets(oracle.host_positions(L, b, sink, chunk, sel, star=star))
        got = lib.pa_phase1_layout(L, b, sink, k * chunk, star)
        assert got == want.tolist()


def test_workspace_sizes(lib):
    assert lib.pa_select_workspace_size(2048, 1000, 512, 32) >= 256 + 8 * 1000
    assert lib.pa_select_workspace_size(2047, 1000, 512, 32) == 0
    assert lib.pa_phase1_workspace_size(2048, 4, 2, 64, 0, 512, 64, 64, False) > 0
    assert lib.pa_phase1_workspace_size(2048, 4, 2, 96, 0, 512, 64, 64, False) == 0
    assert lib.pa_phase2_workspace_size(16, 1, 131072, 8, 32, 8, 128) > 0
    assert lib.pa_phase2_workspace_size(16, 1, 131072, 0, 32, 8, 128) == 0


def _align(x):
    return -(-x // 256) * 256


def test_host_range_workspace_scales_with_the_positions_it_reads(lib):
    # 128K Llama-3.1-8B shape, bf16: one GPU per host.  A range rotates the
    # positions its hosts read -- the sink, the summaries of the blocks before
    # its last host, its own blocks (Star: B_0 and its own blocks) -- not the
    # whole prefix of the sequence.
    L, b, sink, summ, hq, hkv, d = 131072, 16384, 64, 2048, 32, 8, 128
    row = 2 * (hq + hkv) * d                      # fp16 Qr + Kr bytes per rotated row
    full = lib.pa_phase1_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False)
    for h in range(8):
        rows = b if h == 0 else sink + h * summ + b
        want_rows = b if h == 0 else sink + h * summ + b     # host 0 reads B_0 only
        got = lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False, h, h + 1)
        posmap = 0 if h == 0 else _align(4 * want_rows)
        want = 256 + 2 * _align(4 * rows) + posmap + _align(2 * want_rows * hq * d) + _align(2 * want_rows * hkv * d)
        assert got == want, (h, got, want)
        assert got <= full
    last = lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False, 7, 8)
    assert last * 4 < full and 30784 * row < last
    # all hosts: every position once, by position
    assert lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False, 0, 8) <= full
    # Star, the last host: [B_0 || B_7]
    star_last = lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, 0, 0, True, 7, 8)
    assert star_last == 256 + 2 * _align(4 * 2 * b) + _align(4 * 2 * b) + _align(2 * 2 * b * hq * d) + \
        _align(2 * 2 * b * hkv * d)
    assert lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False, 5, 9) == 0
    assert lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, 1, b, sink, summ, False, 3, 2) == 0


def test_host_validation_rejects_before_launch(lib):
    so = lib._lib
    ws = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    dummy = ctypes.c_void_p(4096)
    # L not a multiple of the block
    assert so.pulsar_select_summaries(dummy, 1000, 100, 512, 32, 2, dummy, None, None, ws, 1 << 20, None) == -1
    # k larger than the chunk count
    assert so.pulsar_select_summaries(dummy, 1024, 100, 512, 32, 17, dummy, None, None, ws, 1 << 20, None) == -1
    # more than 64 blocks
    assert so.pulsar_select_summaries(dummy, 65 * 16, 100, 16, 16, 1, dummy, None, None, ws, 1 << 20, None) == -2
    # workspace too small
    assert so.pulsar_select_summaries(dummy, 1024, 100, 512, 32, 2, dummy, None, None, ws, 16, None) == -3
    # head_dim 96 unsupported; hq not a multiple of hkv invalid
    args = (dummy, dummy, dummy, 0, 2048, 4, 2, 96, 10000.0, 512, 64, 32, 2, dummy, dummy, None, dummy, dummy,
            ws, 1 << 30, None)
    assert so.pulsar_phase1_encode(*args) == -2
    args = (dummy, dummy, dummy, 0, 2048, 3, 2, 64, 10000.0, 512, 64, 32, 2, dummy, dummy, None, dummy, dummy,
            ws, 1 << 30, None)
    assert so.pulsar_phase1_encode(*args) == -1
    # sink not a multiple of 16
    args = (dummy, dummy, dummy, 0, 2048, 4, 2, 64, 10000.0, 512, 40, 32, 2, dummy, dummy, None, dummy, dummy,
            ws, 1 << 30, None)
    assert so.pulsar_phase1_encode(*args) == -2
    # misaligned output pointer
    args = (dummy, dummy, dummy, 0, 2048, 4, 2, 64, 10000.0, 512, dummy, None, ctypes.c_void_p(4098), dummy,
            ws, 1 << 30, None)
    assert so.star_phase1_encode(*args) == -2
    # host ranges: begin after end, end past the last host (4 hosts of 512), negative end
    for hb, he in ((3, 2), (0, 5), (0, -1)):
        args = (dummy, dummy, dummy, 0, 2048, 4, 2, 64, 10000.0, 512, 64, 32, 2, dummy, hb, he, dummy, None,
                dummy, dummy, ws, 1 << 30, None)
        assert so.pulsar_phase1_encode_hosts(*args) == -1, (hb, he)
        args = (dummy, dummy, dummy, 0, 2048, 4, 2, 64, 10000.0, 512, hb, he, dummy, None, dummy, dummy, ws,
                1 << 30, None)
        assert so.star_phase1_encode_hosts(*args) == -1, (hb, he)
    # phase 2: zero shards
    assert so.star_phase2_attend(dummy, 1, 1, 1, 0, 0.0, dummy, dummy, 100, 0, 32, 8, 128, dummy, dummy, None,
                                 None, ws, 1 << 30, None) == -1


def test_host_validation_of_the_other_entry_points(lib):
    # argument checks of the scorer, ART, merge and query-step entry points
    # and the status text, all decided on the host before any launch
    so = lib._lib
    ws = ctypes.c_void_p(256)
    dummy = ctypes.c_void_p(4096)
    texts = {c: so.pa_status_string(c).decode() for c in range(-6, 1)}
    assert len(set(texts.values())) == 7 and all(texts.values())
    assert so.pa_status_string(-99).decode() == "unknown status"
    assert so.pa_abi_version() >= 1
    assert so.pa_set_profile_events(dummy, None) == -1
    assert so.pa_set_profile_events(None, dummy) == -1
    assert so.pa_set_profile_events(None, None) == 0
    # scorer: unknown method; missing ids for a scorer that reads them; mean-IDF beyond 4096 chunks per
    # block or beyond 32 tokens per chunk (the exact 256-bit product)
    assert so.pulsar_select_summaries_scored(dummy, 1024, 100, 512, 32, 2, 5, dummy, None, ws, 1 << 20,
                                             None) == -1
    assert so.pulsar_select_summaries_scored(None, 1024, 100, 512, 32, 2, 1, dummy, None, ws, 1 << 20,
                                             None) == -1
    assert so.pulsar_select_summaries_scored(dummy, 8192, 100, 8192, 1, 1, 1, dummy, None, ws, 1 << 30,
                                             None) == -2
    assert so.pulsar_select_summaries_scored(dummy, 4096, 100, 1024, 64, 1, 1, dummy, None, ws, 1 << 30,
                                             None) == -2
    for method in (3, 4):   # entropy and BM25: the same limits as mean IDF
        assert so.pulsar_select_summaries_scored(dummy, 4096, 100, 1024, 64, 1, method, dummy, None, ws, 1 << 30,
                                                 None) == -2

    def art(dtype=1, Tq=1, hq=32, hkv=8, block_keys=128, tau=1e-5, phi=1e-3, patience=5, theta=5e5):
        return so.star_phase2_attend_art(dummy, dtype, 2, Tq, 1000, theta, dummy, dummy, 1000, hq, hkv, 128,
                                         block_keys, tau, phi, patience, dummy, dummy, None, ws, 1 << 30, None)
    assert art(dtype=0) == -2                      # bf16 only
    assert art(block_keys=48) == -1                # a multiple of 32
    assert art(block_keys=0) == -1
    assert art(patience=0) == -1
    assert art(tau=float("nan")) == -1
    assert art(phi=-1.0) == -1
    assert art(theta=float("inf")) == -1
    assert art(Tq=3) == -2                         # 3 tokens x 4 heads = 12 decode rows > 8

    def merge(S=4, d=128, dtype=1, part_o=dummy):
        return so.pa_lse_merge(part_o, dummy, 1, S, 2, 8, d, dtype, dummy, dummy, None)
    assert merge(S=0) == -1
    assert merge(d=96) == -2
    assert merge(dtype=5) == -2
    assert merge(part_o=ctypes.c_void_p(4100)) == -1   # partials must be 16-byte aligned

    def step(n_shards=8, self_cap=64, self_len=0, Tq=4, theta=5e5):
        return so.star_phase2_query_step(dummy, dummy, dummy, 1, 1, Tq, 1000, theta, dummy, dummy, 1000,
                                         n_shards, dummy, dummy, self_cap, self_len, 32, 8, 128, dummy, dummy,
                                         ws, 1 << 30, None)
    assert step(n_shards=0) == -1
    assert step(n_shards=4097) == -1
    assert step(self_len=62) == -1                 # 62 + 4 new tokens > capacity 64
    assert step(self_len=-1) == -1
    assert step(theta=float("nan")) == -1


def test_binding_refuses_mismatched_tensors_before_the_library(lib, monkeypatch):
    # the binding hands raw pointers to the library, so it checks dtypes and
    # sizes first; these calls must all stop there (CPU tensors, with the
    # CUDA-residency check stubbed out, never reach a launch)
    P = lib
    monkeypatch.setattr(P, "_dev", lambda *ts: None)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    L, hq, hkv, d, block = 1024, 8, 2, 64, 256
    q = torch.zeros((L, hq, d), dtype=bf)
    k = torch.zeros((L, hkv, d), dtype=bf)
    sel = torch.zeros((4, 2), dtype=i32)
    with pytest.raises(ValueError, match="ids"):
        P.pulsar_select_summaries(torch.zeros(L, dtype=torch.int64), 100, block, 32, 2)
    with pytest.raises(ValueError, match="sel"):
        P.pulsar_select_summaries(torch.zeros(L, dtype=i32), 100, block, 32, 2, sel=torch.zeros((4, 1), dtype=i32))
    with pytest.raises(ValueError, match="df"):
        P.pulsar_select_summaries_noalloc(torch.zeros(L, dtype=i32), 100, block, 32, 2, sel,
                                          df=torch.zeros(99, dtype=i32))
    with pytest.raises(ValueError, match="k:"):
        P.pulsar_phase1_encode(q, k.float(), k, 1e4, block, 64, 32, 2, sel)
    with pytest.raises(ValueError, match="v:"):
        P.pulsar_phase1_encode(q, k, torch.zeros((L, hkv, d + 64), dtype=bf), 1e4, block, 64, 32, 2, sel)
    with pytest.raises(ValueError, match="sel"):
        P.pulsar_phase1_encode(q, k, k, 1e4, block, 64, 32, 2, sel.long())
    with pytest.raises(ValueError, match="o:"):
        P.star_phase1_encode(q, k, k, 1e4, block, o=torch.zeros((10, hq, d), dtype=bf))
    with pytest.raises(ValueError, match="lse"):
        P.star_phase1_encode(q, k, k, 1e4, block, lse=torch.zeros((L, hq), dtype=bf))
    with pytest.raises(ValueError, match="k_ret"):
        P.star_phase1_encode_hosts(q, k, k, 1e4, block, 0, 2, k_ret=torch.zeros((block, hkv, d), dtype=bf))
    qq = torch.zeros((2, 3, hq, d), dtype=bf)
    kc = torch.zeros((2, 500, hkv, d), dtype=bf)
    with pytest.raises(ValueError, match="k_ret"):
        P.star_phase2_attend(qq, kc.float(), kc.float(), 4)
    with pytest.raises(ValueError, match="v_ret"):
        P.star_phase2_attend(qq, kc, kc[:, :400].contiguous(), 4)
    with pytest.raises(ValueError, match="part_o"):
        P.star_phase2_attend(qq, kc, kc, 4, want_partials=True, part_o=torch.zeros((2, 3, 3, hq, d), dtype=f32))
    with pytest.raises(ValueError, match="o:"):
        P.star_phase2_attend_art(qq, kc, kc, o=torch.zeros_like(qq, dtype=f32))
    with pytest.raises(ValueError, match="part_lse"):
        P.pa_lse_merge(torch.zeros((2, 4, 3, hq, d)), torch.zeros((2, 4, 3, hq), dtype=bf))
    ks = torch.zeros((2, 16, hkv, d), dtype=bf)
    kn = torch.zeros((2, 3, hkv, d), dtype=bf)
    with pytest.raises(ValueError, match="v_new"):
        P.star_phase2_query_step(qq, kn, kn[:, :2].contiguous(), kc, kc, 4, ks, ks, 0, 500, 5e5)
    with pytest.raises(ValueError, match="k_self"):
        P.star_phase2_query_step(qq, kn, kn, kc, kc, 4, torch.zeros((2, 16, 1, d), dtype=bf),
                                 torch.zeros((2, 16, 1, d), dtype=bf), 0, 500, 5e5)
