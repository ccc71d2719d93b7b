"""Python binding of ``libpulsar_b200.so`` (C ABI in ``include/pulsar.h``).

Argument marshalling only: every function checks shapes, dtypes and devices
of torch tensors, allocates missing outputs and workspaces with torch (the
library itself never allocates), and passes raw device pointers and the
current CUDA stream to the C entry point of the same name.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpulsar_b200.so")

PA_F32, PA_BF16 = 0, 1
PA_SCORE_MAX_IDF, PA_SCORE_MEAN_IDF, PA_SCORE_EVENLY_SPACED, PA_SCORE_ENTROPY, PA_SCORE_BM25 = 0, 1, 2, 3, 4
_STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_WORKSPACE",
           -4: "PA_ERR_CUDA", -5: "PA_ERR_TIMEOUT", -6: "PA_ERR_RANGE"}

# Every symbol declared in include/pulsar.h.
ABI_SYMBOLS = (
    "pa_abi_version", "pa_status_string", "pa_workspace_status", "pa_set_profile_events",
    "pa_select_workspace_size", "pulsar_select_summaries", "pulsar_select_summaries_noalloc",
    "pulsar_select_summaries_scored",
    "pa_phase1_layout", "pa_phase1_workspace_size", "pa_phase1_hosts_workspace_size",
    "pulsar_phase1_encode", "star_phase1_encode",
    "pulsar_phase1_encode_hosts", "star_phase1_encode_hosts",
    "pa_phase2_workspace_size", "star_phase2_attend", "star_phase2_query_step", "pa_lse_merge",
    "star_phase2_attend_art",
)


class PulsarError(RuntimeError):
    """A library call returned a negative pa_status."""

    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS.get(code, code)} ({status_string(code)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_blockwise_max_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_double
    sig = {
        "pa_abi_version": (ctypes.c_int, []),
        "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "pa_workspace_status": (ctypes.c_int, [P, P]),
        "pa_set_profile_events": (ctypes.c_int, [P, P]),
        "pa_select_workspace_size": (SZ, [I64, I32, I32, I32]),
        "pulsar_select_summaries": (ctypes.c_int, [P, I64, I32, I32, I32, I32, P, P, P, P, SZ, P]),
        "pulsar_select_summaries_noalloc": (ctypes.c_int, [P, I64, I32, I32, I32, I32, P, P, P, P]),
        "pulsar_select_summaries_scored": (ctypes.c_int, [P, I64, I32, I32, I32, I32, ctypes.c_int, P, P, P, SZ,
                                                          P]),
        "pa_phase1_layout": (ctypes.c_int, [I64, I32, I32, I32, ctypes.c_int, P]),
        "pa_phase1_workspace_size": (SZ, [I64, I32, I32, I32, ctypes.c_int, I32, I32, I32, ctypes.c_int]),
        "pa_phase1_hosts_workspace_size": (SZ, [I64, I32, I32, I32, ctypes.c_int, I32, I32, I32, ctypes.c_int,
                                                I32, I32]),
        "pulsar_phase1_encode": (ctypes.c_int, [P, P, P, ctypes.c_int, I64, I32, I32, I32, D, I32, I32, I32,
                                                I32, P, P, P, P, P, P, SZ, P]),
        "star_phase1_encode": (ctypes.c_int, [P, P, P, ctypes.c_int, I64, I32, I32, I32, D, I32, P, P, P, P,
                                              P, SZ, P]),
        "pulsar_phase1_encode_hosts": (ctypes.c_int, [P, P, P, ctypes.c_int, I64, I32, I32, I32, D, I32, I32,
                                                      I32, I32, P, I32, I32, P, P, P, P, P, SZ, P]),
        "star_phase1_encode_hosts": (ctypes.c_int, [P, P, P, ctypes.c_int, I64, I32, I32, I32, D, I32, I32, I32,
                                                    P, P, P, P, P, SZ, P]),
        "pa_phase2_workspace_size": (SZ, [I32, I32, I64, I32, I32, I32, I32]),
        "star_phase2_attend": (ctypes.c_int, [P, ctypes.c_int, I32, I32, I64, D, P, P, I64, I32, I32, I32,
                                              I32, P, P, P, P, P, SZ, P]),
        "star_phase2_attend_art": (ctypes.c_int, [P, ctypes.c_int, I32, I32, I64, D, P, P, I64, I32, I32, I32, I32,
                                                  D, D, I32, P, P, P, P, SZ, P]),
        "pa_lse_merge": (ctypes.c_int, [P, P, I32, I32, I32, I32, I32, ctypes.c_int, P, P, P]),
        "star_phase2_query_step": (ctypes.c_int, [P, P, P, ctypes.c_int, I32, I32, I64, D, P, P, I64, I32, P, P,
                                                  I64, I64, I32, I32, I32, P, P, P, SZ, P]),
    }
    # test hook (include/pulsar_testing.h)
    sig["pa_testing_phase1_stall"] = (ctypes.c_int, [P, P, P, I64, I32, I32, I32, I32, P, P, P, P, SZ, I32, P])
    sig["pa_testing_phase2_stall"] = (ctypes.c_int, [P, P, P, I32, I32, I64, I32, I32, I32, I32, P, P, P, SZ, I32,
                                                     P])
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc: int, where: str, ws=None):
    """Raise PulsarError for a negative return code; with device-status
    checks on (set_status_checks), also wait for the call and raise for a
    non-zero status its kernels recorded in the workspace ``ws``."""
    if rc != 0:
        raise PulsarError(rc, where)
    if _STATUS_CHECKS and ws is not None:
        code = _lib.pa_workspace_status(_ptr(ws), _stream())
        if code != 0:
            raise PulsarError(code, where + " (device status)")


# Device-status checks after every call (off by default: reading the status
# waits for the stream).  Device-detected errors -- an id or summary index
# out of range, a Phase-1 value beyond the fp16 range used for bf16 inputs,
# an expired bounded wait -- otherwise only land in the workspace's status
# block (pa_workspace_status).
_STATUS_CHECKS = os.environ.get("PULSAR_CHECK_STATUS", "0") not in ("", "0")


def set_status_checks(enabled: bool) -> bool:
    """Turn the device-status check after every call on or off; returns the
    previous setting."""
    global _STATUS_CHECKS
    prev = _STATUS_CHECKS
    _STATUS_CHECKS = bool(enabled)
    return prev


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise PulsarError(-2, f"dtype {t.dtype}")


def _dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _need(t, name: str, dtype, numel: int):
    """A caller-supplied tensor (None: skipped) must have ``dtype`` and at
    least ``numel`` elements: the library reads or writes that many through
    the raw pointer, so a smaller or differently typed buffer is refused
    here rather than overrun on the device."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {numel} needed")


def _same(ref, *named):
    """Tensors that must match ``ref`` in dtype and shape (K and V of one cache)."""
    for name, t in named:
        if t is not None and (t.dtype != ref.dtype or t.shape != ref.shape):
            raise ValueError(f"{name}: {t.dtype} {tuple(t.shape)}, expected {ref.dtype} {tuple(ref.shape)}")


def _workspace(nbytes: int, device, ws=None):
    if ws is not None:
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def pa_abi_version() -> int:
    return _lib.pa_abi_version()


def status_string(code: int) -> str:
    return _lib.pa_status_string(code).decode()


def pa_workspace_status(ws: torch.Tensor) -> int:
    """Device status recorded in ``ws`` by the last call that used it (synchronises)."""
    return _lib.pa_workspace_status(_ptr(ws), _stream())


def pa_set_profile_events(start=None, stop=None) -> None:
    """Record torch.cuda.Event pair around the dominant kernel of later calls
    (None, None: off)."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)
    _check(_lib.pa_set_profile_events(h(start), h(stop)), "pa_set_profile_events")


def pa_select_workspace_size(L, vocab, block, chunk) -> int:
    return _lib.pa_select_workspace_size(L, vocab, block, chunk)


def pulsar_select_summaries(ids: torch.Tensor, vocab: int, block: int, chunk: int, k_chunks: int,
                            sel=None, df=None, chunk_mindf=None, ws=None, want_df=False,
                            want_mindf=False):
    """Max-IDF summary selection. Returns (sel [N][k] int32, df or None, mindf or None, ws)."""
    _dev(ids, sel, df, chunk_mindf)
    L = ids.numel()
    n = L // block if block > 0 else 0
    _need(ids, "ids", torch.int32, L)
    _need(sel, "sel", torch.int32, n * k_chunks)
    _need(df, "df", torch.int32, vocab)
    _need(chunk_mindf, "chunk_mindf", torch.int32, L // chunk if chunk > 0 else 0)
    dev = ids.device
    if sel is None:
        sel = torch.empty((n, k_chunks), dtype=torch.int32, device=dev)
    if want_df and df is None:
        df = torch.empty(vocab, dtype=torch.int32, device=dev)
    if want_mindf and chunk_mindf is None:
        chunk_mindf = torch.empty(L // chunk if chunk > 0 else 0, dtype=torch.int32, device=dev)
    need = pa_select_workspace_size(L, vocab, block, chunk)
    ws = _workspace(need, dev, ws)
    rc = _lib.pulsar_select_summaries(_ptr(ids), L, vocab, block, chunk, k_chunks, _ptr(sel),
                                      _ptr(df), _ptr(chunk_mindf), _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(rc, "pulsar_select_summaries", ws)
    return sel, df, chunk_mindf, ws


def pulsar_select_summaries_noalloc(ids: torch.Tensor, vocab: int, block: int, chunk: int, k_chunks: int,
                                    sel: torch.Tensor, df=None, chunk_mindf=None):
    """Selection with no workspace, for callers that cannot allocate device
    memory: writes into the caller's preallocated ``sel`` (and optional
    ``df`` / ``chunk_mindf``) and allocates nothing.  Returns ``sel``."""
    _dev(ids, sel, df, chunk_mindf)
    L = ids.numel()
    _need(ids, "ids", torch.int32, L)
    _need(sel, "sel", torch.int32, (L // block if block > 0 else 0) * k_chunks)
    _need(df, "df", torch.int32, vocab)
    _need(chunk_mindf, "chunk_mindf", torch.int32, L // chunk if chunk > 0 else 0)
    rc = _lib.pulsar_select_summaries_noalloc(_ptr(ids), ids.numel(), vocab, block, chunk, k_chunks, _ptr(sel),
                                              _ptr(df), _ptr(chunk_mindf), _stream())
    _check(rc, "pulsar_select_summaries_noalloc")
    return sel


def pulsar_select_summaries_scored(ids, vocab: int, block: int, chunk: int, k_chunks: int, method: int,
                                   L: int | None = None, sel=None, want_scores=False, ws=None):
    """Selection with another chunk scorer (PA_SCORE_*).  ``ids`` may be None
    for PA_SCORE_EVENLY_SPACED (then pass ``L``).  Returns (sel, scores or
    None, ws); with ``want_scores`` the int64 scores are each chunk's rank in
    its block (mean IDF, entropy, BM25) or its min df (max IDF)."""
    _dev(ids, sel)
    L = ids.numel() if ids is not None else int(L)
    dev = ids.device if ids is not None else torch.device("cuda", torch.cuda.current_device())
    n = L // block if block > 0 else 0
    _need(ids, "ids", torch.int32, L)
    _need(sel, "sel", torch.int32, n * k_chunks)
    if sel is None:
        sel = torch.empty((n, k_chunks), dtype=torch.int32, device=dev)
    scores = torch.empty(L // chunk if chunk > 0 else 0, dtype=torch.int64, device=dev) if want_scores else None
    ws = _workspace(pa_select_workspace_size(L, vocab, block, chunk), dev, ws)
    rc = _lib.pulsar_select_summaries_scored(_ptr(ids), L, vocab, block, chunk, k_chunks, int(method), _ptr(sel),
                                             _ptr(scores), _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(rc, "pulsar_select_summaries_scored", ws)
    return sel, scores, ws


def pa_phase1_layout(L, block, sink, summary_tokens, star) -> list[int]:
    n = L // block if block > 0 else 0
    buf = (ctypes.c_int64 * (max(n, 0) + 1))()
    _check(_lib.pa_phase1_layout(L, block, sink, summary_tokens, int(star), ctypes.cast(buf, ctypes.c_void_p)),
           "pa_phase1_layout")
    return list(buf)


def pa_phase1_workspace_size(L, hq, hkv, d, dtype, block, sink, summary_tokens, star) -> int:
    return _lib.pa_phase1_workspace_size(L, hq, hkv, d, dtype, block, sink, summary_tokens, int(star))


def pa_phase1_hosts_workspace_size(L, hq, hkv, d, dtype, block, sink, summary_tokens, star, host_begin,
                                   host_end) -> int:
    return _lib.pa_phase1_hosts_workspace_size(L, hq, hkv, d, dtype, block, sink, summary_tokens, int(star),
                                               host_begin, host_end)


def _phase1_check(q, k, v, rows, ret_rows, o, lse, k_ret, v_ret, sel=None, n_sel=0):
    """Inputs [L][h][d] of one dtype (K and V alike); caller-supplied outputs
    large enough for ``rows`` output rows and ``ret_rows`` retained rows."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q, k, v must be [L][heads][d]")
    L, hq, d = q.shape
    hkv = k.shape[1]
    if k.shape[0] != L or k.shape[2] != d or k.dtype != q.dtype:
        raise ValueError(f"k: {k.dtype} {tuple(k.shape)} does not match q {q.dtype} {tuple(q.shape)}")
    _same(k, ("v", v))
    _need(sel, "sel", torch.int32, n_sel)
    _need(o, "o", q.dtype, rows * hq * d)
    _need(lse, "lse", torch.float32, rows * hq)
    _need(k_ret, "k_ret", q.dtype, ret_rows * hkv * d)
    _need(v_ret, "v_ret", q.dtype, ret_rows * hkv * d)


def _phase1_outputs(q, k, rows, o, lse, k_ret, v_ret, want_lse):
    L, hq, d = q.shape
    hkv = k.shape[1]
    if o is None:
        o = torch.empty((rows, hq, d), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((rows, hq), dtype=torch.float32, device=q.device)
    if k_ret is None:
        k_ret = torch.empty((L, hkv, d), dtype=q.dtype, device=q.device)
    if v_ret is None:
        v_ret = torch.empty((L, hkv, d), dtype=q.dtype, device=q.device)
    return o, lse, k_ret, v_ret


def pulsar_phase1_encode(q, k, v, rope_theta, block, sink, chunk, k_chunks, sel, o=None, lse=None,
                         k_ret=None, v_ret=None, ws=None, want_lse=True):
    """Pulsar Phase 1 for all hosts. Returns (o, lse, k_ret, v_ret, row_off, ws)."""
    _dev(q, k, v, sel, o, lse, k_ret, v_ret)
    L, hq, d = q.shape
    hkv = k.shape[1]
    dt = _dtype_code(q)
    row_off = pa_phase1_layout(L, block, sink, k_chunks * chunk, False)
    _phase1_check(q, k, v, row_off[-1], L, o, lse, k_ret, v_ret, sel, (L // block if block > 0 else 0) * k_chunks)
    o, lse, k_ret, v_ret = _phase1_outputs(q, k, row_off[-1], o, lse, k_ret, v_ret, want_lse)
    need = pa_phase1_workspace_size(L, hq, hkv, d, dt, block, sink, k_chunks * chunk, False)
    ws = _workspace(need, q.device, ws)
    rc = _lib.pulsar_phase1_encode(_ptr(q), _ptr(k), _ptr(v), dt, L, hq, hkv, d, float(rope_theta), block,
                                   sink, chunk, k_chunks, _ptr(sel), _ptr(o), _ptr(lse), _ptr(k_ret),
                                   _ptr(v_ret), _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(rc, "pulsar_phase1_encode", ws)
    return o, lse, k_ret, v_ret, row_off, ws


def star_phase1_encode(q, k, v, rope_theta, block, o=None, lse=None, k_ret=None, v_ret=None,
                       ws=None, want_lse=True):
    """Star anchor-variant Phase 1. Returns (o, lse, k_ret, v_ret, row_off, ws)."""
    _dev(q, k, v, o, lse, k_ret, v_ret)
    L, hq, d = q.shape
    hkv = k.shape[1]
    dt = _dtype_code(q)
    row_off = pa_phase1_layout(L, block, 0, 0, True)
    _phase1_check(q, k, v, row_off[-1], L, o, lse, k_ret, v_ret)
    o, lse, k_ret, v_ret = _phase1_outputs(q, k, row_off[-1], o, lse, k_ret, v_ret, want_lse)
    need = pa_phase1_workspace_size(L, hq, hkv, d, dt, block, 0, 0, True)
    ws = _workspace(need, q.device, ws)
    rc = _lib.star_phase1_encode(_ptr(q), _ptr(k), _ptr(v), dt, L, hq, hkv, d, float(rope_theta), block,
                                 _ptr(o), _ptr(lse), _ptr(k_ret), _ptr(v_ret), _ptr(ws), ws.numel(),
                                 _stream())
    _check(rc, "star_phase1_encode", ws)
    return o, lse, k_ret, v_ret, row_off, ws


def _phase1_range_outputs(q, k, block, rows, nh, o, lse, k_ret, v_ret, want_lse):
    _, hq, d = q.shape
    hkv = k.shape[1]
    if o is None:
        o = torch.empty((rows, hq, d), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((rows, hq), dtype=torch.float32, device=q.device)
    if k_ret is None:
        k_ret = torch.empty((nh * block, hkv, d), dtype=q.dtype, device=q.device)
    if v_ret is None:
        v_ret = torch.empty((nh * block, hkv, d), dtype=q.dtype, device=q.device)
    return o, lse, k_ret, v_ret


def pulsar_phase1_encode_hosts(q, k, v, rope_theta, block, sink, chunk, k_chunks, sel, host_begin, host_end,
                               o=None, lse=None, k_ret=None, v_ret=None, ws=None, want_lse=True):
    """Pulsar Phase 1 of hosts [host_begin, host_end) only (one GPU's share of
    a sequence's hosts).  Returns (o, lse, k_ret, v_ret, row_off, ws): o / lse
    hold the range's rows packed from 0, row_off their offsets (starting at
    0), k_ret / v_ret the range's blocks."""
    _dev(q, k, v, sel, o, lse, k_ret, v_ret)
    L, hq, d = q.shape
    hkv = k.shape[1]
    dt = _dtype_code(q)
    full = pa_phase1_layout(L, block, sink, k_chunks * chunk, False)
    row_off = [r - full[host_begin] for r in full[host_begin:host_end + 1]]
    nh = max(host_end - host_begin, 0)
    _phase1_check(q, k, v, row_off[-1] if row_off else 0, nh * block, o, lse, k_ret, v_ret, sel,
                  (L // block if block > 0 else 0) * k_chunks)
    o, lse, k_ret, v_ret = _phase1_range_outputs(q, k, block, row_off[-1] if row_off else 0, nh, o, lse, k_ret,
                                                 v_ret, want_lse)
    need = pa_phase1_hosts_workspace_size(L, hq, hkv, d, dt, block, sink, k_chunks * chunk, False, host_begin,
                                          host_end)
    ws = _workspace(need, q.device, ws)
    rc = _lib.pulsar_phase1_encode_hosts(_ptr(q), _ptr(k), _ptr(v), dt, L, hq, hkv, d, float(rope_theta), block,
                                         sink, chunk, k_chunks, _ptr(sel), host_begin, host_end, _ptr(o), _ptr(lse),
                                         _ptr(k_ret), _ptr(v_ret), _ptr(ws), ws.numel(), _stream())
    _check(rc, "pulsar_phase1_encode_hosts", ws)
    return o, lse, k_ret, v_ret, row_off, ws


def star_phase1_encode_hosts(q, k, v, rope_theta, block, host_begin, host_end, o=None, lse=None, k_ret=None,
                             v_ret=None, ws=None, want_lse=True):
    """Star anchor-variant Phase 1 of hosts [host_begin, host_end) only.
    Returns (o, lse, k_ret, v_ret, row_off, ws) as pulsar_phase1_encode_hosts."""
    _dev(q, k, v, o, lse, k_ret, v_ret)
    L, hq, d = q.shape
    hkv = k.shape[1]
    dt = _dtype_code(q)
    full = pa_phase1_layout(L, block, 0, 0, True)
    row_off = [r - full[host_begin] for r in full[host_begin:host_end + 1]]
    nh = max(host_end - host_begin, 0)
    _phase1_check(q, k, v, row_off[-1] if row_off else 0, nh * block, o, lse, k_ret, v_ret)
    o, lse, k_ret, v_ret = _phase1_range_outputs(q, k, block, row_off[-1] if row_off else 0, nh, o, lse, k_ret,
                                                 v_ret, want_lse)
    need = pa_phase1_hosts_workspace_size(L, hq, hkv, d, dt, block, 0, 0, True, host_begin, host_end)
    ws = _workspace(need, q.device, ws)
    rc = _lib.star_phase1_encode_hosts(_ptr(q), _ptr(k), _ptr(v), dt, L, hq, hkv, d, float(rope_theta), block,
                                       host_begin, host_end, _ptr(o), _ptr(lse), _ptr(k_ret), _ptr(v_ret), _ptr(ws),
                                       ws.numel(), _stream())
    _check(rc, "star_phase1_encode_hosts", ws)
    return o, lse, k_ret, v_ret, row_off, ws


def _phase2_check(q, k_ret, v_ret, o, lse):
    """q [B][Tq][hq][d]; caches [B][T][hkv][d] in q's dtype (K and V alike);
    caller-supplied o / lse large enough."""
    if q.dim() != 4 or k_ret.dim() != 4:
        raise ValueError("q must be [B][Tq][hq][d] and the caches [B][T][hkv][d]")
    B, Tq, hq, d = q.shape
    if k_ret.shape[0] != B or k_ret.shape[3] != d or k_ret.dtype != q.dtype:
        raise ValueError(f"k_ret: {k_ret.dtype} {tuple(k_ret.shape)} does not match q {q.dtype} {tuple(q.shape)}")
    _same(k_ret, ("v_ret", v_ret))
    _need(o, "o", q.dtype, B * Tq * hq * d)
    _need(lse, "lse", torch.float32, B * Tq * hq)


def pa_phase2_workspace_size(B, Tq, T, n_shards, hq, hkv, d) -> int:
    return _lib.pa_phase2_workspace_size(B, Tq, T, n_shards, hq, hkv, d)


def star_phase2_attend(q, k_ret, v_ret, n_shards, q_pos0=0, rope_theta=0.0, o=None, lse=None,
                       want_partials=False, part_o=None, part_lse=None, ws=None):
    """Phase-2 split-KV attention + exact merge. q [B][Tq][hq][d]; caches [B][T][hkv][d].
    Returns (o, lse, part_o, part_lse, ws)."""
    _dev(q, k_ret, v_ret, o, lse, part_o, part_lse)
    _phase2_check(q, k_ret, v_ret, o, lse)
    B, Tq, hq, d = q.shape
    T, hkv = k_ret.shape[1], k_ret.shape[2]
    _need(part_o, "part_o", torch.float32, B * n_shards * Tq * hq * d)
    _need(part_lse, "part_lse", torch.float32, B * n_shards * Tq * hq)
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Tq, hq), dtype=torch.float32, device=q.device)
    if want_partials:
        if part_o is None:
            part_o = torch.empty((B, n_shards, Tq, hq, d), dtype=torch.float32, device=q.device)
        if part_lse is None:
            part_lse = torch.empty((B, n_shards, Tq, hq), dtype=torch.float32, device=q.device)
    need = pa_phase2_workspace_size(B, Tq, T, n_shards, hq, hkv, d)
    ws = _workspace(need, q.device, ws)
    rc = _lib.star_phase2_attend(_ptr(q), dt, B, Tq, int(q_pos0), float(rope_theta), _ptr(k_ret), _ptr(v_ret),
                                 T, n_shards, hq, hkv, d, _ptr(o), _ptr(lse), _ptr(part_o), _ptr(part_lse),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(rc, "star_phase2_attend", ws)
    return o, lse, part_o, part_lse, ws


def star_phase2_attend_art(q, k_ret, v_ret, q_pos0=0, rope_theta=0.0, block_keys=128, tau=1e-5, phi=1e-3,
                           patience=5, o=None, lse=None, ws=None):
    """Phase 2 with run-time early termination of the key walk (newest keys
    first).  bf16; Tq * hq / hkv <= 8.  Returns (o, lse, visited_blocks [B][hkv], ws)."""
    _dev(q, k_ret, v_ret, o, lse)
    _phase2_check(q, k_ret, v_ret, o, lse)
    B, Tq, hq, d = q.shape
    T, hkv = k_ret.shape[1], k_ret.shape[2]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Tq, hq), dtype=torch.float32, device=q.device)
    visited = torch.empty((B, hkv), dtype=torch.int32, device=q.device)
    ws = _workspace(pa_phase2_workspace_size(B, Tq, T, 1, hq, hkv, d), q.device, ws)
    rc = _lib.star_phase2_attend_art(_ptr(q), _dtype_code(q), B, Tq, int(q_pos0), float(rope_theta), _ptr(k_ret),
                                     _ptr(v_ret), T, hq, hkv, d, int(block_keys), float(tau), float(phi),
                                     int(patience), _ptr(o), _ptr(lse), _ptr(visited), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream())
    _check(rc, "star_phase2_attend_art", ws)
    return o, lse, visited, ws


def pa_lse_merge(part_o, part_lse, dtype=torch.bfloat16, o=None, lse=None):
    """Exact merge of partials part_o [B][S][Tq][hq][d], part_lse [B][S][Tq][hq]
    (float32, on the GPU).  Returns (o in ``dtype``, lse)."""
    _dev(part_o, part_lse, o, lse)
    if part_o.dim() != 5:
        raise ValueError("part_o must be [B][S][Tq][hq][d]")
    B, S, Tq, hq, d = part_o.shape
    _need(part_o, "part_o", torch.float32, B * S * Tq * hq * d)
    _need(part_lse, "part_lse", torch.float32, B * S * Tq * hq)
    _need(o, "o", o.dtype if o is not None else dtype, B * Tq * hq * d)
    _need(lse, "lse", torch.float32, B * Tq * hq)
    if o is None:
        o = torch.empty((B, Tq, hq, d), dtype=dtype, device=part_o.device)
    if lse is None:
        lse = torch.empty((B, Tq, hq), dtype=torch.float32, device=part_o.device)
    rc = _lib.pa_lse_merge(_ptr(part_o), _ptr(part_lse), B, S, Tq, hq, d, _dtype_code(o), _ptr(o), _ptr(lse),
                           _stream())
    _check(rc, "pa_lse_merge")
    return o, lse


def star_phase2_query_step(q, k_new, v_new, k_ret, v_ret, n_shards, k_self, v_self, self_len, q_pos0,
                           rope_theta, o=None, lse=None, ws=None):
    """Query-host step: append the new tokens' K/V (K rotated at q_pos0 + j)
    to the own cache at rows self_len + j, then attend (shards + own keys
    0..self_len + j, causal).  q/k_new/v_new [B][Tq][h][d]; caches
    [B][T][hkv][d]; k_self/v_self [B][cap][hkv][d].  Returns (o, lse, ws)."""
    _dev(q, k_new, v_new, k_ret, v_ret, k_self, v_self, o, lse)
    _phase2_check(q, k_ret, v_ret, o, lse)
    _phase2_check(q, k_self, v_self, None, None)
    B, Tq, hq, d = q.shape
    T, hkv = k_ret.shape[1], k_ret.shape[2]
    if k_self.shape[2] != hkv:
        raise ValueError(f"k_self: {k_self.shape[2]} kv heads, the shards have {hkv}")
    _need(k_new, "k_new", q.dtype, B * Tq * hkv * d)
    _same(k_new, ("v_new", v_new))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Tq, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(pa_phase2_workspace_size(B, Tq, T, n_shards, hq, hkv, d), q.device, ws)
    rc = _lib.star_phase2_query_step(_ptr(q), _ptr(k_new), _ptr(v_new), _dtype_code(q), B, Tq, int(q_pos0),
                                     float(rope_theta), _ptr(k_ret), _ptr(v_ret), T, n_shards, _ptr(k_self),
                                     _ptr(v_self), k_self.shape[1], int(self_len), hq, hkv, d, _ptr(o), _ptr(lse),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(rc, "star_phase2_query_step", ws)
    return o, lse, ws


def pa_testing_phase1_stall(q, k, v, block, wait_limit_us):
    """Test hook: Star Phase 1 through the tensor-core kernel with one
    unsatisfiable barrier and waits limited to ``wait_limit_us``; the
    workspace status then reads PA_ERR_TIMEOUT.  Returns the workspace."""
    _dev(q, k, v)
    L, hq, d = q.shape
    hkv = k.shape[1]
    row_off = pa_phase1_layout(L, block, 0, 0, True)
    o, _, k_ret, v_ret = _phase1_outputs(q, k, row_off[-1], None, None, None, None, False)
    ws = _workspace(pa_phase1_workspace_size(L, hq, hkv, d, PA_BF16, block, 0, 0, True), q.device)
    rc = _lib.pa_testing_phase1_stall(_ptr(q), _ptr(k), _ptr(v), L, hq, hkv, d, block, _ptr(o), _ptr(k_ret),
                                      _ptr(v_ret), _ptr(ws), ws.numel(), int(wait_limit_us), _stream())
    _check(rc, "pa_testing_phase1_stall")
    return ws


def pa_testing_phase2_stall(q, k_ret, v_ret, n_shards, wait_limit_us):
    """Test hook: Phase-2 attention (no RoPE) through the tensor-core query
    kernel with one unsatisfiable barrier and waits limited to
    ``wait_limit_us``; the workspace status then reads PA_ERR_TIMEOUT.
    Returns the workspace."""
    _dev(q, k_ret, v_ret)
    B, Tq, hq, d = q.shape
    T, hkv = k_ret.shape[1], k_ret.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty((B, Tq, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(pa_phase2_workspace_size(B, Tq, T, n_shards, hq, hkv, d), q.device)
    rc = _lib.pa_testing_phase2_stall(_ptr(q), _ptr(k_ret), _ptr(v_ret), B, Tq, T, n_shards, hq, hkv, d, _ptr(o),
                                      _ptr(lse), _ptr(ws), ws.numel(), int(wait_limit_us), _stream())
    _check(rc, "pa_testing_phase2_stall")
    return ws
