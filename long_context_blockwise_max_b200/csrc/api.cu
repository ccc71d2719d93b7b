// C ABI of the library (declared in include/pulsar.h): host-side argument
// validation, workspace carving and kernel launches.  No exception crosses
// this boundary, nothing here allocates device memory, and the only
// synchronising call is pa_workspace_status.
#include <cmath>
#include <cstring>

#include "pa_internal.h"
#include "../../include/pulsar_testing.h"

using namespace pa;

namespace pa {
ProfileEvents& profile_events() {
  static thread_local ProfileEvents ev;
  return ev;
}
}  // namespace pa

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < need) return PA_ERR_WORKSPACE;
  return PA_OK;
}

int clear_status(void* ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, kStatusBytes, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Row layout of Phase 1 (see pa_phase1_layout).  Returns PA_OK or an error.
int layout(int64_t L, int32_t block, int32_t sink, int32_t summary_tokens, int star,
           int64_t* row_off, int* n_out) {
  if (block <= 0 || L <= 0 || L % block != 0) return PA_ERR_INVALID;
  const int64_t n = L / block;
  if (sink < 0 || sink > block || summary_tokens < 0 || summary_tokens > block)
    return PA_ERR_INVALID;
  if (n > kMaxBlocks) return PA_ERR_UNSUPPORTED;
  row_off[0] = 0;
  for (int64_t i = 0; i < n; ++i) {
    int64_t ni;
    if (i == 0) ni = block;
    else if (star) ni = 2 * (int64_t)block;
    else ni = sink + i * (int64_t)summary_tokens + block;
    row_off[i + 1] = row_off[i] + ni;
  }
  *n_out = (int)n;
  return PA_OK;
}

// Rows of one Phase-1 call over hosts [h0, h1) and the rows of its rotated
// Q / K: by position (identity, rows 0 .. h1 * block) or, when that reads
// fewer rows, compact: [sink || Sigma_0 .. Sigma_{h1-2} || blocks h0 .. h1-1]
// (Star: [B_0 || blocks h0 .. h1-1]).
struct RangePlan {
  int64_t rows;      // packed output rows of the range
  int64_t qk_rows;   // rows of Qr / Kr
  int compact;
  int64_t ci_blk;    // Qr / Kr row of the range's first block row
};

RangePlan plan_range(const int64_t* off_all, int32_t block, int32_t sink, int64_t summ, int star, int h0,
                     int h1) {
  RangePlan r;
  r.rows = off_all[h1] - off_all[h0];
  r.qk_rows = (int64_t)h1 * block;
  r.compact = 0;
  r.ci_blk = (int64_t)h0 * block;
  if (h1 >= 2 && h1 > h0) {
    const int64_t pre = star ? (int64_t)block : (int64_t)sink + (int64_t)(h1 - 1) * summ;
    const int64_t c = pre + (int64_t)(h1 - h0) * block;
    if (c < r.qk_rows) {
      r.qk_rows = c;
      r.compact = 1;
      r.ci_blk = pre;
    }
  }
  return r;
}

int check_heads(int32_t hq, int32_t hkv, int32_t d, int dtype) {
  if (hq <= 0 || hkv <= 0 || hq % hkv != 0) return PA_ERR_INVALID;
  if (d != 64 && d != 128) return PA_ERR_UNSUPPORTED;
  if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

int phase1_common(const void* q, const void* k, const void* v, int dtype, int64_t L, int32_t hq,
                  int32_t hkv, int32_t d, double rope_theta, int32_t block, int32_t sink,
                  int32_t chunk, int32_t k_chunks, const int32_t* sel, int star, void* o,
                  float* lse_opt, void* k_ret, void* v_ret, void* ws, size_t ws_bytes,
                  cudaStream_t s, uint64_t wait_limit_ns = 1000000000ull, int stall = 0,
                  int32_t host_begin = 0, int32_t host_end = -1) {
  int rc = check_heads(hq, hkv, d, dtype);
  if (rc) return rc;
  if (!q || !k || !v) return PA_ERR_INVALID;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return PA_ERR_INVALID;
  if (!star) {
    if (chunk <= 0 || block % chunk != 0 || k_chunks < 0 || k_chunks > block / chunk)
      return PA_ERR_INVALID;
    if ((int64_t)k_chunks * chunk > block) return PA_ERR_INVALID;
    if (sink % 16 != 0 || chunk % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (k_chunks > 0 && L / block > 1 && sel == nullptr) return PA_ERR_INVALID;
  }
  if (block % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (L > INT32_MAX) return PA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, k_ret, v_ret};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return PA_ERR_UNSUPPORTED;
  HostTable ht;
  std::memset(&ht, 0, sizeof(ht));
  int n_all = 0;
  int64_t off_all[kMaxBlocks + 1];
  rc = layout(L, block, star ? 0 : sink, star ? 0 : k_chunks * chunk, star, off_all, &n_all);
  if (rc) return rc;
  // the encoded hosts: [host_begin, host_end) of the sequence's n_all hosts
  if (host_end < 0) host_end = n_all;
  if (host_begin < 0 || host_begin > host_end || host_end > n_all) return PA_ERR_INVALID;
  const int n = host_end - host_begin;
  if (n > 0 && (!o || !k_ret || !v_ret)) return PA_ERR_INVALID;   // outputs may be null for no host
  for (int i = 0; i <= n; ++i) ht.row_off[i] = off_all[host_begin + i] - off_all[host_begin];
  ht.n_hosts = n;
  ht.host0 = host_begin;
  ht.star = star;
  ht.block = block;
  ht.sink = star ? 0 : sink;
  ht.chunk = star ? 0 : chunk;
  ht.k_chunks = star ? 0 : k_chunks;
  ht.tile_off[0] = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t ni = ht.row_off[i + 1] - ht.row_off[i];
    ht.tile_off[i + 1] = ht.tile_off[i] + (int32_t)((ni + 127) / 128);
  }
  const int64_t R = ht.row_off[n];
  const RangePlan plan = plan_range(off_all, block, ht.sink, (int64_t)ht.k_chunks * ht.chunk, star,
                                    host_begin, host_end);
  ht.compact = plan.compact;
  ht.ci_blk = plan.ci_blk;
  const size_t need =
      phase1_workspace_bytes(plan.qk_rows, hq, hkv, d, dtype, R, plan.compact ? plan.qk_rows : 0);
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  Phase1Args a;
  a.dtype = dtype;
  a.q = q; a.k = k; a.v = v;
  a.L = L; a.hq = hq; a.hkv = hkv; a.d = d;
  a.rope_theta = rope_theta;
  a.sel = sel;
  a.ht = ht;
  a.qk_rows = plan.qk_rows;
  a.kret_lo = plan.ci_blk;
  a.ret_lo = (int64_t)host_begin * block;
  a.ret_hi = (int64_t)host_end * block;
  a.o = o; a.lse = lse_opt; a.k_ret = k_ret; a.v_ret = v_ret;
  char* w = static_cast<char*>(ws);
  a.status = reinterpret_cast<DeviceStatus*>(w);
  size_t off = kStatusBytes;
  a.rowpos = reinterpret_cast<int32_t*>(w + off);
  off += align_up(sizeof(int32_t) * (size_t)R);
  a.rowci = plan.compact ? reinterpret_cast<int32_t*>(w + off) : a.rowpos;
  off += align_up(sizeof(int32_t) * (size_t)R);
  a.posmap = plan.compact ? reinterpret_cast<int32_t*>(w + off) : nullptr;
  off += align_up(sizeof(int32_t) * (size_t)(plan.compact ? plan.qk_rows : 0));
  const size_t qk_elem = dtype == PA_BF16 ? 2 : 4;
  a.qr = w + off;
  off += align_up(qk_elem * (size_t)plan.qk_rows * hq * d);
  a.kr = w + off;
  if (n == 0) return PA_OK;
  a.wait_limit_ns = wait_limit_ns;
  a.stall = stall;
  return launch_phase1(a, s);
}

void carve_phase2(Phase2Args& a, void* ws) {
  char* w = static_cast<char*>(ws);
  a.status = reinterpret_cast<DeviceStatus*>(w);
  const size_t rows = (size_t)a.B * a.Tq * a.hq;
  const size_t units = (size_t)a.n_shards * a.n_split + 1;   // + the own-cache unit
  size_t off = kStatusBytes;
  a.qr = reinterpret_cast<float*>(w + off);
  off += align_up(sizeof(float) * rows * a.d);
  a.unit_o = reinterpret_cast<float*>(w + off);
  off += align_up(sizeof(float) * rows * units * a.d);
  a.unit_lse = reinterpret_cast<float*>(w + off);
  off += align_up(sizeof(float) * rows * units);
  a.q16 = reinterpret_cast<__half*>(w + off);
  off += align_up(sizeof(__half) * rows * a.d);
  a.redo = reinterpret_cast<int32_t*>(w + off);
}

}  // namespace

extern "C" {

int pa_abi_version(void) { return PA_ABI_VERSION; }

int pa_set_profile_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return PA_ERR_INVALID;
  profile_events().start = static_cast<cudaEvent_t>(start);
  profile_events().stop = static_cast<cudaEvent_t>(stop);
  return PA_OK;
}

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PA_ERR_CUDA: return "CUDA launch or copy failed";
    case PA_ERR_TIMEOUT: return "bounded device wait expired";
    case PA_ERR_RANGE: return "value outside the internal fp16 range";
    default: return "unknown status";
  }
}

int pa_workspace_status(const void* ws, void* stream) {
  if (ws == nullptr) return PA_ERR_WORKSPACE;
  int32_t code = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  return code;
}

size_t pa_select_workspace_size(int64_t L, int32_t vocab, int32_t block, int32_t chunk) {
  if (L < 0 || vocab <= 0 || block <= 0 || chunk <= 0 || block % chunk || L % block) return 0;
  size_t b = kStatusBytes;
  b += align_up(sizeof(unsigned long long) * (size_t)vocab);
  b += align_up(sizeof(int32_t) * (size_t)(L / chunk));
  b += align_up(kScoreKeyBytes * (size_t)(L / chunk));      // mean-IDF keys (scorer variants)
  return b;
}

int pulsar_select_summaries_scored(const int32_t* ids, int64_t L, int32_t vocab, int32_t block,
                                   int32_t chunk, int32_t k_chunks, int method, int32_t* sel,
                                   int64_t* chunk_score_opt, void* ws, size_t ws_bytes,
                                   void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (method != PA_SCORE_MAX_IDF && method != PA_SCORE_MEAN_IDF && method != PA_SCORE_EVENLY_SPACED &&
      method != PA_SCORE_ENTROPY && method != PA_SCORE_BM25)
    return PA_ERR_INVALID;
  const bool ranked = method == PA_SCORE_MEAN_IDF || method == PA_SCORE_ENTROPY || method == PA_SCORE_BM25;
  if (L <= 0 || vocab <= 0 || block <= 0 || chunk <= 0) return PA_ERR_INVALID;
  if (L % block != 0 || block % chunk != 0) return PA_ERR_INVALID;
  if (k_chunks < 0 || k_chunks > block / chunk) return PA_ERR_INVALID;
  if ((ids == nullptr && method != PA_SCORE_EVENLY_SPACED) || (sel == nullptr && k_chunks > 0))
    return PA_ERR_INVALID;
  if (L / block > kMaxBlocks) return PA_ERR_UNSUPPORTED;
  if (ranked && (block / chunk > kMaxScoredChunks || chunk > kMaxScoredChunk)) return PA_ERR_UNSUPPORTED;
  const size_t need = pa_select_workspace_size(L, vocab, block, chunk);
  int rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  char* w = static_cast<char*>(ws);
  SelectArgs a;
  a.ids = ids; a.L = L; a.vocab = vocab; a.block = block; a.chunk = chunk; a.k = k_chunks;
  a.sel = sel; a.df_out = nullptr;
  a.status = reinterpret_cast<DeviceStatus*>(w);
  size_t off = kStatusBytes;
  a.mask = reinterpret_cast<unsigned long long*>(w + off);
  off += align_up(sizeof(unsigned long long) * (size_t)vocab);
  int32_t* mindf = reinterpret_cast<int32_t*>(w + off);
  off += align_up(sizeof(int32_t) * (size_t)(L / chunk));
  long long* score = reinterpret_cast<long long*>(chunk_score_opt);
  a.mindf = mindf;
  if (method == PA_SCORE_MAX_IDF) {
    rc = launch_select(a, s);
    if (rc == PA_OK && score != nullptr) {
      // widen the min df of every chunk into the caller's int64 array
      rc = launch_widen_i32(mindf, score, L / chunk, s);
    }
    return rc;
  }
  return launch_select_scored(a, method, w + off, score, s);
}

int pulsar_select_summaries(const int32_t* ids, int64_t L, int32_t vocab, int32_t block,
                            int32_t chunk, int32_t k_chunks, int32_t* sel, int32_t* df_opt,
                            int32_t* chunk_mindf_opt, void* ws, size_t ws_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L <= 0 || vocab <= 0 || block <= 0 || chunk <= 0) return PA_ERR_INVALID;
  if (L % block != 0 || block % chunk != 0) return PA_ERR_INVALID;
  if (k_chunks < 0 || k_chunks > block / chunk) return PA_ERR_INVALID;
  if (ids == nullptr || (sel == nullptr && k_chunks > 0)) return PA_ERR_INVALID;
  if (L / block > kMaxBlocks) return PA_ERR_UNSUPPORTED;
  const size_t need = pa_select_workspace_size(L, vocab, block, chunk);
  int rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  char* w = static_cast<char*>(ws);
  SelectArgs a;
  a.ids = ids; a.L = L; a.vocab = vocab; a.block = block; a.chunk = chunk; a.k = k_chunks;
  a.sel = sel; a.df_out = df_opt;
  a.status = reinterpret_cast<DeviceStatus*>(w);
  size_t off = kStatusBytes;
  a.mask = reinterpret_cast<unsigned long long*>(w + off);
  off += align_up(sizeof(unsigned long long) * (size_t)vocab);
  a.mindf = chunk_mindf_opt ? chunk_mindf_opt : reinterpret_cast<int32_t*>(w + off);
  return launch_select(a, s);
}

int pa_phase1_layout(int64_t L, int32_t block, int32_t sink, int32_t summary_tokens, int star,
                     int64_t* row_off) {
  if (row_off == nullptr) return PA_ERR_INVALID;
  int64_t tmp[kMaxBlocks + 1];
  int n = 0;
  const int rc = layout(L, block, sink, summary_tokens, star, tmp, &n);
  if (rc) return rc;
  std::memcpy(row_off, tmp, sizeof(int64_t) * (size_t)(n + 1));
  return PA_OK;
}

size_t pa_phase1_workspace_size(int64_t L, int32_t hq, int32_t hkv, int32_t d, int dtype,
                                int32_t block, int32_t sink, int32_t summary_tokens, int star) {
  if (check_heads(hq, hkv, d, dtype)) return 0;
  int64_t off[kMaxBlocks + 1];
  int n = 0;
  if (layout(L, block, star ? 0 : sink, star ? 0 : summary_tokens, star, off, &n)) return 0;
  // enough for the call over every host and for any host range (a compact
  // range has fewer than L rotated rows)
  return phase1_workspace_bytes(L, hq, hkv, d, dtype, off[n], L);
}

size_t pa_phase1_hosts_workspace_size(int64_t L, int32_t hq, int32_t hkv, int32_t d, int dtype,
                                      int32_t block, int32_t sink, int32_t summary_tokens, int star,
                                      int32_t host_begin, int32_t host_end) {
  if (check_heads(hq, hkv, d, dtype)) return 0;
  int64_t off[kMaxBlocks + 1];
  int n = 0;
  if (star) sink = summary_tokens = 0;
  if (layout(L, block, sink, summary_tokens, star, off, &n)) return 0;
  if (host_begin < 0 || host_begin > host_end || host_end > n) return 0;
  const RangePlan plan = plan_range(off, block, sink, summary_tokens, star, host_begin, host_end);
  return phase1_workspace_bytes(plan.qk_rows, hq, hkv, d, dtype, plan.rows, plan.compact ? plan.qk_rows : 0);
}

int pulsar_phase1_encode(const void* q, const void* k, const void* v, int dtype, int64_t L,
                         int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                         int32_t sink, int32_t chunk, int32_t k_chunks, const int32_t* sel,
                         void* o, float* lse_opt, void* k_ret, void* v_ret, void* ws,
                         size_t ws_bytes, void* stream) {
  return phase1_common(q, k, v, dtype, L, hq, hkv, d, rope_theta, block, sink, chunk, k_chunks,
                       sel, 0, o, lse_opt, k_ret, v_ret, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

int star_phase1_encode(const void* q, const void* k, const void* v, int dtype, int64_t L,
                       int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                       void* o, float* lse_opt, void* k_ret, void* v_ret, void* ws,
                       size_t ws_bytes, void* stream) {
  return phase1_common(q, k, v, dtype, L, hq, hkv, d, rope_theta, block, 0, 16, 0, nullptr, 1,
                       o, lse_opt, k_ret, v_ret, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int pulsar_phase1_encode_hosts(const void* q, const void* k, const void* v, int dtype, int64_t L,
                               int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                               int32_t sink, int32_t chunk, int32_t k_chunks, const int32_t* sel,
                               int32_t host_begin, int32_t host_end, void* o, float* lse_opt,
                               void* k_ret, void* v_ret, void* ws, size_t ws_bytes, void* stream) {
  if (host_end < 0) return PA_ERR_INVALID;
  return phase1_common(q, k, v, dtype, L, hq, hkv, d, rope_theta, block, sink, chunk, k_chunks,
                       sel, 0, o, lse_opt, k_ret, v_ret, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream), 1000000000ull, 0, host_begin, host_end);
}

int star_phase1_encode_hosts(const void* q, const void* k, const void* v, int dtype, int64_t L,
                             int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                             int32_t host_begin, int32_t host_end, void* o, float* lse_opt,
                             void* k_ret, void* v_ret, void* ws, size_t ws_bytes, void* stream) {
  if (host_end < 0) return PA_ERR_INVALID;
  return phase1_common(q, k, v, dtype, L, hq, hkv, d, rope_theta, block, 0, 16, 0, nullptr, 1,
                       o, lse_opt, k_ret, v_ret, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                       1000000000ull, 0, host_begin, host_end);
}

size_t pa_phase2_workspace_size(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                                int32_t hkv, int32_t d) {
  if (B < 0 || Tq < 0 || T < 0 || n_shards < 1 || n_shards > 4096) return 0;
  if (check_heads(hq, hkv, d, PA_F32)) return 0;
  return phase2_workspace_bytes(B, Tq, T, n_shards, hq, hkv, d);
}

int star_phase2_attend(const void* q, int dtype, int32_t B, int32_t Tq, int64_t q_pos0,
                       double rope_theta, const void* k_ret, const void* v_ret, int64_t T,
                       int32_t n_shards, int32_t hq, int32_t hkv, int32_t d, void* o, float* lse,
                       float* part_o_opt, float* part_lse_opt, void* ws, size_t ws_bytes,
                       void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = check_heads(hq, hkv, d, dtype);
  if (rc) return rc;
  if (B < 0 || Tq < 0 || T < 0 || n_shards < 1 || n_shards > 4096) return PA_ERR_INVALID;
  if (!std::isfinite(rope_theta)) return PA_ERR_INVALID;
  if (B > 0 && Tq > 0) {
    if (!q || !o || !lse) return PA_ERR_INVALID;
    if (T > 0 && (!k_ret || !v_ret)) return PA_ERR_INVALID;
  }
  const void* ptrs[] = {q, k_ret, v_ret, o, part_o_opt};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return PA_ERR_UNSUPPORTED;
  const size_t need = phase2_workspace_bytes(B, Tq, T, n_shards, hq, hkv, d);
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  Phase2Args a;
  a.dtype = dtype;
  a.q = q; a.B = B; a.Tq = Tq; a.q_pos0 = q_pos0; a.rope_theta = rope_theta;
  a.k_ret = k_ret; a.v_ret = v_ret; a.T = T;
  // without per-shard partials the units need not follow shard boundaries
  a.n_shards = phase2_flat_units(B, Tq, n_shards, hq, hkv, part_o_opt || part_lse_opt) ? 1 : n_shards;
  a.n_split = phase2_split(B, Tq, T, a.n_shards, hq, hkv);
  a.hq = hq; a.hkv = hkv; a.d = d;
  a.o = o; a.lse = lse; a.part_o_opt = part_o_opt; a.part_lse_opt = part_lse_opt;
  carve_phase2(a, ws);
  if (B == 0 || Tq == 0) return PA_OK;
  return launch_phase2(a, s);
}

int star_phase2_attend_art(const void* q, int dtype, int32_t B, int32_t Tq, int64_t q_pos0,
                           double rope_theta, const void* k_ret, const void* v_ret, int64_t T,
                           int32_t hq, int32_t hkv, int32_t d, int32_t block_keys, double tau,
                           double phi, int32_t patience, void* o, float* lse,
                           int32_t* visited_blocks_opt, void* ws, size_t ws_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = check_heads(hq, hkv, d, dtype);
  if (rc) return rc;
  if (dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (B < 0 || Tq < 0 || T < 0 || !std::isfinite(rope_theta)) return PA_ERR_INVALID;
  if (block_keys < 32 || block_keys % 32 != 0 || patience < 1 || !(tau >= 0) || !(phi >= 0))
    return PA_ERR_INVALID;
  if ((int64_t)Tq * (hq / hkv) > 8) return PA_ERR_UNSUPPORTED;
  if (B > 0 && Tq > 0 && (!q || !o || !lse || (T > 0 && (!k_ret || !v_ret)))) return PA_ERR_INVALID;
  const void* ptrs[] = {q, k_ret, v_ret, o};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return PA_ERR_UNSUPPORTED;
  const size_t need = phase2_workspace_bytes(B, Tq, T, 1, hq, hkv, d);
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  Phase2Args a;
  a.dtype = dtype;
  a.q = q; a.B = B; a.Tq = Tq; a.q_pos0 = q_pos0; a.rope_theta = rope_theta;
  a.k_ret = k_ret; a.v_ret = v_ret; a.T = T;
  a.n_shards = 1; a.n_split = 1;
  a.hq = hq; a.hkv = hkv; a.d = d;
  a.o = o; a.lse = lse; a.part_o_opt = nullptr; a.part_lse_opt = nullptr;
  carve_phase2(a, ws);
  if (B == 0 || Tq == 0) return PA_OK;
  ArtArgs art;
  art.block_keys = block_keys;
  art.tau = static_cast<float>(tau);
  art.phi = static_cast<float>(phi);
  art.patience = patience;
  art.visited = visited_blocks_opt;
  rc = launch_rope_query(a, s);
  if (rc) return rc;
  return launch_phase2_art(a, art, s);
}

int pa_lse_merge(const float* part_o, const float* part_lse, int32_t B, int32_t S, int32_t Tq,
                 int32_t hq, int32_t d, int dtype, void* o, float* lse, void* stream) {
  if (B < 0 || S < 1 || Tq < 0 || hq < 1) return PA_ERR_INVALID;
  if (d != 64 && d != 128) return PA_ERR_UNSUPPORTED;
  if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (B > 0 && Tq > 0 && (!part_o || !part_lse || !o || !lse)) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(part_o) & 15u) != 0) return PA_ERR_INVALID;   // vector loads
  Phase2Args a;
  a.dtype = dtype;
  a.B = B; a.Tq = Tq; a.hq = hq; a.hkv = hq; a.d = d;
  a.n_shards = S; a.n_split = 1; a.has_self = 0;
  a.unit_o = const_cast<float*>(part_o);
  a.unit_lse = const_cast<float*>(part_lse);
  a.part_o_opt = nullptr; a.part_lse_opt = nullptr;
  a.o = o; a.lse = lse;
  a.status = nullptr;
  return launch_merge_only(a, static_cast<cudaStream_t>(stream));
}

int star_phase2_query_step(const void* q, const void* k_new, const void* v_new, int dtype, int32_t B,
                           int32_t Tq, int64_t q_pos0, double rope_theta, const void* k_ret,
                           const void* v_ret, int64_t T, int32_t n_shards, void* k_self, void* v_self,
                           int64_t self_cap, int64_t self_len, int32_t hq, int32_t hkv, int32_t d,
                           void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = check_heads(hq, hkv, d, dtype);
  if (rc) return rc;
  if (B < 0 || Tq < 0 || T < 0 || n_shards < 1 || n_shards > 4096) return PA_ERR_INVALID;
  if (!std::isfinite(rope_theta)) return PA_ERR_INVALID;
  if (self_len < 0 || self_cap < 0 || self_len + Tq > self_cap) return PA_ERR_INVALID;
  if (B > 0 && Tq > 0) {
    if (!q || !k_new || !v_new || !k_self || !v_self || !o || !lse) return PA_ERR_INVALID;
    if (T > 0 && (!k_ret || !v_ret)) return PA_ERR_INVALID;
  }
  const void* ptrs[] = {q, k_new, v_new, k_ret, v_ret, k_self, v_self, o};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return PA_ERR_UNSUPPORTED;
  const size_t need = phase2_workspace_bytes(B, Tq, T, n_shards, hq, hkv, d);
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  rc = clear_status(ws, s);
  if (rc) return rc;
  Phase2Args a;
  a.dtype = dtype;
  a.q = q; a.B = B; a.Tq = Tq; a.q_pos0 = q_pos0; a.rope_theta = rope_theta;
  a.k_ret = k_ret; a.v_ret = v_ret; a.T = T;
  // no per-shard partials: the context's units need not follow shard boundaries
  a.n_shards = phase2_flat_units(B, Tq, n_shards, hq, hkv, false) ? 1 : n_shards;
  a.n_split = phase2_split(B, Tq, T, a.n_shards, hq, hkv);
  a.hq = hq; a.hkv = hkv; a.d = d;
  a.o = o; a.lse = lse; a.part_o_opt = nullptr; a.part_lse_opt = nullptr;
  a.k_self = k_self; a.v_self = v_self; a.self_cap = self_cap; a.self_len = self_len;
  a.has_self = 1;
  carve_phase2(a, ws);
  if (B == 0 || Tq == 0) return PA_OK;
  rc = launch_self_append(a, k_new, v_new, s);
  if (rc) return rc;
  return launch_phase2(a, s);
}

int pa_testing_phase1_stall(const void* q, const void* k, const void* v, int64_t L, int32_t hq,
                            int32_t hkv, int32_t d, int32_t block, void* o, void* k_ret,
                            void* v_ret, void* ws, size_t ws_bytes, int32_t wait_limit_us,
                            void* stream) {
  if (wait_limit_us <= 0 || wait_limit_us > 10000000) return PA_ERR_INVALID;
  if (hkv <= 0 || hq % hkv != 0 || (hq / hkv) % 2 != 0) return PA_ERR_UNSUPPORTED;   // tensor-core path only
  return phase1_common(q, k, v, PA_BF16, L, hq, hkv, d, 10000.0, block, 0, 16, 0, nullptr, 1, o,
                       nullptr, k_ret, v_ret, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                       static_cast<uint64_t>(wait_limit_us) * 1000ull, 1);
}

int pa_testing_phase2_stall(const void* q, const void* k_ret, const void* v_ret, int32_t B, int32_t Tq,
                            int64_t T, int32_t n_shards, int32_t hq, int32_t hkv, int32_t d, void* o,
                            float* lse, void* ws, size_t ws_bytes, int32_t wait_limit_us, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (wait_limit_us <= 0 || wait_limit_us > 10000000) return PA_ERR_INVALID;
  int rc = check_heads(hq, hkv, d, PA_BF16);
  if (rc) return rc;
  if (B < 1 || Tq < 1 || T < 1 || n_shards < 1 || n_shards > 4096) return PA_ERR_INVALID;
  if (!q || !k_ret || !v_ret || !o || !lse) return PA_ERR_INVALID;
  const size_t need = phase2_workspace_bytes(B, Tq, T, n_shards, hq, hkv, d);
  rc = check_ws(ws, ws_bytes, need);
  if (rc) return rc;
  Phase2Args a;
  a.dtype = PA_BF16;
  a.q = q; a.B = B; a.Tq = Tq; a.q_pos0 = 0; a.rope_theta = 0.0;
  a.k_ret = k_ret; a.v_ret = v_ret; a.T = T;
  a.n_shards = n_shards;
  a.n_split = phase2_split(B, Tq, T, n_shards, hq, hkv);
  a.hq = hq; a.hkv = hkv; a.d = d;
  a.o = o; a.lse = lse; a.part_o_opt = nullptr; a.part_lse_opt = nullptr;
  a.wait_limit_ns = static_cast<uint64_t>(wait_limit_us) * 1000ull;
  a.stall = 1;
  if (!phase2_tc_supported(a)) return PA_ERR_UNSUPPORTED;   // tensor-core query path only
  rc = clear_status(ws, s);
  if (rc) return rc;
  carve_phase2(a, ws);
  return launch_phase2(a, s);
}

}  // extern "C"
