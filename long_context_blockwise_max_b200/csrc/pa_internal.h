// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kMaxBlocks = 64;   // per-token block mask is 64 bits
constexpr int kMaxHalfDim = 64;  // d <= 128

// Caller-provided events bracketing the dominant kernel (pa_set_profile_events).
struct ProfileEvents {
  cudaEvent_t start = nullptr, stop = nullptr;
};
ProfileEvents& profile_events();
inline void profile_begin(cudaStream_t s) {
  if (profile_events().start) cudaEventRecord(profile_events().start, s);
}
inline void profile_end(cudaStream_t s) {
  if (profile_events().stop) cudaEventRecord(profile_events().stop, s);
}

struct SelectArgs {
  const int32_t* ids;
  int64_t L;
  int32_t vocab, block, chunk, k;
  int32_t* sel;
  int32_t* df_out;              // may be null
  int32_t* mindf;               // [L / chunk] (caller's or workspace)
  unsigned long long* mask;     // [vocab] workspace
  DeviceStatus* status;
};
int launch_select(const SelectArgs& a, cudaStream_t s);

// Mean-IDF scorer: chunks are ranked by the exact product of df over their
// tokens, a 256-bit key per chunk (32 bytes of workspace per chunk).
constexpr int kMaxScoredChunks = 4096;   // chunks per block (keys staged in shared memory)
constexpr int kMaxScoredChunk = 32;      // tokens per chunk: 64^32 < 2^256
constexpr size_t kScoreKeyBytes = 32;
int launch_widen_i32(const int32_t* in, long long* out, int64_t n, cudaStream_t s);
// key_ws: [L / chunk] 32-byte keys; a.mindf receives the int32 ranks;
// rank_out (optional) the int64 ranks.
int launch_select_scored(const SelectArgs& a, int method, void* key_ws, long long* rank_out,
                         cudaStream_t s);

// Host-computed RoPE frequencies omega_m = theta^(-2m/d), fp64.
struct RopeFreqs {
  double omega[kMaxHalfDim];
};

// Phase-1 host layout shared by the kernels (small, passed by value).
struct HostTable {
  int32_t n_hosts;                   // hosts in this table (a contiguous range)
  int32_t host0;                     // sequence index of the table's first host
  int32_t star;
  int32_t block, sink, chunk, k_chunks;
  int64_t row_off[kMaxBlocks + 1];   // packed output row offsets
  int32_t tile_off[kMaxBlocks + 1];  // cumulative 128-row tiles per host
  // Rotated Q / K rows: by position (compact == 0), or, for a host range
  // that reads few positions, in the compact order [sink || Sigma_0 ..
  // Sigma_{host_end-2} || the range's blocks] (Star: [B_0 || the range's
  // blocks]), the blocks starting at compact row ci_blk.
  int32_t compact;
  int64_t ci_blk;
};

// Rows at the start of every host that Phase 1 recomputes in fp32 when Q / K
// are carried in fp16 (they see too few keys to average the rounding out).
constexpr int kHeadRows = 32;

struct Phase1Args {
  int dtype;                    // PA_F32 / PA_BF16
  const void *q, *k, *v;        // inputs [L][h][d]
  int64_t L;
  int32_t hq, hkv, d;
  double rope_theta;
  const int32_t* sel;           // [N][k] (Pulsar) or null (Star)
  HostTable ht;
  void* o;                      // [R][hq][d]
  float* lse;                   // [R][hq] or null
  void *k_ret, *v_ret;          // [L][hkv][d]
  // workspace carve
  int32_t* rowpos;              // [R] original position of every packed row (V rows)
  int32_t* rowci;               // [R] row of Qr / Kr of every packed row (== rowpos unless compact)
  int32_t* posmap;              // [qk_rows] original position of each Qr / Kr row, or null (identity)
  void* qr;                     // [qk_rows][hq][d] rotated, scaled Q (fp16 or fp32)
  void* kr;                     // [qk_rows][hkv][d] rotated K in the QK type (fp16 or fp32)
  // Qr / Kr rows [0, qk_rows) are rotated; k_ret receives Qr/Kr rows
  // [kret_lo, kret_lo + ret_hi - ret_lo); k_ret / v_ret hold positions
  // [ret_lo, ret_hi) (the blocks of the table's hosts)
  int64_t qk_rows = 0, kret_lo = 0, ret_lo = 0, ret_hi = 0;
  DeviceStatus* status;
  // bounded-wait limit of the tensor-core kernel and a test-only stall
  uint64_t wait_limit_ns = 1000000000ull;
  int stall = 0;
};
bool phase1_tc_supported(const Phase1Args& a);
int launch_phase1_tc(const Phase1Args& a, cudaStream_t s);
// Scratch of one Phase-1 call: status, rowpos and rowci [rows], posmap
// [posmap_rows], Qr / Kr [qk_rows].
size_t phase1_workspace_bytes(int64_t qk_rows, int32_t hq, int32_t hkv, int32_t d, int dtype,
                              int64_t rows, int64_t posmap_rows);
int launch_phase1(const Phase1Args& a, cudaStream_t s);

struct Phase2Args {
  int dtype;
  const void* q;                // [B][Tq][hq][d]
  int32_t B, Tq;
  int64_t q_pos0;
  double rope_theta;
  const void *k_ret, *v_ret;    // [B][T][hkv][d]
  int64_t T;
  int32_t n_shards, n_split;    // units = n_shards * n_split per batch element
  int32_t hq, hkv, d;
  void* o;                      // [B][Tq][hq][d]
  float* lse;                   // [B][Tq][hq]
  float* part_o_opt;            // [B][n_shards][Tq][hq][d]
  float* part_lse_opt;          // [B][n_shards][Tq][hq]
  float* qr;                    // workspace [B][Tq][hq][d]
  float* unit_o;                // workspace [B][units][Tq][hq][d]
  float* unit_lse;              // workspace [B][units][Tq][hq]
  DeviceStatus* status;
  // optional own cache of the query host ([B][self_cap][hkv][d], K rotated):
  // query row t also sees its rows 0 .. self_len + t (one extra unit)
  const void* k_self = nullptr;
  const void* v_self = nullptr;
  int64_t self_cap = 0, self_len = 0;
  int has_self = 0;
  // bounded-wait limit of the tensor-core query kernel and a test-only stall
  uint64_t wait_limit_ns = 1000000000ull;
  int stall = 0;
  // tensor-core query path: the fp16 query, and per (batch, unit, kv head)
  // flags of units to recompute exactly (+ one flag: the query left fp16
  // range), both in the workspace
  __half* q16 = nullptr;
  int32_t* redo = nullptr;   // [B * units * hkv + 1]
};

// One Phase-2 work unit: a split of a context shard, or (the last unit, when
// the own cache is attached) the own cache with its causal limit.
struct UnitView {
  const void* K;
  const void* V;
  int64_t stride_rows;    // rows per batch element of K / V
  int64_t k0, k1;         // key range
  int64_t causal_base;    // row t sees keys <= causal_base + t; -1: every key
};

__host__ __device__ inline int phase2_units(const Phase2Args& a) {
  return a.n_shards * a.n_split + (a.has_self ? 1 : 0);
}

__device__ inline UnitView phase2_unit(const Phase2Args& a, int u) {
  UnitView v;
  const int ctx = a.n_shards * a.n_split;
  if (u >= ctx) {
    v.K = a.k_self;
    v.V = a.v_self;
    v.stride_rows = a.self_cap;
    v.k0 = 0;
    v.k1 = a.self_len + a.Tq;
    v.causal_base = a.self_len;
    return v;
  }
  v.K = a.k_ret;
  v.V = a.v_ret;
  v.stride_rows = a.T;
  const int64_t step = (a.T + a.n_shards - 1) / a.n_shards;
  const int sh = u / a.n_split, sp = u % a.n_split;
  const int64_t lo = min((int64_t)sh * step, a.T), hi = min((int64_t)(sh + 1) * step, a.T);
  const int64_t len = (hi - lo + a.n_split - 1) / a.n_split;
  v.k0 = min(lo + (int64_t)sp * len, hi);
  v.k1 = min(lo + (int64_t)(sp + 1) * len, hi);
  v.causal_base = -1;
  return v;
}
int launch_phase2_mma(const Phase2Args& a, cudaStream_t s);
bool phase2_flat_units(int32_t B, int32_t Tq, int32_t n_shards, int32_t hq, int32_t hkv, bool want_partials);
// Tensor-core (tcgen05) kernel for queries with at least kPhase2TcMinRows rows
// per kv head; q16 is the rotated query scaled to log2 units, in fp16.
constexpr int kPhase2TcMinRows = 64;
bool phase2_tc_supported(const Phase2Args& a);
int launch_phase2_tc(const Phase2Args& a, const __half* q16, cudaStream_t s);

// ART early termination of the Phase-2 key walk (one warp per (b, kv head)).
struct ArtArgs {
  int block_keys;        // keys per stability check (multiple of 32)
  float tau, phi;        // magnitude / direction thresholds
  int patience;          // consecutive stable blocks before stopping
  int32_t* visited;      // [B][hkv] blocks visited, or null
};
int launch_phase2_art(const Phase2Args& a, const ArtArgs& art, cudaStream_t s);
int launch_rope_query(const Phase2Args& a, cudaStream_t s);
int32_t phase2_split(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                     int32_t hkv);
size_t phase2_workspace_bytes(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                              int32_t hkv, int32_t d);
int launch_phase2(const Phase2Args& a, cudaStream_t s);
int launch_merge_only(const Phase2Args& a, cudaStream_t s);
// rotate the new tokens' K at q_pos0 + j and append K, V to the own cache
int launch_self_append(const Phase2Args& a, const void* k_new, const void* v_new, cudaStream_t s);

}  // namespace pa
