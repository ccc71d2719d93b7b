// Phase-2 global query attention: split-KV partial attention per shard and
// the exact log-sum-exp merge (Pulsar Attention page §2.2; Dutch technical
// summary "Fase 2"; Star Attention review, key_machinery and the referee's
// correction of Algorithm 2: O = sum_h exp(s_h - s_global) A_h).
//
// Work unit = (batch element, shard split, kv head) and a group of query rows.
// A shard may be cut into `n_split` contiguous splits so that small batches
// still fill the GPU; the merge is associative, so splits and shards merge
// with the same algebra.  Kernels by case:
//   bf16, >= 64 query rows per kv head   phase2_tc_kernel (phase2_tc.cu)
//   bf16, <= 8 rows (decode)             phase2_mma_kernel (phase2_mma.cu)
//   bf16, other row counts               phase2_mma_rows_kernel (phase2_mma.cu)
//   fp32                                 phase2_simt_kernel (below)
// followed by merge_kernel; this file also holds the query RoPE, the split
// heuristic and the own-cache append of the query-host step.
#include "pa_internal.h"

namespace pa {

// q [B][Tq][hq][d] -> qr fp32, rotated at q_pos0 + t (theta > 0) and scaled
// by log2(e)/sqrt(d) so that scores come out in log2 units.  With `q16` set,
// also writes that value in fp16 (same layout; the operand of the
// tensor-core query kernel) and, when it is not finite in fp16, sets
// *redo_all so that every unit is recomputed from the fp32 query.
template <typename IT>
__global__ void rope_query_kernel(const IT* __restrict__ q, int B, int Tq, int hq, int d,
                                  int64_t q_pos0, int use_rope, RopeFreqs f, float qscale,
                                  float* __restrict__ qr, __half* __restrict__ q16, int32_t* redo_all) {
  bool bad = false;
  const int half = d / 2;
  const int64_t n = (int64_t)B * Tq * hq * half;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(e % half);
    const int64_t row = e / half;                 // (b, t, h)
    const int t = (int)((row / hq) % Tq);
    const int64_t base = row * d;
    const float x1 = to_f32(q[base + m]), x2 = to_f32(q[base + m + half]);
    float y1 = x1, y2 = x2;
    if (use_rope) {
      double sn, cn;
      sincos((double)(q_pos0 + t) * f.omega[m], &sn, &cn);
      const float c = (float)cn, s = (float)sn;
      y1 = x1 * c - x2 * s;
      y2 = x2 * c + x1 * s;
    }
    const float z1 = y1 * qscale, z2 = y2 * qscale;
    qr[base + m] = z1;
    qr[base + m + half] = z2;
    if (q16 != nullptr) {
      q16[base + m] = __float2half_rn(z1);
      q16[base + m + half] = __float2half_rn(z2);
      bad |= !(fabsf(z1) <= 65504.f) || !(fabsf(z2) <= 65504.f);
    }
  }
  if (bad) atomicExch(redo_all, 1);
}

// fp32 partial attention of one (batch, unit, kv head, 128 query rows): the
// kernel of fp32 inputs, and the exact recomputation of bf16 units flagged
// by the tensor-core query kernel (`redo` non-null: only CTAs whose unit is
// flagged, or all when the query itself was flagged, do any work; bf16 keys
// widen exactly to fp32 and the query is the fp32 rotated one).
template <int D, typename VT>
__global__ void __launch_bounds__(256) phase2_simt_kernel(Phase2Args a, const int32_t* __restrict__ redo) {
  constexpr int BK = 32, HALF = D / 2, G4 = HALF / 4;
  __shared__ __align__(16) float ks[BK][D];
  __shared__ __align__(16) float vs[BK][D];
  const int units = phase2_units(a);
  const int b = blockIdx.x / units, u = blockIdx.x % units;
  const int kvh = blockIdx.y, g = a.hq / a.hkv;
  if (redo != nullptr && redo[(int64_t)blockIdx.x * a.hkv + kvh] == 0 &&
      redo[(int64_t)a.B * units * a.hkv] == 0)
    return;
  const int idx = blockIdx.z * 128 + (threadIdx.x >> 1);
  const int hf = threadIdx.x & 1;
  const bool active = idx < a.Tq * g;
  const int t = active ? idx / g : 0, head = kvh * g + (active ? idx % g : 0);
  const UnitView uv = phase2_unit(a, u);
  const int64_t k0 = uv.k0, k1 = uv.k1;
  const int64_t lim = uv.causal_base < 0 ? INT64_MAX : uv.causal_base + t;   // last visible key
  const VT* K = static_cast<const VT*>(uv.K) + (int64_t)b * uv.stride_rows * a.hkv * D;
  const VT* V = static_cast<const VT*>(uv.V) + (int64_t)b * uv.stride_rows * a.hkv * D;
  float qv[HALF], acc[HALF];
  {
    const float* src = a.qr + (((int64_t)b * a.Tq + t) * a.hq + head) * D;
#pragma unroll
    for (int gg = 0; gg < G4; ++gg)
#pragma unroll
      for (int e = 0; e < 4; ++e) qv[4 * gg + e] = active ? src[8 * gg + 4 * hf + e] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < HALF; ++i) acc[i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  for (int64_t c0 = k0; c0 < k1; c0 += BK) {
    __syncthreads();
    for (int id = threadIdx.x; id < BK * D; id += 256) {
      const int kk = id / D, mm = id % D;
      const int64_t c = c0 + kk;
      float kx = 0.f, vx = 0.f;
      if (c < k1) {
        const int64_t off = (c * a.hkv + kvh) * (int64_t)D + mm;
        kx = to_f32(K[off]);
        vx = to_f32(V[off]);
      }
      ks[kk][mm] = kx;
      vs[kk][mm] = vx;
    }
    __syncthreads();
    float s[BK];
    float mt = m_run;
#pragma unroll
    for (int j = 0; j < BK; ++j) {
      float acc_s = 0.f;
#pragma unroll
      for (int gg = 0; gg < G4; ++gg) {
        const float4 kk4 = *reinterpret_cast<const float4*>(&ks[j][8 * gg + 4 * hf]);
        acc_s = fmaf(qv[4 * gg + 0], kk4.x, acc_s);
        acc_s = fmaf(qv[4 * gg + 1], kk4.y, acc_s);
        acc_s = fmaf(qv[4 * gg + 2], kk4.z, acc_s);
        acc_s = fmaf(qv[4 * gg + 3], kk4.w, acc_s);
      }
      acc_s += __shfl_xor_sync(0xffffffffu, acc_s, 1);
      s[j] = (c0 + j < k1 && c0 + j <= lim) ? acc_s : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    if (mt == -INFINITY) continue;   // every key of this tile is masked for this row
    const float alpha = fast_exp2(m_run - mt);
    l_run *= alpha;
#pragma unroll
    for (int i = 0; i < HALF; ++i) acc[i] *= alpha;
#pragma unroll
    for (int j = 0; j < BK; ++j) {
      const float pj = fast_exp2(s[j] - mt);
      l_run += pj;
#pragma unroll
      for (int gg = 0; gg < G4; ++gg) {
        const float4 vv4 = *reinterpret_cast<const float4*>(&vs[j][8 * gg + 4 * hf]);
        acc[4 * gg + 0] = fmaf(pj, vv4.x, acc[4 * gg + 0]);
        acc[4 * gg + 1] = fmaf(pj, vv4.y, acc[4 * gg + 1]);
        acc[4 * gg + 2] = fmaf(pj, vv4.z, acc[4 * gg + 2]);
        acc[4 * gg + 3] = fmaf(pj, vv4.w, acc[4 * gg + 3]);
      }
    }
    m_run = mt;
  }
  if (!active) return;
  const int64_t orow = (((int64_t)b * units + u) * a.Tq + t) * a.hq + head;
  float* dst = a.unit_o + orow * D;
  const bool empty = (m_run == -INFINITY);
  const float inv = empty ? 0.f : 1.f / l_run;
#pragma unroll
  for (int gg = 0; gg < G4; ++gg)
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[8 * gg + 4 * hf + e] = acc[4 * gg + e] * inv;
  if (hf == 0) a.unit_lse[orow] = empty ? -INFINITY : (m_run + __log2f(l_run)) * kLn2f;
}

// One warp per (b, t, head) row: merge the unit partials (splits of shards,
// then the own cache) into the global result, and, when asked for, into the
// shard partials.  s = ln sum_h exp(s_h) ; O = sum_h exp(s_h - s) A_h.
// Pass 1: the row's log-sum-exp over every unit, lanes over units.  Pass 2:
// the weighted sum of the units' A, each lane holding D/32 consecutive
// elements, units unrolled so that their loads are in flight together.
template <typename OT, int D>
__global__ void merge_kernel(Phase2Args a) {
  constexpr int VPL = D / 32;   // 4 or 2 consecutive floats per lane
  const int lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)a.B * a.Tq * a.hq;
  const int units = phase2_units(a);
  const int64_t rs = (int64_t)a.Tq * a.hq;   // unit stride in rows
  for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < nrows;
       row += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t b = row / rs, th = row % rs;
    const float* lse_u = a.unit_lse + b * units * rs + th;    // unit u at lse_u[u * rs]
    const float* A_u = a.unit_o + (b * units * rs + th) * D + lane * VPL;
    // pass 1: row log-sum-exp
    float m = -INFINITY;
    for (int u = lane; u < units; u += 32) m = fmaxf(m, lse_u[(int64_t)u * rs]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    if (m != -INFINITY)
      for (int u = lane; u < units; u += 32) z += expf(lse_u[(int64_t)u * rs] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float s_all = (m == -INFINITY) ? -INFINITY : m + logf(z);
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
    // adds w * A_u; a unit of weight 0 (lse -inf) adds nothing, whatever its A
    auto add_unit = [&](float* dst, int u, float w) {
      const float* src = A_u + (int64_t)u * rs * D;
      const bool on = w > 0.f;
      if constexpr (VPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        dst[0] += on ? w * v.x : 0.f;
        dst[1] += on ? w * v.y : 0.f;
        dst[2] += on ? w * v.z : 0.f;
        dst[3] += on ? w * v.w : 0.f;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        dst[0] += on ? w * v.x : 0.f;
        dst[1] += on ? w * v.y : 0.f;
      }
    };
    if (s_all != -INFINITY) {
      if (a.part_o_opt == nullptr && a.part_lse_opt == nullptr) {
        // pass 2, no shard partials: one flat sum over every unit (an empty
        // unit has lse -inf, weight 0 and A = 0)
        int u = 0;
        for (; u + 4 <= units; u += 4) {
          float w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = expf(lse_u[(int64_t)(u + i) * rs] - s_all);
#pragma unroll
          for (int i = 0; i < 4; ++i) add_unit(acc, u + i, w[i]);
        }
        for (; u < units; ++u) add_unit(acc, u, expf(lse_u[(int64_t)u * rs] - s_all));
      }
    }
    if (a.part_o_opt != nullptr || a.part_lse_opt != nullptr) {
      // pass 2 with shard partials: shard by shard, then the own cache
      for (int sh = 0; sh < a.n_shards; ++sh) {
        const int u0 = sh * a.n_split;
        float sm = -INFINITY;
        for (int sp = 0; sp < a.n_split; ++sp) sm = fmaxf(sm, lse_u[(int64_t)(u0 + sp) * rs]);
        float sz = 0.f;
        if (sm != -INFINITY)
          for (int sp = 0; sp < a.n_split; ++sp) sz += expf(lse_u[(int64_t)(u0 + sp) * rs] - sm);
        const float s_h = (sm == -INFINITY) ? -INFINITY : sm + logf(sz);
        float hacc[VPL];
#pragma unroll
        for (int e = 0; e < VPL; ++e) hacc[e] = 0.f;
        if (s_h != -INFINITY)
          for (int sp = 0; sp < a.n_split; ++sp)
            add_unit(hacc, u0 + sp, expf(lse_u[(int64_t)(u0 + sp) * rs] - s_h));
        const int64_t prow = (b * a.n_shards + sh) * rs + th;
        if (a.part_o_opt != nullptr) {
#pragma unroll
          for (int e = 0; e < VPL; ++e) a.part_o_opt[prow * D + lane * VPL + e] = hacc[e];
        }
        if (a.part_lse_opt != nullptr && lane == 0) a.part_lse_opt[prow] = s_h;
        if (s_h != -INFINITY && s_all != -INFINITY) {
          const float w = expf(s_h - s_all);
#pragma unroll
          for (int e = 0; e < VPL; ++e) acc[e] += w * hacc[e];
        }
      }
      if (a.has_self && s_all != -INFINITY)
        add_unit(acc, units - 1, expf(lse_u[(int64_t)(units - 1) * rs] - s_all));
    }
    OT* O = static_cast<OT*>(a.o) + row * D + lane * VPL;
#pragma unroll
    for (int e = 0; e < VPL; ++e) O[e] = from_f32<OT>(acc[e]);
    if (lane == 0) a.lse[row] = s_all;
  }
}

template <typename OT>
static void launch_merge_kernel(const Phase2Args& a, cudaStream_t s) {
  const int64_t nrows = (int64_t)a.B * a.Tq * a.hq;
  if (nrows <= 0) return;
  const int64_t want = (nrows * 32 + 255) / 256;
  const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
  if (a.d == 128) merge_kernel<OT, 128><<<grid, 256, 0, s>>>(a);
  else merge_kernel<OT, 64><<<grid, 256, 0, s>>>(a);
}

// Splits per shard so that small batches still fill the GPU.  Independent of
// the dtype, so that the workspace size does not depend on it.
//  - Few rows per kv head (decode, <= 8): work units are (batch, shard split,
//    kv head), one CTA per SM; pick the split count w that minimises
//    waves x (fixed cost + keys per split), waves = ceil(units x w / 148),
//    the fixed cost of a unit taken as 140 keys' streaming, with at least 512
//    keys per split.
//  - Many rows: units are (batch, shard split, kv head, 256 query rows), one
//    CTA per SM, keys in tiles of 128; pick the split count w that minimises
//    waves x (fixed cost + tiles per split), waves = ceil(units x w / 148),
//    the fixed cost of a unit (prologue, first tiles in flight, epilogue)
//    taken as 7 tiles' work, with at least 512 keys per split.
int32_t phase2_split(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                     int32_t hkv) {
  const int g = hq / hkv;
  const int64_t R = (int64_t)Tq * g;
  const int64_t shard_len = (T + n_shards - 1) / n_shards;
  int64_t cap = shard_len / 512;
  if (cap > 64) cap = 64;
  if (cap < 1) cap = 1;
  if (R <= 8) {
    const int64_t base = (int64_t)B * n_shards * hkv;
    if (base <= 0) return 1;
    int64_t best = 1, best_cost = 0;
    for (int64_t w = 1; w <= cap; ++w) {
      const int64_t waves = (base * w + 147) / 148;
      const int64_t cost = waves * (140 + (shard_len + w - 1) / w);
      if (w == 1 || cost < best_cost) {
        best = w;
        best_cost = cost;
      }
    }
    return (int32_t)best;
  }
  const int64_t base = (int64_t)B * n_shards * hkv * ((R + 255) / 256);
  if (base <= 0) return 1;
  int64_t best = 1, best_cost = 0;
  for (int64_t w = 1; w <= cap; ++w) {
    const int64_t waves = (base * w + 147) / 148;
    const int64_t tiles = (shard_len + w * 128 - 1) / (w * 128);
    const int64_t cost = waves * (7 + tiles);
    if (w == 1 || cost < best_cost) {
      best = w;
      best_cost = cost;
    }
  }
  return (int32_t)best;
}

// Work units of the context: by shard (a shard cut into phase2_split
// splits), or -- no per-shard partials asked for, and either a many-row
// query or a decode whose per-shard units would not fill the SMs -- the
// whole cache as one range cut into equal units, so that units need not
// follow shard boundaries (the exact merge does not depend on where the
// units are cut).  Measured on one B200: the 128K 64-token query 0.175 ->
// 0.163 ms, a 1-token step over 128K keys 0.122 -> 0.110 ms; batched
// decodes that already fill the SMs keep their shards.
bool phase2_flat_units(int32_t B, int32_t Tq, int32_t n_shards, int32_t hq, int32_t hkv, bool want_partials) {
  if (want_partials) return false;
  return (int64_t)Tq * (hq / hkv) > 8 || (int64_t)B * n_shards * hkv < 148;
}

size_t phase2_workspace_bytes(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                              int32_t hkv, int32_t d) {
  const int32_t ns = phase2_split(B, Tq, T, n_shards, hq, hkv);
  const int32_t ns_flat = phase2_split(B, Tq, T, 1, hq, hkv);
  size_t units = (size_t)n_shards * ns;
  if ((size_t)ns_flat > units) units = ns_flat;
  units += 1;                                       // + the query host's own cache
  const size_t rows = (size_t)B * Tq * hq;
  size_t b = kStatusBytes;
  b += align_up(sizeof(float) * rows * d);          // rotated query
  b += align_up(sizeof(float) * rows * units * d);  // unit partial outputs
  b += align_up(sizeof(float) * rows * units);      // unit partial lse
  b += align_up(sizeof(__half) * rows * d);         // fp16 query (tensor-core path)
  b += align_up(sizeof(int32_t) * ((size_t)B * units * hkv + 1));   // redo flags
  return b;
}

template <typename IT>
static int launch_phase2_t(const Phase2Args& a, cudaStream_t s) {
  RopeFreqs f;
  for (int m = 0; m < kMaxHalfDim; ++m)
    f.omega[m] = (m < a.d / 2 && a.rope_theta > 0) ? pow(a.rope_theta, -2.0 * m / a.d) : 0.0;
  const float qscale = (float)(kLog2e / sqrt((double)a.d));
  const int64_t nq = (int64_t)a.B * a.Tq * a.hq * (a.d / 2);
  // the tensor-core query kernel reads the query in fp16; units it cannot
  // carry in fp16 (a key, or the query, outside fp16 range) are flagged and
  // recomputed in fp32 by phase2_simt_kernel afterwards
  const bool tc = phase2_tc_supported(a);
  const int units = phase2_units(a);
  const size_t n_flags = (size_t)a.B * units * a.hkv + 1;
  if (tc && cudaMemsetAsync(a.redo, 0, sizeof(int32_t) * n_flags, s) != cudaSuccess) return PA_ERR_CUDA;
  if (nq > 0) {
    const int64_t want = (nq + 255) / 256;
    rope_query_kernel<IT><<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
        static_cast<const IT*>(a.q), a.B, a.Tq, a.hq, a.d, a.q_pos0, a.rope_theta > 0, f, qscale,
        a.qr, tc ? a.q16 : nullptr, a.redo + (n_flags - 1));
  }
  const int g = a.hq / a.hkv;
  const dim3 grid((unsigned)(a.B * units), a.hkv, (unsigned)((a.Tq * g + 127) / 128));
  int rc = PA_OK;
  profile_begin(s);
  if (tc) {
    rc = launch_phase2_tc(a, a.q16, s);
  } else if (a.dtype == PA_BF16) {
    rc = launch_phase2_mma(a, s);
  } else if (grid.x > 0 && grid.z > 0) {
    if (a.d == 128) phase2_simt_kernel<128, IT><<<grid, 256, 0, s>>>(a, nullptr);
    else phase2_simt_kernel<64, IT><<<grid, 256, 0, s>>>(a, nullptr);
  }
  profile_end(s);
  if (rc != PA_OK) return rc;
  if (tc && grid.x > 0 && grid.z > 0) {   // exact recomputation of the flagged units (usually none)
    if (a.d == 128) phase2_simt_kernel<128, IT><<<grid, 256, 0, s>>>(a, a.redo);
    else phase2_simt_kernel<64, IT><<<grid, 256, 0, s>>>(a, a.redo);
  }
  launch_merge_kernel<IT>(a, s);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Own-cache append: K of the new token j is rotated at q_pos0 + j and written
// with its V at row self_len + j of the query host's cache.
template <typename IT>
__global__ void self_append_kernel(const IT* __restrict__ k_new, const IT* __restrict__ v_new, int B,
                                   int Tq, int hkv, int d, int64_t q_pos0, int use_rope, RopeFreqs f,
                                   IT* __restrict__ k_self, IT* __restrict__ v_self, int64_t self_cap,
                                   int64_t self_len) {
  const int half = d / 2;
  const int64_t n = (int64_t)B * Tq * hkv * half;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(e % half);
    const int64_t row = e / half;               // (b, t, h)
    const int h = (int)(row % hkv);
    const int t = (int)((row / hkv) % Tq);
    const int64_t b = row / ((int64_t)hkv * Tq);
    const int64_t src = row * d;
    const int64_t dst = ((b * self_cap + self_len + t) * hkv + h) * (int64_t)d;
    const float x1 = to_f32(k_new[src + m]), x2 = to_f32(k_new[src + m + half]);
    float y1 = x1, y2 = x2;
    if (use_rope) {
      double sn, cn;
      sincos((double)(q_pos0 + t) * f.omega[m], &sn, &cn);
      const float c = (float)cn, sv = (float)sn;
      y1 = x1 * c - x2 * sv;
      y2 = x2 * c + x1 * sv;
    }
    k_self[dst + m] = from_f32<IT>(y1);
    k_self[dst + m + half] = from_f32<IT>(y2);
    v_self[dst + m] = v_new[src + m];
    v_self[dst + m + half] = v_new[src + m + half];
  }
}

template <typename IT>
static int launch_self_append_t(const Phase2Args& a, const void* k_new, const void* v_new, cudaStream_t s) {
  RopeFreqs f;
  for (int m = 0; m < kMaxHalfDim; ++m)
    f.omega[m] = (m < a.d / 2 && a.rope_theta > 0) ? pow(a.rope_theta, -2.0 * m / a.d) : 0.0;
  const int64_t n = (int64_t)a.B * a.Tq * a.hkv * (a.d / 2);
  if (n > 0) {
    const int64_t want = (n + 255) / 256;
    self_append_kernel<IT><<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
        static_cast<const IT*>(k_new), static_cast<const IT*>(v_new), a.B, a.Tq, a.hkv, a.d, a.q_pos0,
        a.rope_theta > 0, f, static_cast<IT*>(const_cast<void*>(a.k_self)),
        static_cast<IT*>(const_cast<void*>(a.v_self)), a.self_cap, a.self_len);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_self_append(const Phase2Args& a, const void* k_new, const void* v_new, cudaStream_t s) {
  if (a.dtype == PA_F32) return launch_self_append_t<float>(a, k_new, v_new, s);
  return launch_self_append_t<__nv_bfloat16>(a, k_new, v_new, s);
}

int launch_rope_query(const Phase2Args& a, cudaStream_t s) {
  RopeFreqs f;
  for (int m = 0; m < kMaxHalfDim; ++m)
    f.omega[m] = (m < a.d / 2 && a.rope_theta > 0) ? pow(a.rope_theta, -2.0 * m / a.d) : 0.0;
  const float qscale = (float)(kLog2e / sqrt((double)a.d));
  const int64_t nq = (int64_t)a.B * a.Tq * a.hq * (a.d / 2);
  if (nq > 0) {
    const int64_t want = (nq + 255) / 256;
    if (a.dtype == PA_F32)
      rope_query_kernel<float><<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
          static_cast<const float*>(a.q), a.B, a.Tq, a.hq, a.d, a.q_pos0, a.rope_theta > 0, f, qscale, a.qr,
          nullptr, nullptr);
    else
      rope_query_kernel<__nv_bfloat16><<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.q), a.B, a.Tq, a.hq, a.d, a.q_pos0, a.rope_theta > 0, f, qscale,
          a.qr, nullptr, nullptr);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_merge_only(const Phase2Args& a, cudaStream_t s) {
  if (a.dtype == PA_F32) launch_merge_kernel<float>(a, s);
  else launch_merge_kernel<__nv_bfloat16>(a, s);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_phase2(const Phase2Args& a, cudaStream_t s) {
  if (a.dtype == PA_F32) return launch_phase2_t<float>(a, s);
  return launch_phase2_t<__nv_bfloat16>(a, s);
}

}  // namespace pa
