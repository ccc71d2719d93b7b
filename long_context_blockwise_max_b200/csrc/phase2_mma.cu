// Phase-2 split-KV partial attention for bf16 caches on warp-level tensor-core
// MMAs (mma.sync m16n8k16), the HBM-streaming path of the query phase
// (Pulsar Attention page §2.2; Star Attention review, key_machinery).
//
// Work unit = (batch b, kv head, shard split u, group of 8 query rows).  The
// 8 real rows of a unit (token t, query head of the GQA group) fill MMA rows
// 0-7 with the bf16 "high" part of the rotated query and rows 8-15 with the
// bf16 residual ("low" part): one MMA then yields both halves of every score
// in the same thread (accumulator rows r and r + 8), and s = s_hi + s_lo is
// the fp32-accurate q.k against the stored bf16 key at no extra MMA cost.
//
// Each of the 4 warps owns every 4th tile of 32 keys of the unit's range and
// streams it through its own 3-stage cp.async ring (16-byte copies, 128-byte
// XOR swizzle so that ldmatrix is conflict-free).  Warp partials are merged
// in shared memory at the end (same log-sum-exp algebra as the shard merge)
// and written as the unit's normalised partial (A, lse).
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kWarps = 4;
constexpr int kKT = 32;      // keys per warp tile
constexpr int kStages = 3;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0: fill the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D>
struct P2Cfg {
  static constexpr int CH = D / 8;                    // 16-byte chunks per key row
  static constexpr int ROWB = D * 2;
  static constexpr int TILE = kKT * ROWB;             // K (or V) tile bytes
  static constexpr int STAGE = 2 * TILE;              // K + V
  static constexpr int WARP_BYTES = kStages * STAGE;
  static constexpr int SMEM = kWarps * WARP_BYTES;
};

// byte offset of (key row, 16-byte chunk) inside a swizzled tile
template <int D>
__device__ __forceinline__ uint32_t swz(int key, int chunk) {
  return key * P2Cfg<D>::ROWB + ((chunk ^ (key & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) phase2_mma_kernel(Phase2Args a, int row_groups) {
  using C = P2Cfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = phase2_units(a);
  const int rg = blockIdx.x % row_groups;
  const int bu = blockIdx.x / row_groups;
  const int b = bu / units, u = bu % units;
  const int kvh = blockIdx.y;
  const int g = a.hq / a.hkv;
  const int R = a.Tq * g;

  const UnitView uv = phase2_unit(a, u);
  const int64_t k0 = uv.k0, k1 = uv.k1;

  // ---- query fragments: rows 0-7 high part, rows 8-15 residual ----------
  const int qi = lane >> 2;            // real row of this thread (0..7)
  const int qc = (lane & 3) * 2;       // column pair inside an 8-wide block
  const int rr = rg * 8 + qi;          // real row index in [0, R)
  const bool row_ok = rr < R;
  const int t_row = row_ok ? rr / g : 0;
  const int head = kvh * g + (row_ok ? rr % g : 0);
  uint32_t qa[D / 16][4];
  {
    const float* qp = a.qr + (((int64_t)b * a.Tq + t_row) * a.hq + head) * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      float x[4];
      x[0] = row_ok ? qp[16 * ks + qc] : 0.f;
      x[1] = row_ok ? qp[16 * ks + qc + 1] : 0.f;
      x[2] = row_ok ? qp[16 * ks + qc + 8] : 0.f;
      x[3] = row_ok ? qp[16 * ks + qc + 9] : 0.f;
      float h[4], l[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        h[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
        l[e] = x[e] - h[e];
      }
      qa[ks][0] = pack_bf16(h[0], h[1]);   // row qi,   k = qc, qc+1
      qa[ks][1] = pack_bf16(l[0], l[1]);   // row qi+8
      qa[ks][2] = pack_bf16(h[2], h[3]);   // row qi,   k = qc+8, qc+9
      qa[ks][3] = pack_bf16(l[2], l[3]);   // row qi+8
    }
  }

  // ---- this warp's key tiles: kt = warp, warp + 4, ... ------------------
  const int64_t n_tiles = (k1 - k0 + kKT - 1) / kKT;
  const int my_tiles = n_tiles > warp ? (int)((n_tiles - 1 - warp) / kWarps + 1) : 0;
  const uint32_t wbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem)) + warp * C::WARP_BYTES;
  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(uv.K);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(uv.V);
  const int64_t key_stride = (int64_t)a.hkv * D;   // elements between consecutive keys
  const int64_t base_off = ((int64_t)b * uv.stride_rows) * key_stride + (int64_t)kvh * D;
  const int64_t lim = uv.causal_base < 0 ? INT64_MAX : uv.causal_base + t_row;   // last visible key

  auto issue = [&](int it) {
    if (it < my_tiles) {
      const int64_t key0 = k0 + (int64_t)(warp + it * kWarps) * kKT;
      const uint32_t sbase = wbase + (it % kStages) * C::STAGE;
#pragma unroll
      for (int e = 0; e < (kKT * C::CH) / 32; ++e) {
        const int idx = e * 32 + lane;
        const int key = idx / C::CH, ch = idx % C::CH;
        const int64_t kg = key0 + key;
        const bool valid = kg < k1;
        const int64_t off = base_off + (valid ? kg : k0) * key_stride + ch * 8;
        cp_async16(sbase + swz<D>(key, ch), Kg + off, valid);
        cp_async16(sbase + C::TILE + swz<D>(key, ch), Vg + off, valid);
      }
    }
    cp_async_commit();
  };

  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) issue(s);
  for (int it = 0; it < my_tiles; ++it) {
    issue(it + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint32_t sK = wbase + (it % kStages) * C::STAGE;
    const uint32_t sV = sK + C::TILE;
    const int64_t key0 = k0 + (int64_t)(warp + it * kWarps) * kKT;
    // S = Q K^T over 32 keys: 4 n8 tiles
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        uint32_t b0, b1, b2, b3;
        const int key = nt * 8 + (lane & 7);
        const int ch = kk * 4 + (lane >> 3);
        ldsm_x4(sK + swz<D>(key, ch), b0, b1, b2, b3);
        mma_bf16(s[nt], qa[2 * kk][0], qa[2 * kk][1], qa[2 * kk][2], qa[2 * kk][3], b0, b1);
        mma_bf16(s[nt], qa[2 * kk + 1][0], qa[2 * kk + 1][1], qa[2 * kk + 1][2], qa[2 * kk + 1][3], b2, b3);
      }
    }
    // combine high + residual rows, mask the ragged end, online softmax
    float sv[4][2];
    float mt = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t kg = key0 + nt * 8 + qc + e;
        const float x = (kg < k1 && kg <= lim) ? s[nt][e] + s[nt][e + 2] : -INFINITY;
        sv[nt][e] = x;
        mt = fmaxf(mt, x);
      }
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float m_new = fmaxf(m_run, mt);
    const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
    const float m_sub = (m_new == -INFINITY) ? 0.f : m_new;   // rows that see no key yet
    m_run = m_new;
    l_run *= alpha;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }
    uint32_t pa_[4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = fast_exp2(sv[nt][0] - m_sub), p1 = fast_exp2(sv[nt][1] - m_sub);
      l_run += p0 + p1;
      pa_[nt] = pack_bf16(p0, p1);
    }
    // O += P V over 32 keys: 2 k16 steps x D/8 n8 tiles
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
      for (int cj = 0; cj < D / 16; ++cj) {
        uint32_t b0, b1, b2, b3;
        const int mtx = lane >> 3;
        const int key = k2 * 16 + (mtx & 1) * 8 + (lane & 7);
        const int ch = cj * 2 + (mtx >> 1);
        ldsm_x4_t(sV + swz<D>(key, ch), b0, b1, b2, b3);
        mma_bf16(o[2 * cj], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b0, b1);
        mma_bf16(o[2 * cj + 1], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b2, b3);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the 4 warp partials (rows qi of each warp) -----------------
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  float* red = reinterpret_cast<float*>(smem);              // [warp][8 rows][D]
  float* red_m = red + kWarps * 8 * D;                      // [warp][8]
  float* red_l = red_m + kWarps * 8;                        // [warp][8]
#pragma unroll
  for (int j = 0; j < D / 8; ++j) {
    red[(warp * 8 + qi) * D + 8 * j + qc] = o[j][0];
    red[(warp * 8 + qi) * D + 8 * j + qc + 1] = o[j][1];
  }
  if ((lane & 3) == 0) {
    red_m[warp * 8 + qi] = m_run;
    red_l[warp * 8 + qi] = l_run;
  }
  __syncthreads();
  // thread -> (row, 8-wide column chunk): 8 rows x D/8 chunks <= 128 threads
  const int row = threadIdx.x / (D / 8), cch = threadIdx.x % (D / 8);
  if (row < 8) {
    const int rr2 = rg * 8 + row;
    if (rr2 < R) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * 8 + row]);
      float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float mw = red_m[w * 8 + row];
          if (mw == -INFINITY) continue;
          const float c = fast_exp2(mw - M);
          L += c * red_l[w * 8 + row];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += c * red[(w * 8 + row) * D + 8 * cch + e];
        }
      }
      const int t2 = rr2 / g, h2 = kvh * g + rr2 % g;
      const int64_t orow = (((int64_t)b * units + u) * a.Tq + t2) * a.hq + h2;
      const float inv = (M == -INFINITY) ? 0.f : 1.f / L;
      float4* dst = reinterpret_cast<float4*>(a.unit_o + orow * D + 8 * cch);
      dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      if (cch == 0) a.unit_lse[orow] = (M == -INFINITY) ? -INFINITY : (M + __log2f(L)) * kLn2f;
    }
  }
}

// Variant for many query rows per kv head (a multi-token query): the four
// warps own four different groups of 8 rows and share every K / V tile,
// which the whole CTA streams through one 3-stage cp.async ring, so a
// unit's keys are read once per 32 rows instead of once per 8 rows.
template <int D>
__global__ void __launch_bounds__(kWarps * 32) phase2_mma_rows_kernel(Phase2Args a, int row_blocks) {
  using C = P2Cfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = phase2_units(a);
  const int rb = blockIdx.x % row_blocks;
  const int bu = blockIdx.x / row_blocks;
  const int b = bu / units, u = bu % units;
  const int kvh = blockIdx.y;
  const int g = a.hq / a.hkv;
  const int R = a.Tq * g;
  const int rg = rb * kWarps + warp;   // this warp's group of 8 rows

  const UnitView uv = phase2_unit(a, u);
  const int64_t k0 = uv.k0, k1 = uv.k1;
  const int qi = lane >> 2, qc = (lane & 3) * 2;
  const int rr = rg * 8 + qi;
  const bool row_ok = rr < R;
  const int t_row = row_ok ? rr / g : 0;
  const int head = kvh * g + (row_ok ? rr % g : 0);
  uint32_t qa[D / 16][4];
  {
    const float* qp = a.qr + (((int64_t)b * a.Tq + t_row) * a.hq + head) * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      float x[4];
      x[0] = row_ok ? qp[16 * ks + qc] : 0.f;
      x[1] = row_ok ? qp[16 * ks + qc + 1] : 0.f;
      x[2] = row_ok ? qp[16 * ks + qc + 8] : 0.f;
      x[3] = row_ok ? qp[16 * ks + qc + 9] : 0.f;
      float h[4], l[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        h[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
        l[e] = x[e] - h[e];
      }
      qa[ks][0] = pack_bf16(h[0], h[1]);
      qa[ks][1] = pack_bf16(l[0], l[1]);
      qa[ks][2] = pack_bf16(h[2], h[3]);
      qa[ks][3] = pack_bf16(l[2], l[3]);
    }
  }
  const int n_tiles = static_cast<int>((k1 - k0 + kKT - 1) / kKT);
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(uv.K);
  const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(uv.V);
  const int64_t key_stride = (int64_t)a.hkv * D;
  const int64_t base_off = ((int64_t)b * uv.stride_rows) * key_stride + (int64_t)kvh * D;
  const int64_t lim = uv.causal_base < 0 ? INT64_MAX : uv.causal_base + t_row;   // last visible key
  auto issue = [&](int it) {
    if (it < n_tiles) {
      const int64_t key0 = k0 + (int64_t)it * kKT;
      const uint32_t sbase = base + (it % kStages) * C::STAGE;
#pragma unroll
      for (int e = 0; e < (kKT * C::CH) / (kWarps * 32); ++e) {
        const int idx = e * kWarps * 32 + threadIdx.x;
        const int key = idx / C::CH, ch = idx % C::CH;
        const int64_t kg = key0 + key;
        const bool valid = kg < k1;
        const int64_t off = base_off + (valid ? kg : k0) * key_stride + ch * 8;
        cp_async16(sbase + swz<D>(key, ch), Kg + off, valid);
        cp_async16(sbase + C::TILE + swz<D>(key, ch), Vg + off, valid);
      }
    }
    cp_async_commit();
  };
  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) issue(s);
  for (int it = 0; it < n_tiles; ++it) {
    issue(it + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const uint32_t sK = base + (it % kStages) * C::STAGE;
    const uint32_t sV = sK + C::TILE;
    const int64_t key0 = k0 + (int64_t)it * kKT;
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        uint32_t b0, b1, b2, b3;
        const int key = nt * 8 + (lane & 7);
        const int ch = kk * 4 + (lane >> 3);
        ldsm_x4(sK + swz<D>(key, ch), b0, b1, b2, b3);
        mma_bf16(s[nt], qa[2 * kk][0], qa[2 * kk][1], qa[2 * kk][2], qa[2 * kk][3], b0, b1);
        mma_bf16(s[nt], qa[2 * kk + 1][0], qa[2 * kk + 1][1], qa[2 * kk + 1][2], qa[2 * kk + 1][3], b2, b3);
      }
    }
    float sv[4][2];
    float mt = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t kg = key0 + nt * 8 + qc + e;
        const float x = (kg < k1 && kg <= lim) ? s[nt][e] + s[nt][e + 2] : -INFINITY;
        sv[nt][e] = x;
        mt = fmaxf(mt, x);
      }
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float m_new = fmaxf(m_run, mt);
    const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
    const float m_sub = (m_new == -INFINITY) ? 0.f : m_new;   // rows that see no key yet
    m_run = m_new;
    l_run *= alpha;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }
    uint32_t pa_[4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = fast_exp2(sv[nt][0] - m_sub), p1 = fast_exp2(sv[nt][1] - m_sub);
      l_run += p0 + p1;
      pa_[nt] = pack_bf16(p0, p1);
    }
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
      for (int cj = 0; cj < D / 16; ++cj) {
        uint32_t b0, b1, b2, b3;
        const int mtx = lane >> 3;
        const int key = k2 * 16 + (mtx & 1) * 8 + (lane & 7);
        const int ch = cj * 2 + (mtx >> 1);
        ldsm_x4_t(sV + swz<D>(key, ch), b0, b1, b2, b3);
        mma_bf16(o[2 * cj], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b0, b1);
        mma_bf16(o[2 * cj + 1], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b2, b3);
      }
    }
    __syncthreads();   // the stage is refilled by the next issue
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (!row_ok) return;
  const int64_t orow = (((int64_t)b * units + u) * a.Tq + t_row) * a.hq + head;
  const bool empty = (m_run == -INFINITY);
  const float inv = empty ? 0.f : 1.f / l_run;
  float* dst = a.unit_o + orow * D;
#pragma unroll
  for (int j = 0; j < D / 8; ++j)
    *reinterpret_cast<float2*>(dst + 8 * j + qc) = make_float2(o[j][0] * inv, o[j][1] * inv);
  if ((lane & 3) == 0) a.unit_lse[orow] = empty ? -INFINITY : (m_run + __log2f(l_run)) * kLn2f;
}

// ---------------------------------------------------------------------------
// ART (run-time early termination, ART review page): the cache of each
// (batch, kv head) is walked from the newest key backwards in blocks of
// `block_keys` keys; after every block the normalised running output of
// each query row is compared with the previous block's (magnitude change
// <= tau * |x_prev|, 1 - cos <= phi), and the walk stops once `patience`
// consecutive blocks were stable for every row.
//
// CTA = one (batch, kv head), 5 warps.  Warps 0-3 compute, in rounds of four
// blocks, the partial (m, l, A) of one block each (32-key tiles through a
// private 3-stage cp.async ring, hi/lo query MMAs as in the decode kernel)
// into a double-buffered shared-memory slot.  Warp 4 folds the partials into
// the running result in block order (the exact log-sum-exp merge) and runs
// the stability test after each block, while the compute warps work on the
// next round.  A stop discards the rest of the round and the round computed
// ahead; the result is attention over the blocks folded.
// ---------------------------------------------------------------------------
constexpr int kArtWarps = 4;       // compute warps
constexpr int kArtStages = 3;      // cp.async stages per compute warp

template <int D>
struct ArtCfg {
  static constexpr int RING = kArtStages * P2Cfg<D>::STAGE;        // per compute warp
  static constexpr int OFF_PART = kArtWarps * RING;
  static constexpr int PART_O = 8 * D;                             // floats per warp slot
  static constexpr int PART = PART_O + 16;                         // + m[8], l[8]
  static constexpr int SMEM = OFF_PART + 2 * kArtWarps * PART * 4 + 16;
};

template <int D>
__global__ void __launch_bounds__((kArtWarps + 1) * 32) phase2_art_kernel(Phase2Args a, ArtArgs art) {
  using C = P2Cfg<D>;
  using AC = ArtCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x, kvh = blockIdx.y;
  const int g = a.hq / a.hkv;
  const int R = a.Tq * g;
  const int qi = lane >> 2, qc = (lane & 3) * 2;
  const bool row_ok = qi < R;
  const int64_t T = a.T;
  const int n_tiles = static_cast<int>((T + kKT - 1) / kKT);
  const int tpb = art.block_keys / kKT;                       // tiles per block
  const int n_blocks = (n_tiles + tpb - 1) / tpb;
  const int n_rounds = (n_blocks + kArtWarps - 1) / kArtWarps;
  float* part = reinterpret_cast<float*>(smem + AC::OFF_PART);  // [2][warp][PART]
  // round in which the folder decided to stop (n_rounds: not yet).  Every
  // warp runs the same barriers: one per round, after the round's partials
  // are published; after barrier r all warps leave the loop together when
  // the stop was decided in a round < r (written before that barrier, so
  // every warp sees it), and a value written during round r's fold never
  // passes the test in round r.
  volatile int* stop_round =
      reinterpret_cast<volatile int*>(smem + AC::OFF_PART + 2 * kArtWarps * AC::PART * 4);
  if (threadIdx.x == 0) *stop_round = n_rounds;
  __syncthreads();

  if (warp < kArtWarps) {
    // ------------------------------------------------------- compute warp
    const int t_row = row_ok ? qi / g : 0;
    const int head = kvh * g + (row_ok ? qi % g : 0);
    uint32_t qa[D / 16][4];
    {
      const float* qp = a.qr + (((int64_t)b * a.Tq + t_row) * a.hq + head) * D;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        float x[4];
        x[0] = row_ok ? qp[16 * ks + qc] : 0.f;
        x[1] = row_ok ? qp[16 * ks + qc + 1] : 0.f;
        x[2] = row_ok ? qp[16 * ks + qc + 8] : 0.f;
        x[3] = row_ok ? qp[16 * ks + qc + 9] : 0.f;
        float h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
          l[e] = x[e] - h[e];
        }
        qa[ks][0] = pack_bf16(h[0], h[1]);
        qa[ks][1] = pack_bf16(l[0], l[1]);
        qa[ks][2] = pack_bf16(h[2], h[3]);
        qa[ks][3] = pack_bf16(l[2], l[3]);
      }
    }
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem)) + warp * AC::RING;
    const __nv_bfloat16* Kg = static_cast<const __nv_bfloat16*>(a.k_ret);
    const __nv_bfloat16* Vg = static_cast<const __nv_bfloat16*>(a.v_ret);
    const int64_t key_stride = (int64_t)a.hkv * D;
    const int64_t base_off = ((int64_t)b * T) * key_stride + (int64_t)kvh * D;
    // this warp's k-th tile: tile (4 * (k / tpb) + warp) * tpb + k % tpb of
    // the walk; walk tile s covers keys [T - 32 (s + 1), T - 32 s), clipped at 0
    auto walk_tile = [&](int k) { return ((k / tpb) * kArtWarps + warp) * tpb + k % tpb; };
    auto issue = [&](int k) {
      const int it = walk_tile(k);
      if (k < n_rounds * tpb && it < n_tiles && ((k / tpb) * kArtWarps + warp) < n_blocks) {
        const int64_t key0 = T - (int64_t)kKT * (it + 1);
        const uint32_t sbase = base + (k % kArtStages) * C::STAGE;
#pragma unroll
        for (int e = 0; e < (kKT * C::CH) / 32; ++e) {
          const int idx = e * 32 + lane;
          const int key = idx / C::CH, ch = idx % C::CH;
          const int64_t kg = key0 + key;
          const bool valid = kg >= 0;
          const int64_t off = base_off + (valid ? kg : 0) * key_stride + ch * 8;
          cp_async16(sbase + swz<D>(key, ch), Kg + off, valid);
          cp_async16(sbase + C::TILE + swz<D>(key, ch), Vg + off, valid);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int s2 = 0; s2 < kArtStages - 1; ++s2) issue(s2);
    int k = 0;
    for (int r = 0; r < n_rounds; ++r) {
      const int blk = r * kArtWarps + warp;
      float o[D / 8][4];
#pragma unroll
      for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      float m_b = -INFINITY, l_b = 0.f;
      for (int t = 0; t < tpb; ++t, ++k) {
        issue(k + kArtStages - 1);
        cp_async_wait<kArtStages - 1>();
        __syncwarp();
        const int it = walk_tile(k);
        if (blk < n_blocks && it < n_tiles) {
          const uint32_t sK = base + (k % kArtStages) * C::STAGE;
          const uint32_t sV = sK + C::TILE;
          const int64_t key0 = T - (int64_t)kKT * (it + 1);
          float sc[4][4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
              uint32_t b0, b1, b2, b3;
              const int key = nt * 8 + (lane & 7);
              const int ch = kk * 4 + (lane >> 3);
              ldsm_x4(sK + swz<D>(key, ch), b0, b1, b2, b3);
              mma_bf16(sc[nt], qa[2 * kk][0], qa[2 * kk][1], qa[2 * kk][2], qa[2 * kk][3], b0, b1);
              mma_bf16(sc[nt], qa[2 * kk + 1][0], qa[2 * kk + 1][1], qa[2 * kk + 1][2], qa[2 * kk + 1][3], b2, b3);
            }
          }
          float sv[4][2];
          float mt = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int64_t kg = key0 + nt * 8 + qc + e;
              const float x = (kg >= 0) ? sc[nt][e] + sc[nt][e + 2] : -INFINITY;
              sv[nt][e] = x;
              mt = fmaxf(mt, x);
            }
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
          const float m_new = fmaxf(m_b, mt);
          const float alpha = fast_exp2(m_b - m_new);
          m_b = m_new;
          l_b *= alpha;
#pragma unroll
          for (int j = 0; j < D / 8; ++j) {
            o[j][0] *= alpha;
            o[j][1] *= alpha;
          }
          uint32_t pa_[4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const float p0 = fast_exp2(sv[nt][0] - m_new), p1 = fast_exp2(sv[nt][1] - m_new);
            l_b += p0 + p1;
            pa_[nt] = pack_bf16(p0, p1);
          }
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
            for (int cj = 0; cj < D / 16; ++cj) {
              uint32_t b0, b1, b2, b3;
              const int mtx = lane >> 3;
              const int key = k2 * 16 + (mtx & 1) * 8 + (lane & 7);
              const int ch = cj * 2 + (mtx >> 1);
              ldsm_x4_t(sV + swz<D>(key, ch), b0, b1, b2, b3);
              mma_bf16(o[2 * cj], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b0, b1);
              mma_bf16(o[2 * cj + 1], pa_[2 * k2], 0u, pa_[2 * k2 + 1], 0u, b2, b3);
            }
          }
        }
        __syncwarp();   // the stage is refilled by a later issue
      }
      // the block's partial (unnormalised A, m, l) into the round's slot
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      float* slot = part + ((r & 1) * kArtWarps + warp) * AC::PART;
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<float2*>(slot + qi * D + 8 * j + qc) = make_float2(o[j][0], o[j][1]);
      if ((lane & 3) == 0) {
        slot[AC::PART_O + qi] = m_b;
        slot[AC::PART_O + 8 + qi] = l_b;
      }
      __syncthreads();   // round r published; the folder takes it while this warp goes on
      if (*stop_round < r) break;
    }
    cp_async_wait<0>();
  } else {
    // ------------------------------------------------------------- folder
    float O[D / 8][2];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) O[j][0] = O[j][1] = 0.f;
    float prev[D / 8][2];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) prev[j][0] = prev[j][1] = 0.f;
    float prev_sq = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    int run = 0, blocks = 0;
    bool done = false;
    for (int r = 0; r < n_rounds; ++r) {
      __syncthreads();   // round r published
      if (*stop_round < r) break;
      for (int w = 0; w < kArtWarps && !done; ++w) {
        const int blk = r * kArtWarps + w;
        if (blk >= n_blocks) break;
        const float* slot = part + ((r & 1) * kArtWarps + w) * AC::PART;
        const float mb = slot[AC::PART_O + qi], lb = slot[AC::PART_O + 8 + qi];
        const float m_new = fmaxf(m_run, mb);
        const float ca = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        const float cb = (mb == -INFINITY) ? 0.f : fast_exp2(mb - m_new);
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const float2 v = *reinterpret_cast<const float2*>(slot + qi * D + 8 * j + qc);
          O[j][0] = O[j][0] * ca + v.x * cb;
          O[j][1] = O[j][1] * ca + v.y * cb;
        }
        l_run = l_run * ca + lb * cb;
        m_run = m_new;
        // stability of the normalised output after this block
        ++blocks;
        const float inv = 1.f / l_run;
        float sq = 0.f, dot = 0.f;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
          const float x0 = O[j][0] * inv, x1 = O[j][1] * inv;
          sq = fmaf(x0, x0, fmaf(x1, x1, sq));
          dot = fmaf(x0, prev[j][0], fmaf(x1, prev[j][1], dot));
          prev[j][0] = x0;
          prev[j][1] = x1;
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        bool stable = true;
        if (blocks >= 2 && row_ok) {
          const float nx = sqrtf(sq), np = sqrtf(prev_sq);
          stable = fabsf(nx - np) <= art.tau * np && 1.f - dot / (nx * np) <= art.phi;
        } else if (row_ok) {
          stable = false;
        }
        prev_sq = sq;
        run = __all_sync(0xffffffffu, stable) ? run + 1 : 0;
        if (run >= art.patience) done = true;
      }
      if (done) {
        if (lane == 0) *stop_round = r;
        __syncwarp();
      }
    }
    if (lane == 0 && art.visited) art.visited[(int64_t)b * a.hkv + kvh] = blocks;
    if (row_ok) {
      const int t_row = qi / g;
      const int head = kvh * g + qi % g;
      const bool empty = (m_run == -INFINITY) || !(l_run > 0.f);
      const float inv = empty ? 0.f : 1.f / l_run;
      const int64_t orow = ((int64_t)b * a.Tq + t_row) * a.hq + head;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.o) + orow * D;
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<__nv_bfloat162*>(dst + 8 * j + qc) = __floats2bfloat162_rn(O[j][0] * inv, O[j][1] * inv);
      if ((lane & 3) == 0) a.lse[orow] = empty ? -INFINITY : (m_run + __log2f(l_run)) * kLn2f;
    }
  }
}

template <int D>
int launch_d(const Phase2Args& a, cudaStream_t s) {
  const int g = a.hq / a.hkv;
  const int R = a.Tq * g;
  const int units = phase2_units(a);
  if (R <= 8) {
    // a few rows per kv head (decode): the 4 warps split the keys
    const int64_t gx = (int64_t)a.B * units;
    if (gx <= 0) return PA_OK;
    const int sm = P2Cfg<D>::SMEM;
    if (cudaFuncSetAttribute(phase2_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    phase2_mma_kernel<D><<<dim3(static_cast<unsigned>(gx), a.hkv), kWarps * 32, sm, s>>>(a, 1);
  } else {
    // many rows per kv head: the 4 warps split the rows and share K / V
    const int row_blocks = (R + 8 * kWarps - 1) / (8 * kWarps);
    const int64_t gx = (int64_t)a.B * units * row_blocks;
    if (gx <= 0) return PA_OK;
    const int sm = kStages * P2Cfg<D>::STAGE;
    if (cudaFuncSetAttribute(phase2_mma_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    phase2_mma_rows_kernel<D><<<dim3(static_cast<unsigned>(gx), a.hkv), kWarps * 32, sm, s>>>(a, row_blocks);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

int launch_phase2_mma(const Phase2Args& a, cudaStream_t s) {
  return a.d == 128 ? launch_d<128>(a, s) : launch_d<64>(a, s);
}

int launch_phase2_art(const Phase2Args& a, const ArtArgs& art, cudaStream_t s) {
  const dim3 grid(a.B, a.hkv);
  if (a.B <= 0) return PA_OK;
  if (a.d == 128) {
    const int sm = ArtCfg<128>::SMEM;
    if (cudaFuncSetAttribute(phase2_art_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    phase2_art_kernel<128><<<grid, (kArtWarps + 1) * 32, sm, s>>>(a, art);
  } else {
    const int sm = ArtCfg<64>::SMEM;
    if (cudaFuncSetAttribute(phase2_art_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    phase2_art_kernel<64><<<grid, (kArtWarps + 1) * 32, sm, s>>>(a, art);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
