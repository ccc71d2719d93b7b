// Phase-2 split-KV partial attention of a multi-token query on the sm_100a
// tensor cores (tcgen05 + TMEM + TMA): the query phase of the Pulsar
// Attention page (§2.2) and of the Star Attention review (key_machinery)
// when the query holds enough rows per kv head to make QK^T and PV dense
// contractions (a query of Tq tokens gives Tq x (hq / hkv) rows per kv head).
//
// CTA = one work unit (a split of one shard, or the query host's own cache)
// x one kv head x two 128-row tiles of that kv head's query rows (row
// r = token * g + head-in-group, g = hq / hkv).  Both tiles read every K / V
// tile of the unit, so the unit's keys cross HBM once per 256 rows.
//
// Operands.  The rotated query, scaled to log2 units, is stored as fp16
// (rounding error 2^-11 relative).  The cache is bf16; every K tile is
// converted to fp16 in shared memory after it lands (exact for |k| in fp16's
// normal range, which holds every bf16 value from 2^-14 to 65504), so that
// QK^T is one fp16 x fp16 tcgen05 MMA per k-step.  A rotated query or key
// outside fp16 range sets PA_ERR_RANGE.  PV is bf16 P x bf16 V.  Every
// tcgen05 MMA of M = 128 costs about the same time whatever its N here, so
// the kernel uses the widest tiles TMEM allows: 128 keys per QK^T.
//
// 12 warps:
//   warp 0      TMA producer: the two Q tiles once, then K tiles through a
//               3-stage ring and V tiles through a 2-stage ring (128 keys).
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (fp16, fp32 in TMEM)
//               and O_t += P_t V (P bf16 from TMEM, V bf16 MN-major); the two
//               row tiles ping-pong as in the Phase-1 kernel.
//   warps 2-3   K converters: bf16 -> fp16 in place, then a proxy fence so
//               that the tensor core sees the converted tile (warp 2 also
//               allocates TMEM: 512 columns, S0 | O0 | S1 | O1).
//   warps 4-11  softmax, one thread per row of tile 0 (warps 4-7) or tile 1
//               (warps 8-11); masks keys past the unit's end (and, for the
//               own cache, past the row's causal limit); lazy rescale of O.
// Output: the unit's normalised partial A and its lse per row, the same
// contract as the other Phase-2 kernels, merged by merge_kernel.
// Every wait is bounded (1 s by default); on expiry the CTA records
// PA_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "pa_internal.h"
#include "sm100.cuh"

namespace pa {
using namespace sm100;

namespace {

constexpr int kKT = 128;           // keys per tile
constexpr int kMaxStages = 4;
constexpr int kConvThreads = 64;   // warps 2-3

template <int D>
struct QtCfg {
  static constexpr int NKB = D / 64;                 // 128-byte column blocks along d
  static constexpr int KB_BYTES = 128 * 128;         // 128 rows x 128 B
  static constexpr int TILE = NKB * KB_BYTES;        // 128 rows x D x 2 B
  static constexpr int KST = D == 128 ? 3 : 4;       // K stages
  static constexpr int VST = D == 128 ? 2 : 4;       // V stages
  static constexpr int OFF_Q = 0;                    // [row tile]
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = OFF_K + KST * TILE;
  static constexpr int OFF_BAR = OFF_V + VST * TILE;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
  static constexpr uint32_t IDESC_QK = idesc_f16(128, kKT, 0, 0, 0, 0);   // f16 Q . f16 K
  static constexpr uint32_t IDESC_PV = idesc_f16(128, D, 1, 1, 0, 1);     // bf16 P . bf16 V (MN-major)
  static_assert(KST <= kMaxStages && VST <= kMaxStages, "stage count");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct QtBars {
  uint64_t q_full;
  uint64_t k_full[kMaxStages], k_conv[kMaxStages], k_empty[kMaxStages];
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[2], p_full[2], o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct QtParams {
  Phase2Args a;
  int pairs;   // pairs of 128-row tiles per (batch, kv head)
  int units;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two bf16 (one 32-bit word) -> two fp16.  bf16 -> fp32 is exact (the bf16
// bits are the top half of the fp32 word); fp32 -> fp16 rounds to nearest,
// which is exact for bf16 values in fp16's normal range.  `flags` collects
// results that are not finite: each half's exponent field plus 0x0400
// carries into that half's top bit only when the field is all ones (inf or
// NaN), and a half's sum stays below 0x10000, so the halves never carry into
// each other; flags & 0x80008000 is non-zero iff some result was not finite.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, uint32_t& flags) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  const __half2 h = __floats2half2_rn(lo, hi);
  const uint32_t r = *reinterpret_cast<const uint32_t*>(&h);
  flags |= (r & 0x7C007C00u) + 0x04000400u;
  return r;
}

template <int D>
__global__ void __launch_bounds__(384, 1) phase2_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                           const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const __grid_constant__ CUtensorMap tmKs,
                                                           const __grid_constant__ CUtensorMap tmVs,
                                                           const __grid_constant__ QtParams p) {
  using C = QtCfg<D>;
  constexpr int KST = C::KST, VST = C::VST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  QtBars* bars = reinterpret_cast<QtBars*>(smem + C::OFF_BAR);
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Phase2Args& a = p.a;
  const uint64_t wait_ns = a.wait_limit_ns;   // limit of every bounded wait

  // work item: pair fastest (CTAs that share a unit's K / V run together)
  int idx = blockIdx.x;
  const int pair = idx % p.pairs;
  idx /= p.pairs;
  const int kvh = idx % a.hkv;
  idx /= a.hkv;
  const int u = idx % p.units;
  const int b = idx / p.units;
  const int g = a.hq / a.hkv;
  const int R = a.Tq * g;
  const UnitView uv = phase2_unit(a, u);
  const bool own = uv.causal_base >= 0;
  const int nkv = static_cast<int>((uv.k1 - uv.k0 + kKT - 1) / kKT);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_conv[s], kConvThreads);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
      mbar_init(&bars->o_final[t], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  const volatile int* gabort = &a.status->code;   // set by any CTA that gave up
  auto fail = [&](int where) {
    *abort = 1;
    set_status(a.status, PA_ERR_TIMEOUT, static_cast<int>(blockIdx.x), where);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nkv > 0) {
      const CUtensorMap* mk = own ? &tmKs : &tmK;
      const CUtensorMap* mv = own ? &tmVs : &tmV;
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(mk);
      tma_prefetch_desc(mv);
      // Q: row tile t covers tokens [mt * 128 / g, +128 / g) of batch b; the
      // box (64 x g heads x 128 / g tokens) lands as rows token * g + head
      const int tpt = 128 / g;
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE + (a.stall ? 16 : 0));
      for (int t = 0; t < 2; ++t) {
        const int tok = b * a.Tq + (2 * pair + t) * tpt;
        for (int kb = 0; kb < C::NKB; ++kb)
          tma_load_3d(sQ + t * C::TILE + kb * C::KB_BYTES, &tmQ, &bars->q_full, kb * 64, kvh * g, tok);
      }
      const int row_base = static_cast<int>(static_cast<int64_t>(b) * uv.stride_rows + uv.k0);
      int armed_k[KST], armed_v[VST];
      for (int s = 0; s < KST; ++s) armed_k[s] = 0;
      for (int s = 0; s < VST; ++s) armed_v[s] = 0;
      for (int j = 0; j < nkv; ++j) {
        const int row = row_base + j * kKT;
        const int sk = j % KST, sv = j % VST;
        if (!mbar_wait(&bars->k_empty[sk], ((j / KST) & 1) ^ 1, abort, wait_ns, gabort)) { fail(1); break; }
        mbar_arrive_expect_tx(&bars->k_full[sk], C::TILE);
        for (int kb = 0; kb < C::NKB; ++kb)
          tma_load_3d(sK + sk * C::TILE + kb * C::KB_BYTES, mk, &bars->k_full[sk], kb * 64, kvh, row);
        ++armed_k[sk];
        if (!mbar_wait(&bars->v_empty[sv], ((j / VST) & 1) ^ 1, abort, wait_ns, gabort)) { fail(2); break; }
        mbar_arrive_expect_tx(&bars->v_full[sv], C::TILE);
        for (int kb = 0; kb < C::NKB; ++kb)
          tma_load_3d(sV + sv * C::TILE + kb * C::KB_BYTES, mv, &bars->v_full[sv], kb * 64, kvh, row);
        ++armed_v[sv];
      }
      // Drain: every copy this thread started has landed before the CTA ends.
      int zero = 0;
      mbar_wait(&bars->q_full, 0, &zero, wait_ns);
      for (int s = 0; s < KST; ++s)
        if (armed_k[s]) mbar_wait(&bars->k_full[s], (armed_k[s] - 1) & 1, &zero, wait_ns);
      for (int s = 0; s < VST; ++s)
        if (armed_v[s]) mbar_wait(&bars->v_full[s], (armed_v[s] - 1) & 1, &zero, wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && nkv > 0) {
      // base descriptors, computed once; each MMA adds a constant offset
      const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t v_desc = sdesc_sw128(smem_u32(sV), C::KB_BYTES, 1024);
      auto qk = [&](int t, int sk) {
        const uint32_t d_tmem = tmem + t * 256;
        const uint64_t qd = sdesc_add(q_desc, t * C::TILE);
        const uint64_t kd = sdesc_add(k_desc, sk * C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::NKB; ++kb)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss(d_tmem, sdesc_add(qd, kb * C::KB_BYTES + ks * 32), sdesc_add(kd, kb * C::KB_BYTES + ks * 32),
                   C::IDESC_QK, (kb | ks) != 0);
      };
      auto pv = [&](int t, int sv, int acc) {
        const uint32_t d_tmem = tmem + t * 256 + 128;
        const uint64_t vd = sdesc_add(v_desc, sv * C::TILE);
#pragma unroll
        for (int ks = 0; ks < kKT / 16; ++ks)
          mma_ts(d_tmem, tmem + t * 256 + ks * 8, sdesc_add(vd, ks * 2048), C::IDESC_PV, (acc | ks) != 0);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, wait_ns, gabort);
      if (!ok) fail(3);
      for (int j = 0; ok && j < nkv; ++j) {
        const int sv = j % VST;
        const int sk1 = (j + 1) % KST;
        const uint32_t pk1 = ((j + 1) / KST) & 1;
        if (j == 0) {
          if (!mbar_wait(&bars->k_conv[0], 0, abort, wait_ns, gabort)) { fail(4); break; }
          tc_fence_after();
          qk(0, 0);
          mma_commit(&bars->s_full[0]);
          qk(1, 0);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->k_empty[0]);
        }
        // tile 0: O0 += P0 V_j, then S0 = Q0 K_{j+1}
        if (!mbar_wait(&bars->p_full[0], j & 1, abort, wait_ns, gabort)) { fail(5); break; }
        if (!mbar_wait(&bars->v_full[sv], (j / VST) & 1, abort, wait_ns, gabort)) { fail(6); break; }
        tc_fence_after();
        pv(0, sv, j > 0);
        if (j == nkv - 1) mma_commit(&bars->o_final[0]);
        if (j + 1 < nkv) {
          if (!mbar_wait(&bars->k_conv[sk1], pk1, abort, wait_ns, gabort)) { fail(7); break; }
          tc_fence_after();
          qk(0, sk1);
          mma_commit(&bars->s_full[0]);
        }
        // tile 1: O1 += P1 V_j, then S1 = Q1 K_{j+1}
        if (!mbar_wait(&bars->p_full[1], j & 1, abort, wait_ns, gabort)) { fail(8); break; }
        tc_fence_after();
        pv(1, sv, j > 0);
        if (j == nkv - 1) mma_commit(&bars->o_final[1]);
        mma_commit(&bars->v_empty[sv]);
        if (j + 1 < nkv) {
          qk(1, sk1);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->k_empty[sk1]);
        }
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      int zero = 0;
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &zero, wait_ns);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------- K converters
    const int ct = threadIdx.x - 64;   // 0 .. 63
    uint32_t flags = 0;
    for (int j = 0; j < nkv; ++j) {
      const int sk = j % KST;
      if (!mbar_wait(&bars->k_full[sk], (j / KST) & 1, abort, wait_ns, gabort)) { fail(12); break; }
      uint4* tile = reinterpret_cast<uint4*>(sK + sk * C::TILE);
      constexpr int N16 = C::TILE / 16;   // 16-byte chunks per tile
#pragma unroll 4
      for (int c = ct; c < N16; c += kConvThreads) {
        uint4 v = tile[c];
        v.x = bf16x2_to_f16x2(v.x, flags);
        v.y = bf16x2_to_f16x2(v.y, flags);
        v.z = bf16x2_to_f16x2(v.z, flags);
        v.w = bf16x2_to_f16x2(v.w, flags);
        tile[c] = v;
      }
      // generic-proxy stores -> visible to the tensor core's async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars->k_conv[sk]);
    }
    // a key of this unit outside fp16 range: the unit is recomputed exactly
    // (mma.sync row kernel, high / low bf16 query) after this kernel
    if (flags & 0x80008000u) atomicExch(a.redo + (static_cast<int64_t>(b) * p.units + u) * a.hkv + kvh, 1);
  } else {
    // -------------------------------------------------------------- softmax
    const int t = warp >= 8 ? 1 : 0;
    const int sub = warp & 3;
    const int rl = sub * 32 + lane;
    // last visible key of this row, counted from the unit's first key
    const int64_t vis = (own ? min(uv.k1 - 1, uv.causal_base + ((2 * pair + t) * 128 + rl) / g) : uv.k1 - 1) - uv.k0;
    const uint32_t s_tmem = tmem + (static_cast<uint32_t>(sub * 32) << 16) + t * 256;
    const uint32_t o_tmem = s_tmem + 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&bars->s_full[t], j & 1, abort, wait_ns, gabort)) { fail(9); ok = false; break; }
      tc_fence_after();
      uint32_t sr[kKT];
      tmem_ld_x128(s_tmem, sr);
      const int64_t lim64 = vis - static_cast<int64_t>(j) * kKT;   // columns <= lim visible
      const int lim = lim64 < 0 ? -1 : (lim64 > kKT ? kKT : static_cast<int>(lim64));
      if (__any_sync(0xffffffffu, lim < kKT - 1)) {
#pragma unroll
        for (int i = 0; i < kKT; ++i)
          if (i > lim) sr[i] = __float_as_uint(-INFINITY);
      }
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
#pragma unroll
      for (int i = 0; i < kKT / 2; ++i)
        mx[i & 7] = fmax3(mx[i & 7], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
      const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
      const float m_new = fmaxf(m_run, mt);
      const bool need = m_new > m_run + 8.f;   // lazy rescale: only when P could exceed 2^8
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc2[e] = 0ull;   // two 0.0f
#pragma unroll
      for (int c = 0; c < kKT / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2_unpack(f2_add(f2_pack(__uint_as_float(sr[32 * c + 2 * i]), __uint_as_float(sr[32 * c + 2 * i + 1])),
                           nm2), x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          acc2[i & 3] = f2_add(acc2[i & 3], f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st_x16(s_tmem + 16 * c, pk);
      }
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a0, a1;
        f2_unpack(acc2[e], a0, a1);
        sum += a0 + a1;
      }
      l_run = l_run * alpha + sum;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O was last written by PV_{j-1}, which completed before S_j (the
        // commit signalling S_j covers every earlier MMA).
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld_x32(o_tmem + 32 * c, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st_x32(o_tmem + 32 * c, ov);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[t]);
    }
    const int r = (2 * pair + t) * 128 + rl;   // row of this (batch, kv head)
    const bool valid = r < R;
    const int64_t orow = ((static_cast<int64_t>(b) * p.units + u) * a.Tq + r / g) * a.hq + kvh * g + r % g;
    float* dst = a.unit_o + orow * D;
    if (nkv == 0) {
      if (valid) {
#pragma unroll
        for (int c = 0; c < D / 4; ++c) reinterpret_cast<float4*>(dst)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.unit_lse[orow] = -INFINITY;
      }
    } else if (ok && mbar_wait(&bars->o_final[t], 0, abort, wait_ns, gabort)) {
      tc_fence_after();
      const bool empty = !(l_run > 0.f);
      const float inv = empty ? 0.f : 1.f / l_run;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld_x32(o_tmem + 32 * c, ov);
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            d4[v4] = make_float4(__uint_as_float(ov[4 * v4]) * inv, __uint_as_float(ov[4 * v4 + 1]) * inv,
                                 __uint_as_float(ov[4 * v4 + 2]) * inv, __uint_as_float(ov[4 * v4 + 3]) * inv);
        }
      }
      if (valid) a.unit_lse[orow] = empty ? -INFINITY : (m_run + __log2f(l_run)) * kLn2f;
    } else if (ok) {
      fail(10);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

template <int D>
int launch_qt(const Phase2Args& a, const __half* q16, cudaStream_t s) {
  using C = QtCfg<D>;
  const int g = a.hq / a.hkv;
  CUtensorMap mq, mk, mv, mks, mvs;
  const int64_t q_rows = static_cast<int64_t>(a.B) * a.Tq;
  const int64_t k_rows = static_cast<int64_t>(a.B) * a.T;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!tma_map_3d(&mq, q16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, D, a.hq, q_rows, 64, g, 128 / g)) return PA_ERR_CUDA;
  // an empty context cache still needs a valid map: point it at the query
  const void* kc = k_rows > 0 ? a.k_ret : static_cast<const void*>(q16);
  const void* vc = k_rows > 0 ? a.v_ret : static_cast<const void*>(q16);
  const int64_t kc_rows = k_rows > 0 ? k_rows : 1;
  if (!tma_map_3d(&mk, kc, BF, D, a.hkv, kc_rows, 64, 1, kKT) ||
      !tma_map_3d(&mv, vc, BF, D, a.hkv, kc_rows, 64, 1, kKT))
    return PA_ERR_CUDA;
  if (a.has_self) {
    const int64_t s_rows = static_cast<int64_t>(a.B) * a.self_cap;
    if (!tma_map_3d(&mks, a.k_self, BF, D, a.hkv, s_rows, 64, 1, kKT) ||
        !tma_map_3d(&mvs, a.v_self, BF, D, a.hkv, s_rows, 64, 1, kKT))
      return PA_ERR_CUDA;
  } else {
    mks = mk;
    mvs = mv;
  }
  QtParams p;
  p.a = a;
  p.units = phase2_units(a);
  const int tiles = (a.Tq * g + 127) / 128;
  p.pairs = (tiles + 1) / 2;
  const int64_t grid = static_cast<int64_t>(a.B) * p.units * a.hkv * p.pairs;
  if (grid <= 0) return PA_OK;
  if (cudaFuncSetAttribute(phase2_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  phase2_tc_kernel<D><<<static_cast<unsigned>(grid), 384, C::SMEM_BYTES, s>>>(mq, mk, mv, mks, mvs, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

bool phase2_tc_supported(const Phase2Args& a) {
  if (a.dtype != PA_BF16 || (a.d != 64 && a.d != 128)) return false;
  const int g = a.hq / a.hkv;
  if (g < 1 || 128 % g != 0) return false;
  if (static_cast<int64_t>(a.Tq) * g < kPhase2TcMinRows) return false;
  // TMA coordinates are 32-bit; base addresses must be 16-byte aligned
  const int64_t lim = (int64_t{1} << 31) - 2 * kKT;
  if (static_cast<int64_t>(a.B) * a.T > lim || static_cast<int64_t>(a.B) * a.Tq > lim) return false;
  if (a.T > 0 && (!aligned16(a.k_ret) || !aligned16(a.v_ret))) return false;
  if (a.has_self) {
    if (static_cast<int64_t>(a.B) * a.self_cap > lim) return false;
    if (!aligned16(a.k_self) || !aligned16(a.v_self)) return false;
  }
  return true;
}

int launch_phase2_tc(const Phase2Args& a, const __half* q16, cudaStream_t s) {
  return a.d == 128 ? launch_qt<128>(a, q16, s) : launch_qt<64>(a, q16, s);
}

}  // namespace pa
