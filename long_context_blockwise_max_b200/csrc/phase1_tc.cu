// Phase-1 causal attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes is the Phase-1 encoding of the Pulsar Attention page (§2,
// §2.1) and of the Star Attention anchor variant: for every host, causal
// softmax attention over the host's packed rows, every row reading its
// original position's rotated Q / K (see phase1.cu for the position map).
//
// CTA = one 128-row tile of one host x two query heads of the same GQA group
// (they share every K / V tile).  12 warps:
//   warp 0      TMA producer: Q tiles once, then K / V tiles through a
//               2-stage ring; each 128-row tile is 8 boxes of 16 rows, since
//               the packed rows are runs of 16 contiguous positions.
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (fp16 x fp16 -> fp32
//               TMEM) and O_t += P_t V (P bf16 read from TMEM, V bf16 from
//               shared memory, MN-major).  The two heads ping-pong: while one
//               warpgroup runs its softmax the tensor core works on the other.
//   warp 2      TMEM allocation (512 columns: S0 | O0 | S1 | O1).
//   warps 4-7   softmax of head 0, warps 8-11 softmax of head 1: one thread
//               per row; online softmax in log2 units with a lazy rescale of
//               O (only when the running max grows by more than 2^8); P is
//               written back over S in TMEM as bf16.
// Every wait on an mbarrier is bounded (1 s); on expiry the CTA records
// PA_ERR_TIMEOUT in the status block, drains its copies and MMAs, frees
// TMEM and returns.
//
// Scheduling: one CTA per (host, kv head, row tile, head pair), host-major
// so that concurrent CTAs share one host's K / V in L2 (see decode_item).
#include <cudaTypedefs.h>

#include <algorithm>

#include "pa_internal.h"
#include "sm100.cuh"

namespace pa {
using namespace sm100;

namespace {


template <int D>
struct TcCfg {
  static constexpr int NKB = D / 64;                 // 128-byte column blocks along d
  static constexpr int KB_BYTES = 128 * 128;         // 128 rows x 128 B
  static constexpr int TILE_BYTES = NKB * KB_BYTES;  // 128 rows x D x 2 B
  static constexpr int STAGES = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr uint32_t IDESC_QK = idesc_f16(128, 128, 0, 0, 0, 0);  // f16 Q . f16 K
  static constexpr uint32_t IDESC_PV = idesc_f16(128, D, 1, 1, 0, 1);    // bf16 P . bf16 V (MN-major)
};

struct TcBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int host, tile, kvh, pair;
};

struct TcParams {
  HostTable ht;
  const int32_t* rowpos;   // packed row -> position (V)
  const int32_t* rowci;    // packed row -> row of Qr / Kr
  __nv_bfloat16* o;
  float* lse;
  int hq, hkv, pairs;   // pairs = (hq / hkv) / 2 head pairs per kv head
  int max_tiles;
  DeviceStatus* status;
  uint64_t wait_ns;   // limit of every bounded wait
  int stall;          // test only: the Q barrier expects 16 bytes more than are copied
};

__device__ __forceinline__ int host_tiles(const HostTable& ht, int i) {
  return ht.tile_off[i + 1] - ht.tile_off[i];
}

// Work order: hosts from the longest to the shortest (host lengths never
// decrease with the host index), then kv head, then row tile from the
// deepest (most key tiles) to the shallowest, then head pair.  CTAs that run
// at the same time therefore share one host's K / V for one kv head, which
// stays in L2, and the shortest tiles come last.
__device__ void decode_item(const HostTable& ht, int hkv, int pairs, int idx, int* host, int* kvh,
                            int* tile, int* pair) {
  int h = ht.n_hosts - 1;
  for (; h > 0; --h) {
    const int cnt = host_tiles(ht, h) * hkv * pairs;
    if (idx < cnt) break;
    idx -= cnt;
  }
  const int nt = host_tiles(ht, h);
  *host = h;
  *kvh = idx / (nt * pairs);
  const int rem = idx % (nt * pairs);
  *tile = nt - 1 - rem / pairs;
  *pair = rem % pairs;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(384, 1) phase1_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                           const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(smem + C::OFF_BAR);
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    int host, kvh_, tile, pair_;
    decode_item(p.ht, p.hkv, p.pairs, blockIdx.x, &host, &kvh_, &tile, &pair_);
    bars->host = host;
    bars->tile = tile;
    bars->kvh = kvh_;
    bars->pair = pair_;
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
      mbar_init(&bars->o_final[s], 1);
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
  const volatile int* gabort = &p.status->code;   // set by any CTA that gave up
  const int host = bars->host, tile = bars->tile;
  const int kvh = bars->kvh;
  const int h0 = kvh * (2 * p.pairs) + 2 * bars->pair;
  const int64_t row0 = p.ht.row_off[host];
  const int n = static_cast<int>(p.ht.row_off[host + 1] - row0);
  const int r0 = tile * 128;
  const int nkv = tile + 1;   // causal: key tiles 0..tile
  auto fail = [&](int where) {
    *abort = 1;
    set_status(p.status, PA_ERR_TIMEOUT, static_cast<int>(blockIdx.x), where);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      auto pos_of = [&](int r) -> int { return p.rowpos[row0 + (r < n ? r : 0)]; };
      auto ci_of = [&](int r) -> int { return p.rowci[row0 + (r < n ? r : 0)]; };
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE_BYTES + (p.stall ? 16 : 0));
      for (int grp = 0; grp < 8; ++grp) {
        const int pq = ci_of(r0 + 16 * grp);
        for (int t = 0; t < 2; ++t)
          for (int kb = 0; kb < C::NKB; ++kb)
            tma_load_3d(sQ + t * C::TILE_BYTES + kb * C::KB_BYTES + grp * 2048, &tmQ, &bars->q_full,
                        kb * 64, h0 + t, pq);
      }
      int armed_k[2] = {0, 0}, armed_v[2] = {0, 0};
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        int pk[8], ck[8];
        for (int grp = 0; grp < 8; ++grp) {
          pk[grp] = pos_of(j * 128 + 16 * grp);
          ck[grp] = ci_of(j * 128 + 16 * grp);
        }
        if (!mbar_wait(&bars->k_empty[st], ph ^ 1, abort, p.wait_ns, gabort)) { fail(1); break; }
        mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
        for (int grp = 0; grp < 8; ++grp)
          for (int kb = 0; kb < C::NKB; ++kb)
            tma_load_3d(sK + st * C::TILE_BYTES + kb * C::KB_BYTES + grp * 2048, &tmK, &bars->k_full[st],
                        kb * 64, kvh, ck[grp]);
        ++armed_k[st];
        if (!mbar_wait(&bars->v_empty[st], ph ^ 1, abort, p.wait_ns, gabort)) { fail(2); break; }
        mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
        for (int grp = 0; grp < 8; ++grp)
          for (int kb = 0; kb < C::NKB; ++kb)
            tma_load_3d(sV + st * C::TILE_BYTES + kb * C::KB_BYTES + grp * 2048, &tmV, &bars->v_full[st],
                        kb * 64, kvh, pk[grp]);
        ++armed_v[st];
      }
      // Drain: every copy this thread started has landed before the CTA ends.
      int zero = 0;
      mbar_wait(&bars->q_full, 0, &zero, p.wait_ns);
      for (int s = 0; s < 2; ++s) {
        if (armed_k[s]) mbar_wait(&bars->k_full[s], (armed_k[s] - 1) & 1, &zero, p.wait_ns);
        if (armed_v[s]) mbar_wait(&bars->v_full[s], (armed_v[s] - 1) & 1, &zero, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      // base descriptors, computed once; each MMA adds a constant offset
      const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t v_desc = sdesc_sw128(smem_u32(sV), C::KB_BYTES, 1024);
      auto qk = [&](int t, int st) {
        const uint32_t d_tmem = tmem + t * 256;
        const uint64_t qd = sdesc_add(q_desc, t * C::TILE_BYTES);
        const uint64_t kd = sdesc_add(k_desc, st * C::TILE_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::NKB; ++kb)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss(d_tmem, sdesc_add(qd, kb * C::KB_BYTES + ks * 32), sdesc_add(kd, kb * C::KB_BYTES + ks * 32),
                   C::IDESC_QK, (kb | ks) != 0);
      };
      auto pv = [&](int t, int st, int acc) {
        const uint32_t d_tmem = tmem + t * 256 + 128;
        const uint64_t vd = sdesc_add(v_desc, st * C::TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts(d_tmem, tmem + t * 256 + ks * 8, sdesc_add(vd, ks * 2048), C::IDESC_PV, (acc | ks) != 0);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, p.wait_ns, gabort);
      if (!ok) fail(3);
      for (int j = 0; ok && j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int st1 = (j + 1) & 1;
        const uint32_t ph1 = ((j + 1) >> 1) & 1;
        if (j == 0) {
          if (!mbar_wait(&bars->k_full[0], 0, abort, p.wait_ns, gabort)) { fail(4); break; }
          tc_fence_after();
          qk(0, 0);
          mma_commit(&bars->s_full[0]);
          qk(1, 0);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->k_empty[0]);
        }
        // head 0: O0 += P0 V_j, then S0 = Q0 K_{j+1}.  V_j and K_{j+1} are
        // waited for first, while the tensor pipe still runs head 1's MMAs,
        // so that nothing stands between P0 and the MMAs that consume it.
        if (!mbar_wait(&bars->v_full[st], ph, abort, p.wait_ns, gabort)) { fail(6); break; }
        if (j + 1 < nkv && !mbar_wait(&bars->k_full[st1], ph1, abort, p.wait_ns, gabort)) { fail(7); break; }
        if (!mbar_wait(&bars->p_full[0], j & 1, abort, p.wait_ns, gabort)) { fail(5); break; }
        tc_fence_after();
        pv(0, st, j > 0);
        if (j == nkv - 1) mma_commit(&bars->o_final[0]);
        if (j + 1 < nkv) {
          qk(0, st1);
          mma_commit(&bars->s_full[0]);
        }
        // head 1: O1 += P1 V_j, then S1 = Q1 K_{j+1}
        if (!mbar_wait(&bars->p_full[1], j & 1, abort, p.wait_ns, gabort)) { fail(8); break; }
        tc_fence_after();
        pv(1, st, j > 0);
        if (j == nkv - 1) mma_commit(&bars->o_final[1]);
        mma_commit(&bars->v_empty[st]);
        if (j + 1 < nkv) {
          qk(1, st1);
          mma_commit(&bars->s_full[1]);
          mma_commit(&bars->k_empty[st1]);
        }
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      int zero = 0;
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &zero, p.wait_ns);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int t = warp >= 8 ? 1 : 0;
    const int sub = warp & 3;
    const int rl = sub * 32 + lane;
    const int r = r0 + rl;
    const int head = h0 + t;
    const uint32_t s_tmem = tmem + (static_cast<uint32_t>(sub * 32) << 16) + t * 256;
    const uint32_t o_tmem = s_tmem + 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&bars->s_full[t], j & 1, abort, p.wait_ns, gabort)) { fail(9); ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128(s_tmem, sr);
      // row max with 8 independent partial maxima (three-input max, short
      // dependency chains); only the diagonal tile needs the causal /
      // ragged-end mask
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
      const bool diag = (j == nkv - 1);
      if (diag) {
        const int lim = min(r, n - 1) - j * 128;   // columns <= lim are visible
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > lim) sr[i] = __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int i = 0; i < 64; ++i)
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
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1, p0, p1;
          f2_unpack(f2_add(f2_pack(__uint_as_float(sr[32 * c + 2 * i]), __uint_as_float(sr[32 * c + 2 * i + 1])),
                           nm2), x0, x1);
          p0 = fast_exp2(x0);
          p1 = fast_exp2(x1);
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
    if (ok && mbar_wait(&bars->o_final[t], 0, abort, p.wait_ns, gabort)) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      __nv_bfloat16* dst = p.o + ((row0 + r) * p.hq + head) * static_cast<int64_t>(D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld_x32(o_tmem + 32 * c, ov);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
        if (r < n) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (r < n && p.lse != nullptr) p.lse[(row0 + r) * p.hq + head] = (m_run + __log2f(l_run)) * kLn2f;
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

// [rows][heads][d] 16-bit tensor, boxes of 16 rows x 1 head x 64 elements.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int64_t rows, int heads, int d) {
  return tma_map_3d(m, base, dt, d, heads, rows, 64, 1, 16);
}

template <int D>
int launch_tc(const Phase1Args& a, cudaStream_t s) {
  using C = TcCfg<D>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.qr, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.qk_rows, a.hq, D) ||
      !make_map(&mk, a.kr, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.qk_rows, a.hkv, D) ||
      !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L, a.hkv, D))
    return PA_ERR_CUDA;
  TcParams p;
  p.ht = a.ht;
  p.rowpos = a.rowpos;
  p.rowci = a.rowci;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.hq = a.hq;
  p.hkv = a.hkv;
  p.pairs = (a.hq / a.hkv) / 2;
  p.max_tiles = 0;
  for (int i = 0; i < a.ht.n_hosts; ++i)
    p.max_tiles = std::max(p.max_tiles, a.ht.tile_off[i + 1] - a.ht.tile_off[i]);
  p.status = a.status;
  p.wait_ns = a.wait_limit_ns;
  p.stall = a.stall;
  const int64_t items = a.ht.tile_off[a.ht.n_hosts];
  const int64_t grid = items * a.hkv * p.pairs;
  if (grid <= 0) return PA_OK;
  if (cudaFuncSetAttribute(phase1_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  phase1_tc_kernel<D><<<static_cast<unsigned>(grid), 384, C::SMEM_BYTES, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

namespace sm100 {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool tma_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int64_t dim0, int64_t dim1,
                int64_t dim2, int box0, int box1, int box2) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(dim0), static_cast<cuuint64_t>(dim1),
                        static_cast<cuuint64_t>(dim2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(dim0) * 2, static_cast<cuuint64_t>(dim1) * dim0 * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(box1),
                       static_cast<cuuint32_t>(box2)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sm100

bool phase1_tc_supported(const Phase1Args& a) {
  const int g = a.hq / a.hkv;
  return a.dtype == PA_BF16 && (a.d == 64 || a.d == 128) && g % 2 == 0;
}

int launch_phase1_tc(const Phase1Args& a, cudaStream_t s) {
  return a.d == 128 ? launch_tc<128>(a, s) : launch_tc<64>(a, s);
}

}  // namespace pa
