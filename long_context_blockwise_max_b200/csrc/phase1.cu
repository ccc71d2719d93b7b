// Phase-1 context encoding (Pulsar Attention page §2, §2.1; Dutch technical
// summary "Fase 1"; Star Attention review, key_machinery).
//
// Layout idea: every Phase-1 row of every host is a token of the original
// sequence carrying its original position id, and RoPE depends only on that
// position.  So Q and K are rotated ONCE per token (rope_qk_kernel) and each
// host's rows are read through `rowpos` (packed row -> position): the sink,
// the summary chunks and the block itself are runs of contiguous tokens,
// nothing is copied per host, and the retained cache (B_i's rotated K and V
// for every host) is simply the whole sequence's rotated K and V.
//
// A call over a range of hosts that reads few of the sequence's positions
// (the later hosts of a sequence spread over GPUs) rotates only those: its
// Qr / Kr rows are [sink || Sigma_0 .. Sigma_{host_end-2} || the range's
// blocks] (Star: [B_0 || the range's blocks]), so its RoPE work and
// workspace scale with the positions it reads, not with L.  Every host's
// prefix rows are the first rows of that order, so a prefix row's Qr / Kr
// row is its row index within the host.
//
//  rowpos_kernel     : packed row -> original position (V rows) and -> Qr /
//                      Kr row (the same unless compact).
//  posmap_kernel     : compact Qr / Kr row -> original position.
//  rope_qk_kernel    : Q -> Qr (scaled by log2(e)/sqrt(d)), K -> Kr (QK
//                      operand type) and k_ret (input dtype).
//  phase1_simt_kernel: causal attention over a host's rows, fp32 SIMT with an
//                      online softmax (used for fp32 inputs, and for bf16
//                      inputs when the tensor-core kernel is not selected).
//  phase1_head_rows_kernel: the first kHeadRows rows of every host again, in
//                      fp32 from the unrounded inputs (bf16 inputs only).
#include "pa_internal.h"

namespace pa {

__global__ void rowpos_kernel(HostTable ht, const int32_t* __restrict__ sel,
                              int32_t* __restrict__ rowpos, int32_t* __restrict__ rowci,
                              DeviceStatus* st) {
  const int64_t R = ht.row_off[ht.n_hosts];
  const int64_t summ = (int64_t)ht.k_chunks * ht.chunk;
  const int C = ht.chunk > 0 ? ht.block / ht.chunk : 0;
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R;
       r += (int64_t)gridDim.x * blockDim.x) {
    int li = 0;
    while (li + 1 < ht.n_hosts && r >= ht.row_off[li + 1]) ++li;
    const int64_t u = r - ht.row_off[li];
    const int i = ht.host0 + li;                     // the host's index in the sequence
    int64_t p;
    // own-block rows start at row `pre` of the host
    const int64_t pre = i == 0 ? 0 : (ht.star ? ht.block : ht.sink + (int64_t)i * summ);
    if (i == 0) {
      p = u;                                         // host 0: B_0 alone
    } else if (ht.star) {
      p = (u < ht.block) ? u : (int64_t)i * ht.block + (u - ht.block);  // [B_0 || B_i]
    } else if (u < ht.sink) {
      p = u;                                         // attention sink
    } else if (u < ht.sink + (int64_t)i * summ) {    // Sigma_0 .. Sigma_{i-1}
      const int64_t w = u - ht.sink;
      const int64_t j = w / summ, x = w % summ;
      const int m = (int)(x / ht.chunk), t = (int)(x % ht.chunk);
      int c = sel[j * ht.k_chunks + m];
      if (c < 0 || c >= C) {
        set_status(st, PA_ERR_INVALID, (int)(j * ht.k_chunks + m), c);
        c = 0;
      }
      p = j * ht.block + (int64_t)c * ht.chunk + t;
    } else {
      p = (int64_t)i * ht.block + (u - ht.sink - (int64_t)i * summ);   // B_i
    }
    rowpos[r] = (int32_t)p;
    if (rowci != rowpos) {
      const int64_t ci = u < pre ? u : ht.ci_blk + (int64_t)(i - ht.host0) * ht.block + (u - pre);
      rowci[r] = (int32_t)ci;
    }
  }
}

// Compact Qr / Kr row -> original position (the inverse of rowci over one
// copy of every position the range reads).
__global__ void posmap_kernel(HostTable ht, int64_t n, const int32_t* __restrict__ sel,
                              int32_t* __restrict__ posmap, DeviceStatus* st) {
  const int64_t summ = (int64_t)ht.k_chunks * ht.chunk;
  const int C = ht.chunk > 0 ? ht.block / ht.chunk : 0;
  for (int64_t ci = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; ci < n;
       ci += (int64_t)gridDim.x * blockDim.x) {
    int64_t p;
    if (ci >= ht.ci_blk) {
      p = (int64_t)ht.host0 * ht.block + (ci - ht.ci_blk);           // the range's blocks
    } else if (ht.star || ci < ht.sink) {
      p = ci;                                                        // B_0 anchor / sink
    } else {
      const int64_t w = ci - ht.sink;                                // Sigma_j, chunk m, token t
      const int64_t j = w / summ, x = w % summ;
      const int m = (int)(x / ht.chunk), t = (int)(x % ht.chunk);
      int c = sel[j * ht.k_chunks + m];
      if (c < 0 || c >= C) {
        set_status(st, PA_ERR_INVALID, (int)(j * ht.k_chunks + m), c);
        c = 0;
      }
      p = j * ht.block + (int64_t)c * ht.chunk + t;
    }
    posmap[ci] = (int32_t)p;
  }
}

// RoPE (rotate-half): for m < d/2, a = p * omega_m,
//   x'[m] = x[m] cos a - x[m + d/2] sin a,  x'[m + d/2] = x[m + d/2] cos a + x[m] sin a.
// The angle and its sine/cosine are evaluated in fp64, the rotation in fp32.
// Each thread rotates one 16-byte vector of x[m..] together with the
// matching vector of x[m + d/2 ..]; a CTA covers POS positions, all heads.
template <typename T, int N>
struct alignas(16) Vec {
  T v[N];
};

// Row ci of Qr / Kr holds position posmap[ci] (ci itself when posmap is
// null); Kr rows [kret_lo, kret_lo + kret_n) are also written to k_ret.
template <typename IT, typename QT, int POS>
__global__ void __launch_bounds__(256) rope_qk_kernel(
    const IT* __restrict__ q, const IT* __restrict__ k, int64_t n_rows, const int32_t* __restrict__ posmap,
    int hq, int hkv, int d, RopeFreqs f, float qscale, QT* __restrict__ qr, QT* __restrict__ kr,
    IT* __restrict__ k_ret, int64_t kret_lo, int64_t kret_n, DeviceStatus* st) {
  constexpr int VEC = 16 / sizeof(IT);          // input elements per 16-byte vector
  __shared__ float2 cs[POS][kMaxHalfDim];
  __shared__ int64_t spos[POS];
  const int half = d / 2;
  const int64_t ci0 = (int64_t)blockIdx.x * POS;
  if (threadIdx.x < POS) {
    const int64_t ci = ci0 + threadIdx.x;
    spos[threadIdx.x] = ci < n_rows ? (posmap != nullptr ? (int64_t)posmap[ci] : ci) : 0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < POS * half; e += blockDim.x) {
    const int pp = e / half, m = e % half;
    double sn, cn;
    sincos((double)spos[pp] * f.omega[m], &sn, &cn);
    cs[pp][m] = make_float2((float)cn, (float)sn);
  }
  __syncthreads();
  const int vpr = half / VEC;                         // vectors per half row
  const int per_pos = (hq + hkv) * vpr;
  bool bad = false;
  for (int e = threadIdx.x; e < POS * per_pos; e += blockDim.x) {
    const int pp = e / per_pos;
    const int64_t ci = ci0 + pp;
    if (ci >= n_rows) continue;
    const int64_t p = spos[pp];
    const int w = e % per_pos;
    const int row = w / vpr, m0 = (w % vpr) * VEC;
    const bool is_q = row < hq;
    const int h = is_q ? row : row - hq;
    const int nh = is_q ? hq : hkv;
    const int64_t base = (p * nh + h) * (int64_t)d;        // input row (position p)
    const int64_t obase = (ci * nh + h) * (int64_t)d;      // output row ci
    const IT* src = is_q ? q : k;
    const Vec<IT, VEC> a = *reinterpret_cast<const Vec<IT, VEC>*>(src + base + m0);
    const Vec<IT, VEC> b = *reinterpret_cast<const Vec<IT, VEC>*>(src + base + m0 + half);
    float y1[VEC], y2[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      const float2 c = cs[pp][m0 + i];
      const float x1 = to_f32(a.v[i]), x2 = to_f32(b.v[i]);
      y1[i] = x1 * c.x - x2 * c.y;
      y2[i] = x2 * c.x + x1 * c.y;
    }
    if (is_q) {
      Vec<QT, VEC> o1, o2;
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float u1 = y1[i] * qscale, u2 = y2[i] * qscale;
        if (sizeof(QT) == 2) bad |= !(fabsf(u1) <= 65504.f) || !(fabsf(u2) <= 65504.f);
        o1.v[i] = from_f32<QT>(u1);
        o2.v[i] = from_f32<QT>(u2);
      }
      *reinterpret_cast<Vec<QT, VEC>*>(qr + obase + m0) = o1;
      *reinterpret_cast<Vec<QT, VEC>*>(qr + obase + m0 + half) = o2;
    } else {
      if (ci >= kret_lo && ci < kret_lo + kret_n) {   // retained: the blocks of the encoded hosts
        Vec<IT, VEC> r1, r2;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          r1.v[i] = from_f32<IT>(y1[i]);
          r2.v[i] = from_f32<IT>(y2[i]);
        }
        const int64_t rb = obase - kret_lo * hkv * (int64_t)d;
        *reinterpret_cast<Vec<IT, VEC>*>(k_ret + rb + m0) = r1;
        *reinterpret_cast<Vec<IT, VEC>*>(k_ret + rb + m0 + half) = r2;
      }
      {
        Vec<QT, VEC> o1, o2;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          if (sizeof(QT) == 2) bad |= !(fabsf(y1[i]) <= 65504.f) || !(fabsf(y2[i]) <= 65504.f);
          o1.v[i] = from_f32<QT>(y1[i]);
          o2.v[i] = from_f32<QT>(y2[i]);
        }
        *reinterpret_cast<Vec<QT, VEC>*>(kr + obase + m0) = o1;
        *reinterpret_cast<Vec<QT, VEC>*>(kr + obase + m0 + half) = o2;
      }
    }
  }
  if (bad) set_status(st, PA_ERR_RANGE, 0, 0);
}

// ---------------------------------------------------------------------------
// SIMT causal attention.  CTA = 128 rows of one host x one query head; two
// threads per row, each owning interleaved groups of 4 head-dim elements.
// Scores are in log2 units (Q carries log2(e)/sqrt(d)).
// ---------------------------------------------------------------------------
template <int D, typename QT, typename VT, typename OT>
__global__ void __launch_bounds__(256) phase1_simt_kernel(
    const QT* __restrict__ qr, const QT* __restrict__ kr, const VT* __restrict__ v,
    const int32_t* __restrict__ rowpos, const int32_t* __restrict__ rowci, HostTable ht, int hq, int hkv,
    OT* __restrict__ o, float* __restrict__ lse) {
  constexpr int BK = 32, HALF = D / 2, G4 = HALF / 4;
  __shared__ __align__(16) float ks[BK][D];
  __shared__ __align__(16) float vs[BK][D];
  const int h = blockIdx.y, kvh = h / (hq / hkv);
  int host = 0;
  while (host + 1 < ht.n_hosts && (int)blockIdx.x >= ht.tile_off[host + 1]) ++host;
  const int64_t row0 = ht.row_off[host];
  const int n = (int)(ht.row_off[host + 1] - row0);
  const int tile_r0 = ((int)blockIdx.x - ht.tile_off[host]) * 128;
  const int r = tile_r0 + (threadIdx.x >> 1);
  const int hf = threadIdx.x & 1;
  const bool active = r < n;
  // element index of group g, lane-half hf: 8*g + 4*hf + {0..3}
  float qv[HALF], acc[HALF];
  if (active) {
    const int64_t pq = rowci[row0 + r];
    const QT* src = qr + (pq * hq + h) * (int64_t)D;
#pragma unroll
    for (int g = 0; g < G4; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) qv[4 * g + e] = to_f32(src[8 * g + 4 * hf + e]);
  } else {
#pragma unroll
    for (int i = 0; i < HALF; ++i) qv[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < HALF; ++i) acc[i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const int last = min(n, tile_r0 + 128) - 1;
  for (int c0 = 0; c0 <= last; c0 += BK) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < BK * D; idx += 256) {
      const int kk = idx / D, mm = idx % D, c = c0 + kk;
      float kx = 0.f, vx = 0.f;
      if (c < n) {
        const int64_t ck = rowci[row0 + c], pv = rowpos[row0 + c];
        kx = to_f32(kr[(ck * hkv + kvh) * (int64_t)D + mm]);
        vx = to_f32(v[(pv * hkv + kvh) * (int64_t)D + mm]);
      }
      ks[kk][mm] = kx;
      vs[kk][mm] = vx;
    }
    __syncthreads();
    float s[BK];
    float mt = m_run;
#pragma unroll
    for (int j = 0; j < BK; ++j) {
      float a = 0.f;
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        const float4 kk4 = *reinterpret_cast<const float4*>(&ks[j][8 * g + 4 * hf]);
        a = fmaf(qv[4 * g + 0], kk4.x, a);
        a = fmaf(qv[4 * g + 1], kk4.y, a);
        a = fmaf(qv[4 * g + 2], kk4.z, a);
        a = fmaf(qv[4 * g + 3], kk4.w, a);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      s[j] = (c0 + j <= r) ? a : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    if (mt == -INFINITY) continue;   // row sees no key of this tile (uniform per pair)
    const float alpha = fast_exp2(m_run - mt);   // exp2(-inf) = 0 on the first tile
    l_run *= alpha;
#pragma unroll
    for (int i = 0; i < HALF; ++i) acc[i] *= alpha;
#pragma unroll
    for (int j = 0; j < BK; ++j) {
      const float pj = fast_exp2(s[j] - mt);
      l_run += pj;
#pragma unroll
      for (int g = 0; g < G4; ++g) {
        const float4 vv4 = *reinterpret_cast<const float4*>(&vs[j][8 * g + 4 * hf]);
        acc[4 * g + 0] = fmaf(pj, vv4.x, acc[4 * g + 0]);
        acc[4 * g + 1] = fmaf(pj, vv4.y, acc[4 * g + 1]);
        acc[4 * g + 2] = fmaf(pj, vv4.z, acc[4 * g + 2]);
        acc[4 * g + 3] = fmaf(pj, vv4.w, acc[4 * g + 3]);
      }
    }
    m_run = mt;
  }
  if (!active) return;
  const float inv = 1.f / l_run;
  OT* dst = o + ((row0 + r) * hq + h) * (int64_t)D;
#pragma unroll
  for (int g = 0; g < G4; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[8 * g + 4 * hf + e] = from_f32<OT>(acc[4 * g + e] * inv);
  if (lse != nullptr && hf == 0) lse[(row0 + r) * hq + h] = (m_run + __log2f(l_run)) * kLn2f;
}

// ---------------------------------------------------------------------------
// Head rows in fp32.  For bf16 inputs the attention kernels read rotated Q / K
// rounded to fp16, so every logit carries up to 2^-11 relative rounding per
// operand.  A row that sees many keys averages those errors in its lse, but
// the first rows of a host see only a few keys (row r sees r + 1), and their
// lse keeps one logit's error: on unit-normal inputs up to ~1.2e-3.  This
// kernel recomputes the first kHeadRows rows of every host from the bf16
// inputs, rotating in fp32 (fp64 angles, as rope_qk_kernel) without the
// fp16 rounding, and overwrites their O and lse.  CTA = one host x one kv
// head: the keys of those rows are rotated once into shared memory; one warp
// per (row, query head of the group), each lane owning D / 32 elements.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) phase1_head_rows_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ rowpos, HostTable ht, int hq, int hkv, RopeFreqs f, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse) {
  constexpr int HALF = D / 2, PER = D / 64;   // per lane: PER elements of each half
  __shared__ float ks[kHeadRows][D];
  __shared__ float vs[kHeadRows][D];
  __shared__ float2 cs[kHeadRows][HALF];      // (cos, sin) of row j's position, frequency m
  const int host = blockIdx.x, kvh = blockIdx.y;
  const int64_t row0 = ht.row_off[host];
  const int64_t n_host = ht.row_off[host + 1] - row0;
  const int R = n_host < kHeadRows ? (int)n_host : kHeadRows;
  // query row r and key row r share a position: the angles once per row
  for (int e = threadIdx.x; e < R * HALF; e += blockDim.x) {
    const int j = e / HALF, m = e % HALF;
    double sn, cn;
    sincos((double)rowpos[row0 + j] * f.omega[m], &sn, &cn);
    cs[j][m] = make_float2((float)cn, (float)sn);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R * HALF; e += blockDim.x) {
    const int j = e / HALF, m = e % HALF;
    const int64_t pos = rowpos[row0 + j];
    const float c = cs[j][m].x, sg = cs[j][m].y;
    const __nv_bfloat16* kr = k + (pos * hkv + kvh) * (int64_t)D;
    const __nv_bfloat16* vr = v + (pos * hkv + kvh) * (int64_t)D;
    const float x1 = __bfloat162float(kr[m]), x2 = __bfloat162float(kr[m + HALF]);
    ks[j][m] = x1 * c - x2 * sg;
    ks[j][m + HALF] = x2 * c + x1 * sg;
    vs[j][m] = __bfloat162float(vr[m]);
    vs[j][m + HALF] = __bfloat162float(vr[m + HALF]);
  }
  __syncthreads();
  const int g = hq / hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = (float)(1.0 / sqrt((double)D));
  for (int w = warp; w < R * g; w += blockDim.x / 32) {
    const int r = w / g, h = kvh * g + w % g;
    const int64_t pos = rowpos[row0 + r];
    const __nv_bfloat16* qr = q + (pos * hq + h) * (int64_t)D;
    float qa[PER], qb[PER];   // elements lane + 32 i and lane + 32 i + D / 2
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int m = lane + 32 * i;
      const float c = cs[r][m].x, sg = cs[r][m].y;
      const float x1 = __bfloat162float(qr[m]), x2 = __bfloat162float(qr[m + HALF]);
      qa[i] = x1 * c - x2 * sg;
      qb[i] = x2 * c + x1 * sg;
    }
    float sc[kHeadRows];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kHeadRows; ++j) {
      float a = 0.f;
      if (j <= r) {
#pragma unroll
        for (int i = 0; i < PER; ++i) a = fmaf(qa[i], ks[j][lane + 32 * i], fmaf(qb[i], ks[j][lane + 32 * i + HALF], a));
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) a += __shfl_xor_sync(0xffffffffu, a, sh);
      }
      sc[j] = j <= r ? a * scale : -INFINITY;
      mx = fmaxf(mx, sc[j]);
    }
    float l = 0.f, oa[PER], ob[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) oa[i] = ob[i] = 0.f;
#pragma unroll
    for (int j = 0; j < kHeadRows; ++j) {
      if (j > r) break;
      const float pj = expf(sc[j] - mx);
      l += pj;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        oa[i] = fmaf(pj, vs[j][lane + 32 * i], oa[i]);
        ob[i] = fmaf(pj, vs[j][lane + 32 * i + HALF], ob[i]);
      }
    }
    const float inv = 1.f / l;
    __nv_bfloat16* dst = o + ((row0 + r) * hq + h) * (int64_t)D;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      dst[lane + 32 * i] = __float2bfloat16(oa[i] * inv);
      dst[lane + 32 * i + HALF] = __float2bfloat16(ob[i] * inv);
    }
    if (lse != nullptr && lane == 0) lse[(row0 + r) * hq + h] = mx + logf(l);
  }
}

size_t phase1_workspace_bytes(int64_t qk_rows, int32_t hq, int32_t hkv, int32_t d, int dtype,
                              int64_t rows, int64_t posmap_rows) {
  const size_t qk_elem = dtype == PA_BF16 ? 2 : 4;
  size_t b = kStatusBytes;
  b += 2 * align_up(sizeof(int32_t) * (size_t)rows);
  b += align_up(sizeof(int32_t) * (size_t)posmap_rows);
  b += align_up(qk_elem * (size_t)qk_rows * hq * d);
  b += align_up(qk_elem * (size_t)qk_rows * hkv * d);
  return b;
}

template <typename IT, typename QT, typename VT, typename OT>
static int launch_phase1_t(const Phase1Args& a, cudaStream_t s) {
  const int64_t R = a.ht.row_off[a.ht.n_hosts];
  {
    const int threads = 256;
    const int64_t want = (R + threads - 1) / threads;
    rowpos_kernel<<<(int)(want < 148 * 8 ? want : 148 * 8), threads, 0, s>>>(a.ht, a.sel, a.rowpos, a.rowci,
                                                                             a.status);
    if (a.posmap != nullptr && a.qk_rows > 0) {
      const int64_t wp = (a.qk_rows + threads - 1) / threads;
      posmap_kernel<<<(int)(wp < 148 * 8 ? wp : 148 * 8), threads, 0, s>>>(a.ht, a.qk_rows, a.sel, a.posmap,
                                                                          a.status);
    }
  }
  RopeFreqs f;
  for (int m = 0; m < kMaxHalfDim; ++m)
    f.omega[m] = (m < a.d / 2) ? pow(a.rope_theta, -2.0 * m / a.d) : 0.0;
  const float qscale = (float)(kLog2e / sqrt((double)a.d));
  constexpr int POS = 8;
  if (a.qk_rows > 0) {
    rope_qk_kernel<IT, QT, POS><<<(unsigned)((a.qk_rows + POS - 1) / POS), 256, 0, s>>>(
        static_cast<const IT*>(a.q), static_cast<const IT*>(a.k), a.qk_rows, a.posmap, a.hq, a.hkv, a.d, f,
        qscale, static_cast<QT*>(a.qr), static_cast<QT*>(a.kr), static_cast<IT*>(a.k_ret), a.kret_lo,
        a.ret_hi - a.ret_lo, a.status);
  }
  const size_t vrow = sizeof(IT) * (size_t)a.hkv * a.d;
  if (a.ret_hi > a.ret_lo) {
    const void* vsrc = static_cast<const char*>(a.v) + vrow * (size_t)a.ret_lo;
    if (a.v_ret != vsrc &&
        cudaMemcpyAsync(a.v_ret, vsrc, vrow * (size_t)(a.ret_hi - a.ret_lo), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
      return PA_ERR_CUDA;
  }
  const QT* kq = static_cast<const QT*>(a.kr);
  const dim3 grid(a.ht.tile_off[a.ht.n_hosts], a.hq);
  int rc = PA_OK;
  profile_begin(s);
  if (phase1_tc_supported(a)) {
    rc = launch_phase1_tc(a, s);
  } else if (grid.x > 0) {
    if (a.d == 128)
      phase1_simt_kernel<128, QT, VT, OT><<<grid, 256, 0, s>>>(
          static_cast<const QT*>(a.qr), kq, static_cast<const VT*>(a.v), a.rowpos, a.rowci, a.ht,
          a.hq, a.hkv, static_cast<OT*>(a.o), a.lse);
    else
      phase1_simt_kernel<64, QT, VT, OT><<<grid, 256, 0, s>>>(
          static_cast<const QT*>(a.qr), kq, static_cast<const VT*>(a.v), a.rowpos, a.rowci, a.ht,
          a.hq, a.hkv, static_cast<OT*>(a.o), a.lse);
  }
  // fp16-carried Q / K: the first rows of every host again in fp32
  if (rc == PA_OK && sizeof(QT) == 2 && a.ht.n_hosts > 0) {
    const dim3 hg(a.ht.n_hosts, a.hkv);
    if (a.d == 128)
      phase1_head_rows_kernel<128><<<hg, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
          static_cast<const __nv_bfloat16*>(a.v), a.rowpos, a.ht, a.hq, a.hkv, f, static_cast<__nv_bfloat16*>(a.o),
          a.lse);
    else
      phase1_head_rows_kernel<64><<<hg, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
          static_cast<const __nv_bfloat16*>(a.v), a.rowpos, a.ht, a.hq, a.hkv, f, static_cast<__nv_bfloat16*>(a.o),
          a.lse);
  }
  profile_end(s);
  if (rc != PA_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_phase1(const Phase1Args& a, cudaStream_t s) {
  if (a.dtype == PA_F32) return launch_phase1_t<float, float, float, float>(a, s);
  return launch_phase1_t<__nv_bfloat16, __half, __nv_bfloat16, __nv_bfloat16>(a, s);
}

}  // namespace pa
