// Max-IDF summary selection kernels (Pulsar Attention page, §2.1 and
// Figure 2; Dutch technical summary, "Fase 1").
//
// Integer formulation: the chunk score max_t ln(N / df(t)) is strictly
// decreasing in df, so ranking chunks by score equals ranking them by their
// minimum document frequency, with identical ties.  Everything here is
// integer arithmetic and bit-exact.
//
//  presence_tile_kernel : mask[t] |= 1 << j for every token t of block j
//                         (blocks are the documents); df(t) = popc(mask[t]);
//                         per-tile dedupe in shared memory (presence_mask_kernel
//                         for vocabularies above 2^20 ids).
//  chunk_mindf_kernel   : one warp per chunk, min over its tokens of df.
//  topk_kernel          : one CTA per block; histogram of min-df values
//                         (1..N) -> threshold -> ordered compaction that keeps
//                         the lowest-index chunks among equal scores.
#include "pa_internal.h"

namespace pa {

__global__ void presence_mask_kernel(const int32_t* __restrict__ ids, int64_t L, int32_t vocab,
                                     int32_t block, unsigned long long* __restrict__ mask,
                                     DeviceStatus* st) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // Warp-uniform loop so that every lane takes part in __match_any_sync.
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < L;
       base += stride) {
    const int64_t i = base + lane;
    const bool valid = i < L;
    const int t = valid ? ids[i] : 0;
    const int j = valid ? (int)(i / block) : 0;
    const bool ok = valid && t >= 0 && t < vocab;
    if (valid && !ok) set_status(st, PA_ERR_INVALID, (int)(i & 0x7fffffff), t);
    // Lanes holding the same (token, block) pair elect one leader, which
    // sets the block's bit unless it is already visible in L2.
    const unsigned long long key = ok ? (((unsigned long long)(unsigned)t << 6) | (unsigned)j)
                                      : ~0ull;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (ok && lane == __ffs(peers) - 1) {
      const unsigned long long bit = 1ull << j;
      if (!(ld_cg_u64(mask + t) & bit)) atomicOr(mask + t, bit);
    }
  }
}

// Presence with a per-CTA dedupe: CTA = one tile of up to `tile` consecutive
// ids inside one block (512 .. 4096 ids, about four CTAs per SM).  The tile's distinct ids are first
// collected in a shared-memory bitmap of the vocabulary, then each distinct
// id sets the block's bit in global memory once.  With Zipf-distributed ids
// the frequent ids would otherwise send most of the tile's requests to the
// same few global words.
constexpr size_t kPresenceSmemMax = 128 * 1024;   // vocabularies up to 2^20 ids

__global__ void __launch_bounds__(256) presence_tile_kernel(const int32_t* __restrict__ ids, int64_t L,
                                                            int32_t vocab, int32_t block, int32_t tile,
                                                            unsigned long long* __restrict__ mask,
                                                            DeviceStatus* st) {
  extern __shared__ uint32_t bm[];   // [ceil(vocab / 32)]
  const int words = (vocab + 31) >> 5;
  const int tiles_per_block = (block + tile - 1) / tile;
  const int j = blockIdx.x / tiles_per_block;
  const int64_t i0 = (int64_t)j * block + (int64_t)(blockIdx.x % tiles_per_block) * tile;
  const int64_t i1 = min(min(i0 + tile, (int64_t)(j + 1) * block), L);
  for (int w = threadIdx.x; w < words; w += blockDim.x) bm[w] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  // warp-uniform loop: lanes with equal ids elect one leader (__match_any_sync)
  for (int64_t base = i0 + (threadIdx.x & ~31); base < i1; base += blockDim.x) {
    const int64_t i = base + lane;
    const bool valid = i < i1;
    const int t = valid ? ids[i] : 0;
    const bool ok = valid && t >= 0 && t < vocab;
    if (valid && !ok) set_status(st, PA_ERR_INVALID, (int)(i & 0x7fffffff), t);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? t : -1);
    if (ok && lane == __ffs(peers) - 1) atomicOr(&bm[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  // one atomic OR per distinct id of the tile; its result is unused, so it is
  // issued without waiting for it and the tile's ORs overlap in flight
  const unsigned long long bit = 1ull << j;
  for (int w = threadIdx.x; w < words; w += blockDim.x) {
    uint32_t x = bm[w];
    while (x) {
      const int t = (w << 5) + __ffs(x) - 1;
      x &= x - 1u;
      atomicOr(mask + t, bit);
    }
  }
}

__global__ void df_from_mask_kernel(const unsigned long long* __restrict__ mask, int32_t vocab,
                                    int32_t* __restrict__ df) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < vocab;
       t += (int64_t)gridDim.x * blockDim.x)
    df[t] = __popcll(mask[t]);
}

__global__ void chunk_mindf_kernel(const int32_t* __restrict__ ids, int64_t n_chunks,
                                   int32_t chunk, int32_t vocab,
                                   const unsigned long long* __restrict__ mask,
                                   int32_t* __restrict__ mindf) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < n_chunks;
       c += nwarps) {
    unsigned best = 0xffffffffu;
    const int32_t* tok = ids + c * chunk;
    for (int u = lane; u < chunk; u += 32) {
      const int t = tok[u];
      if (t >= 0 && t < vocab) best = min(best, (unsigned)__popcll(mask[t]));
    }
    best = __reduce_min_sync(0xffffffffu, best);
    if (lane == 0) mindf[c] = (int32_t)best;  // all-invalid chunk -> -1 (status already set)
  }
}

// Exclusive block-wide prefix count of `flag`; also returns the tile total.
template <int THREADS>
__device__ __forceinline__ int block_exclusive_count(bool flag, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned b = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(b & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(b);
  __syncthreads();
  int before = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < THREADS / 32; ++w) {
    const int x = warp_tot[w];
    before += (w < warp) ? x : 0;
    sum += x;
  }
  __syncthreads();  // warp_tot is reused by the next call
  *total = sum;
  return before + in_warp;
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS) topk_kernel(const int32_t* __restrict__ mindf,
                                                       int32_t C, int32_t k, int32_t n_blocks,
                                                       int32_t* __restrict__ sel) {
  constexpr int kBins = 66;  // 1..64 valid df values, 65 = invalid entry
  __shared__ int hist[kBins];
  __shared__ int warp_tot[THREADS / 32];
  __shared__ int s_tau, s_need;
  const int j = blockIdx.x;
  const int32_t* md = mindf + (int64_t)j * C;
  for (int i = threadIdx.x; i < kBins; i += THREADS) hist[i] = 0;
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += THREADS) {
    int v = md[c];
    if (v < 1 || v > n_blocks) v = 65;
    atomicAdd(&hist[v], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Threshold tau: the smallest df value at which the k-th best chunk sits;
    // every chunk below tau is kept, plus the first `need` chunks equal to tau.
    int tau = 0, need = 0, cum = 0;
    if (k > 0) {
      for (int v = 1; v < kBins; ++v) {
        if (cum + hist[v] >= k) { tau = v; need = k - cum; break; }
        cum += hist[v];
      }
    }
    s_tau = tau;
    s_need = need;
  }
  __syncthreads();
  const int tau = s_tau, need = s_need;
  int base_eq = 0, base_sel = 0;
  for (int base = 0; base < C; base += THREADS) {
    const int c = base + threadIdx.x;
    int v = kBins;
    if (c < C) {
      v = md[c];
      if (v < 1 || v > n_blocks) v = 65;
    }
    const bool eq = (c < C) && v == tau;
    const bool less = (c < C) && v < tau;
    int tot_eq, tot_sel;
    const int eq_rank = base_eq + block_exclusive_count<THREADS>(eq, warp_tot, &tot_eq);
    const bool take = less || (eq && eq_rank < need);
    const int pos = base_sel + block_exclusive_count<THREADS>(take, warp_tot, &tot_sel);
    if (take) sel[(int64_t)j * k + pos] = c;
    base_eq += tot_eq;
    base_sel += tot_sel;
  }
}

// ---------------------------------------------------------------------------
// Alternative scorers (Pulsar Attention page §3.1, Table 1).
//  Mean IDF.  Every chunk holds the same number c of tokens, so
//    mean IDF = (1/c) sum_t ln(N / df(t)) = ln N - (1/c) ln prod_t df(t):
//  a higher mean is exactly a smaller product of df, and equal means are
//  exactly equal products.  The product of at most 32 values in 1..64 is
//  below 2^193, so it is kept exactly as a 256-bit integer (four 64-bit
//  limbs, least significant first) and chunks are ranked by it.
//  chunk_df_product_kernel: one warp per chunk, product tree in 64 bits over
//    groups of 8 lanes (at most 2^48 each), then four multiword products.
//  rank_kernel: the rank of a chunk in its block is the number of chunks
//    with a smaller key, or an equal key and a lower index (a permutation of
//    0..C-1); a chunk is kept when its rank is below k.  Without a rank
//    output the count stops at k.
//  select_by_rank_kernel: ordered compaction of the chunks with rank < k.
//  Entropy.  With a fixed chunk length c, H = ln c - (1/c) sum_t tf ln tf, so
//    a higher entropy is exactly a smaller prod_t tf^tf, and that product is
//    the product over the chunk's positions of their token's frequency in
//    the chunk (a 256-bit key as above, __match_any_sync counting).
//  BM25.  fp64 sum over the chunk's distinct tokens, in order of first
//    occurrence, of idf(df) * tf (k1 + 1) / (tf + k1), k1 = 1.2 (the length
//    normalisation is 1: every chunk has the average length); ranked by
//    that score, descending.
//  evenly_spaced_kernel: chunk floor(m * C / k) in every block.
// ---------------------------------------------------------------------------
struct Key256 {
  unsigned long long w[4];
};

__device__ __forceinline__ void key_mul_small(Key256& a, unsigned long long f) {
  unsigned long long carry = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long lo = a.w[i] * f;
    const unsigned long long hi = __umul64hi(a.w[i], f);
    const unsigned long long sum = lo + carry;
    carry = hi + (sum < lo ? 1ull : 0ull);
    a.w[i] = sum;
  }
}

__device__ __forceinline__ bool key_less(const Key256& a, const Key256& b) {
#pragma unroll
  for (int i = 3; i >= 0; --i)
    if (a.w[i] != b.w[i]) return a.w[i] < b.w[i];
  return false;
}

__device__ __forceinline__ bool key_equal(const Key256& a, const Key256& b) {
  return a.w[0] == b.w[0] && a.w[1] == b.w[1] && a.w[2] == b.w[2] && a.w[3] == b.w[3];
}

__global__ void chunk_df_product_kernel(const int32_t* __restrict__ ids, int64_t n_chunks, int32_t chunk,
                                        int32_t vocab, const unsigned long long* __restrict__ mask,
                                        Key256* __restrict__ key) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < n_chunks;
       c += nwarps) {
    unsigned long long f = 1;   // lanes past the chunk, and invalid ids, contribute 1
    if (lane < chunk) {
      const int t = ids[c * chunk + lane];
      if (t >= 0 && t < vocab) f = (unsigned long long)__popcll(mask[t]);
    }
    // products of 8 consecutive lanes: at most 64^8 = 2^48
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) f *= __shfl_xor_sync(0xffffffffu, f, off);
    const unsigned long long p8 = __shfl_sync(0xffffffffu, f, 8);
    const unsigned long long p16 = __shfl_sync(0xffffffffu, f, 16);
    const unsigned long long p24 = __shfl_sync(0xffffffffu, f, 24);
    if (lane == 0) {
      Key256 k;
      k.w[0] = f;
      k.w[1] = k.w[2] = k.w[3] = 0;
      key_mul_small(k, p8);
      key_mul_small(k, p16);
      key_mul_small(k, p24);
      key[c] = k;
    }
  }
}

// chunk entropy key: prod over the chunk's positions of tf(token) (= prod_t tf^tf)
__global__ void chunk_tf_product_kernel(const int32_t* __restrict__ ids, int64_t n_chunks, int32_t chunk,
                                        Key256* __restrict__ key) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < n_chunks;
       c += nwarps) {
    // lanes past the chunk get keys no token has, and contribute 1
    const int t = lane < chunk ? ids[c * chunk + lane] : 0;
    const unsigned long long tk = lane < chunk ? (unsigned long long)(unsigned)t
                                               : (0x100000000ull | (unsigned)lane);
    const unsigned peers = __match_any_sync(0xffffffffu, tk);
    unsigned long long f = lane < chunk ? (unsigned long long)__popc(peers) : 1ull;
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) f *= __shfl_xor_sync(0xffffffffu, f, off);
    const unsigned long long p8 = __shfl_sync(0xffffffffu, f, 8);
    const unsigned long long p16 = __shfl_sync(0xffffffffu, f, 16);
    const unsigned long long p24 = __shfl_sync(0xffffffffu, f, 24);
    if (lane == 0) {
      Key256 k;
      k.w[0] = f;
      k.w[1] = k.w[2] = k.w[3] = 0;
      key_mul_small(k, p8);
      key_mul_small(k, p16);
      key_mul_small(k, p24);
      key[c] = k;
    }
  }
}

// chunk BM25 score (fp64), summed in lane order over first occurrences
__global__ void chunk_bm25_kernel(const int32_t* __restrict__ ids, int64_t n_chunks, int32_t chunk, int32_t vocab,
                                  int32_t n_blocks, const unsigned long long* __restrict__ mask,
                                  double* __restrict__ score) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  constexpr double k1 = 1.2;
  for (int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < n_chunks;
       c += nwarps) {
    const int t = lane < chunk ? ids[c * chunk + lane] : 0;
    const unsigned long long tk = lane < chunk ? (unsigned long long)(unsigned)t
                                               : (0x100000000ull | (unsigned)lane);
    const unsigned peers = __match_any_sync(0xffffffffu, tk);
    double term = 0.0;
    if (lane < chunk && lane == __ffs(peers) - 1 && t >= 0 && t < vocab) {
      const double d = (double)__popcll(mask[t]);
      const double tf = (double)__popc(peers);
      const double idf = log(1.0 + ((double)n_blocks - d + 0.5) / (d + 0.5));
      term = idf * (tf * (k1 + 1.0)) / (tf + k1);
    }
    double total = 0.0;
    for (int l = 0; l < 32; ++l) total += __shfl_sync(0xffffffffu, term, l);   // lane order
    if (lane == 0) score[c] = total;
  }
}

// a better than b: a smaller 256-bit key (mean IDF, entropy) ...
__device__ __forceinline__ bool key_better(const Key256& a, const Key256& b) { return key_less(a, b); }
__device__ __forceinline__ bool key_same(const Key256& a, const Key256& b) { return key_equal(a, b); }
// ... or a larger score (BM25)
__device__ __forceinline__ bool key_better(double a, double b) { return a > b; }
__device__ __forceinline__ bool key_same(double a, double b) { return a == b; }

// grid (ceil(C / 256), n_blocks); the block's keys are staged in shared memory.
template <typename K>
__global__ void __launch_bounds__(256) rank_kernel(const K* __restrict__ key, int32_t C, int32_t k,
                                                   int32_t* __restrict__ rank,
                                                   long long* __restrict__ rank_out) {
  extern __shared__ __align__(16) uint8_t sk_raw[];
  K* sk = reinterpret_cast<K*>(sk_raw);
  const int j = blockIdx.y;
  const K* kb = key + (int64_t)j * C;
  for (int o = threadIdx.x; o < C; o += blockDim.x) sk[o] = kb[o];
  __syncthreads();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  const K v = sk[c];
  const int stop = rank_out != nullptr ? C : k;   // the count only decides rank < k
  int better = 0;
  for (int o = 0; o < C && better < stop; ++o) {
    const K w = sk[o];
    better += key_better(w, v) || (o < c && key_same(w, v));
  }
  rank[(int64_t)j * C + c] = better;
  if (rank_out != nullptr) rank_out[(int64_t)j * C + c] = better;
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS) select_by_rank_kernel(const int32_t* __restrict__ rank, int32_t C,
                                                                 int32_t k, int32_t* __restrict__ sel) {
  __shared__ int warp_tot[THREADS / 32];
  const int j = blockIdx.x;
  int base_sel = 0;
  for (int base = 0; base < C; base += THREADS) {
    const int c = base + threadIdx.x;
    const bool take = c < C && rank[(int64_t)j * C + c] < k;
    int tot;
    const int pos = base_sel + block_exclusive_count<THREADS>(take, warp_tot, &tot);
    if (take) sel[(int64_t)j * k + pos] = c;
    base_sel += tot;
  }
}

__global__ void evenly_spaced_kernel(int32_t n_blocks, int32_t C, int32_t k, int32_t* __restrict__ sel) {
  const int64_t n = (int64_t)n_blocks * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(i % k);
    sel[i] = (int32_t)(((int64_t)m * C) / k);
  }
}

// mask[t] = the set of blocks containing t (zeroed first)
static int launch_presence(const SelectArgs& a, cudaStream_t s) {
  if (cudaMemsetAsync(a.mask, 0, sizeof(unsigned long long) * (size_t)a.vocab, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (a.L <= 0) return PA_OK;
  const int threads = 256;
  const size_t bm_bytes = sizeof(uint32_t) * (size_t)((a.vocab + 31) / 32);
  if (bm_bytes <= kPresenceSmemMax) {
    int64_t tile = a.L / (4 * 148);
    tile = tile < 512 ? 512 : (tile > 4096 ? 4096 : (tile + 255) / 256 * 256);
    const int tiles_per_block = (int)((a.block + tile - 1) / tile);
    const int64_t n_tiles = (int64_t)(a.L / a.block) * tiles_per_block;
    if (bm_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(presence_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bm_bytes) !=
            cudaSuccess)
      return PA_ERR_CUDA;
    presence_tile_kernel<<<(unsigned)n_tiles, threads, bm_bytes, s>>>(a.ids, a.L, a.vocab, a.block, (int)tile,
                                                                     a.mask, a.status);
  } else {
    const int64_t want = (a.L + threads - 1) / threads;
    presence_mask_kernel<<<(int)(want < 148 * 16 ? want : 148 * 16), threads, 0, s>>>(a.ids, a.L, a.vocab,
                                                                                      a.block, a.mask, a.status);
  }
  return PA_OK;
}

int launch_select_scored(const SelectArgs& a, int method, void* key_ws, long long* rank_out,
                         cudaStream_t s) {
  const int64_t n_chunks = a.L / a.chunk;
  const int C = a.block / a.chunk;
  const int n_blocks = (int)(a.L / a.block);
  if (method == PA_SCORE_EVENLY_SPACED) {
    if (a.k > 0) {
      const int64_t n = (int64_t)n_blocks * a.k;
      evenly_spaced_kernel<<<(int)((n + 255) / 256), 256, 0, s>>>(n_blocks, C, a.k, a.sel);
    }
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  int rc = method == PA_SCORE_ENTROPY ? PA_OK : launch_presence(a, s);
  if (rc) return rc;
  const int threads = 256;
  const int64_t wgrid = (n_chunks * 32 + threads - 1) / threads;
  const int wblocks = (int)(wgrid < 148 * 32 ? wgrid : 148 * 32);
  if (method == PA_SCORE_MEAN_IDF)
    chunk_df_product_kernel<<<wblocks, threads, 0, s>>>(a.ids, n_chunks, a.chunk, a.vocab, a.mask,
                                                        static_cast<Key256*>(key_ws));
  else if (method == PA_SCORE_ENTROPY)
    chunk_tf_product_kernel<<<wblocks, threads, 0, s>>>(a.ids, n_chunks, a.chunk, static_cast<Key256*>(key_ws));
  else
    chunk_bm25_kernel<<<wblocks, threads, 0, s>>>(a.ids, n_chunks, a.chunk, a.vocab, n_blocks, a.mask,
                                                  static_cast<double*>(key_ws));
  if (a.k > 0 || rank_out != nullptr) {
    const dim3 grid((unsigned)((C + 255) / 256), (unsigned)n_blocks);
    if (method == PA_SCORE_BM25) {
      const size_t sm = sizeof(double) * (size_t)C;
      if (cudaFuncSetAttribute(rank_kernel<double>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
          cudaSuccess)
        return PA_ERR_CUDA;
      rank_kernel<double><<<grid, 256, sm, s>>>(static_cast<double*>(key_ws), C, a.k, a.mindf, rank_out);
    } else {
      const size_t sm = sizeof(Key256) * (size_t)C;
      if (cudaFuncSetAttribute(rank_kernel<Key256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
          cudaSuccess)
        return PA_ERR_CUDA;
      rank_kernel<Key256><<<grid, 256, sm, s>>>(static_cast<Key256*>(key_ws), C, a.k, a.mindf, rank_out);
    }
  }
  if (a.k > 0) select_by_rank_kernel<1024><<<n_blocks, 1024, 0, s>>>(a.mindf, C, a.k, a.sel);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

__global__ void widen_i32_kernel(const int32_t* __restrict__ in, long long* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = in[i];
}

int launch_widen_i32(const int32_t* in, long long* out, int64_t n, cudaStream_t s) {
  if (n > 0) {
    const int64_t want = (n + 255) / 256;
    widen_i32_kernel<<<(int)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(in, out, n);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_select(const SelectArgs& a, cudaStream_t s) {
  const int64_t n_chunks = a.L / a.chunk;
  const int C = a.block / a.chunk;
  const int n_blocks = (int)(a.L / a.block);
  int rc = launch_presence(a, s);
  if (rc) return rc;
  if (a.L > 0) {
    const int threads = 256;
    const int64_t wwarps = n_chunks;
    const int64_t wgrid = (wwarps * 32 + threads - 1) / threads;
    chunk_mindf_kernel<<<(int)(wgrid < 148 * 32 ? wgrid : 148 * 32), threads, 0, s>>>(
        a.ids, n_chunks, a.chunk, a.vocab, a.mask, a.mindf);
    if (a.k > 0) topk_kernel<1024><<<n_blocks, 1024, 0, s>>>(a.mindf, C, a.k, n_blocks, a.sel);
  }
  if (a.df_out) {
    const int threads = 256;
    const int64_t want = ((int64_t)a.vocab + threads - 1) / threads;
    df_from_mask_kernel<<<(int)(want < 148 * 8 ? want : 148 * 8), threads, 0, s>>>(
        a.mask, a.vocab, a.df_out);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
