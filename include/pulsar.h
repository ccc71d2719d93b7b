/*
 * pulsar.h -- C ABI of the B200 (sm_100a) Star / Pulsar two-phase blockwise
 * attention path.
 *
 * Sources (web pages, cited by title and section):
 *  [P]  "Dropping the Anchor: Statistical Context Summarization for
 *       Distributed Systems via Pulsar Attention" (project page): §1 the
 *       anchor problem, §2 method, §2.1 Max-IDF selection, Figure 2,
 *       §2.2 query phase, §4 efficiency, §5 code and CLI flags.
 *  [PS] "Technische Samenvatting: Pulsar Attention", sections "Fase 1"
 *       (host input [S_sink || Sigma_0 .. Sigma_{i-1} || B_i], KV discard)
 *       and "Fase 2" (broadcast query, online-softmax merge).
 *  [S]  Star Attention machine review (arXiv 2411.17116): summary,
 *       key_machinery (anchor block with original positions, distributed
 *       log-sum-exp aggregation), referee minor comments (Algorithm 2 uses
 *       exp(s_h - s_global) * A_h; the first block has no anchor).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *    the argument is documented as a host pointer.  The library allocates
 *    nothing and keeps no state between calls.
 *  - Scratch memory is the caller's `ws` buffer of at least the size the
 *    matching *_workspace_size() returns, 256-byte aligned.  Its first 256
 *    bytes hold a status block that each call clears at its start and that
 *    kernels set when they detect an error on the device (see
 *    pa_workspace_status).  A workspace must not be shared by calls that may
 *    run concurrently.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    is stream-ordered and asynchronous: it validates its arguments on the
 *    host, enqueues kernels and returns; nothing synchronises the device
 *    except pa_workspace_status.
 *  - Tensors are dense, row-major, with the innermost dimension listed last,
 *    e.g. [L][H][d] means element (t, h, m) is at ((t * H) + h) * d + m.
 *  - dtype is PA_F32 (float) or PA_BF16 (bfloat16, stored as uint16).
 *  - Return value: PA_OK or a negative pa_status.  On a host-side error no
 *    kernel is launched and no output is written.
 */
#ifndef PULSAR_B200_H
#define PULSAR_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 1

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,     /* bad argument: NULL pointer, size mismatch, out-of-range id/index */
  PA_ERR_UNSUPPORTED = -2, /* valid but not implemented: dtype, head_dim, block count, alignment */
  PA_ERR_WORKSPACE = -3,   /* ws NULL, misaligned, or smaller than *_workspace_size() */
  PA_ERR_CUDA = -4,        /* a CUDA launch or memset failed */
  PA_ERR_TIMEOUT = -5,     /* a bounded device-side wait expired (device status only) */
  PA_ERR_RANGE = -6        /* a value left the range of an internal format (device status only) */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

/* Version of this ABI (PA_ABI_VERSION of the built library). */
int pa_abi_version(void);

/* Static text for a pa_status value. */
const char* pa_status_string(int status);

/*
 * Waits for `stream`, then returns the device status recorded in `ws` by the
 * last call that used this workspace: PA_OK, PA_ERR_INVALID (an id out of
 * [0, vocab) or a chunk index out of range met on the device), PA_ERR_RANGE
 * (a Phase-1 rotated Q/K value outside the fp16 range used internally for
 * bf16 inputs) or PA_ERR_TIMEOUT.  Returns PA_ERR_CUDA if the copy fails.  This
 * is the only synchronising call of the library.
 */
int pa_workspace_status(const void* ws, void* stream);

/*
 * Measurement hook.  When both arguments are non-NULL cudaEvent_t handles
 * (created by the caller), every later Phase-1 or Phase-2 call made from
 * this host thread records `start` on its stream right before its dominant
 * kernel (the attention kernel of Phase 1, the split-KV partial kernel of
 * Phase 2) and `stop` right after it.  (NULL, NULL) turns recording off.
 * Returns PA_ERR_INVALID if exactly one argument is NULL.
 */
int pa_set_profile_events(void* start, void* stop);

/* ------------------------------------------------------------------------ */
/* (a1-a3) Max-IDF summary selection        [P] §2.1, Figure 2; [PS] Fase 1 */
/* ------------------------------------------------------------------------ */

/* Bytes of scratch pulsar_select_summaries needs. 0 if arguments are invalid. */
size_t pa_select_workspace_size(int64_t L, int32_t vocab, int32_t block, int32_t chunk);

/*
 * Selects each block's summary: the context of L tokens is cut into
 * N = L / block contiguous blocks (the documents); df(t) is the number of
 * blocks containing token t; each block is cut into block / chunk
 * non-overlapping chunks scored by their rarest token,
 * max_t ln(N / df(t)) -- computed exactly as the integer min_t df(t), since
 * ln(N / df) is strictly decreasing in df; the k_chunks best chunks of every
 * block are kept in original order, equal scores going to the lower chunk
 * index.
 *
 *  ids            [L] int32 token ids, each in [0, vocab).
 *  L, block       L % block == 0, 1 <= N = L / block <= 64.
 *  chunk          block % chunk == 0.
 *  k_chunks       0 <= k_chunks <= block / chunk (the page's budget is
 *                 floor(0.125 * block / chunk)).
 *  sel            out [N][k_chunks] int32 local chunk indices, ascending.
 *  df_opt         out [vocab] int32 document frequency, or NULL.
 *  chunk_mindf_opt out [L / chunk] int32 min df of every chunk, or NULL.
 *
 * Errors: PA_ERR_INVALID for the size rules above or NULL ids/sel (sel may
 * be NULL only when k_chunks == 0); PA_ERR_UNSUPPORTED for N > 64.  An id
 * outside [0, vocab) is skipped and sets PA_ERR_INVALID in the workspace
 * status; the outputs are then unspecified.  Results are bit-exact and
 * deterministic.
 */
int pulsar_select_summaries(const int32_t* ids, int64_t L, int32_t vocab, int32_t block,
                            int32_t chunk, int32_t k_chunks, int32_t* sel, int32_t* df_opt,
                            int32_t* chunk_mindf_opt, void* ws, size_t ws_bytes, void* stream);

/* Chunk scorers of pulsar_select_summaries_scored. */
typedef enum {
  PA_SCORE_MAX_IDF = 0,       /* the method: max IDF over the chunk (= pulsar_select_summaries) */
  PA_SCORE_MEAN_IDF = 1,      /* mean IDF over the chunk's tokens */
  PA_SCORE_EVENLY_SPACED = 2, /* no score: chunks floor(m * C / k), m = 0..k-1, in every block */
  PA_SCORE_ENTROPY = 3,       /* Shannon entropy of the chunk's token frequencies */
  PA_SCORE_BM25 = 4           /* Okapi BM25 weight of the chunk over its own tokens */
} pa_score_method;

/*
 * Summary selection with another chunk scorer, for the scorer ablation of
 * [P] §3.1 (Table 1 compares Max-IDF with other statistical scores and with
 * non-statistical baselines; §2.1 contrasts the maximum with the mean).
 * Same sizes, rules, outputs and tie-break as pulsar_select_summaries.
 *  - PA_SCORE_MEAN_IDF ranks chunks by their mean IDF,
 *    (1/chunk) sum_t ln(N / df(t)), exactly: with a fixed chunk length the
 *    mean is ln N - ln(prod_t df(t)) / chunk, so the order is that of the
 *    integer product of df over the chunk (ascending), compared as exact
 *    256-bit integers; equal means go to the lower chunk index.  Requires
 *    chunk <= 32 and block / chunk <= 4096 (PA_ERR_UNSUPPORTED otherwise).
 *  - PA_SCORE_ENTROPY ranks chunks by -sum_t p_t ln p_t, p_t = tf(t) /
 *    chunk, exactly: the order is that of the integer prod_t tf^tf
 *    (ascending), compared as 256-bit integers.  Same limits as mean IDF.
 *  - PA_SCORE_BM25 ranks chunks by sum over their distinct tokens (in order
 *    of first occurrence) of ln(1 + (N - df + 0.5)/(df + 0.5)) *
 *    tf (k1 + 1)/(tf + k1), k1 = 1.2 (length normalisation 1: every chunk
 *    has the average length), in fp64; equal scores go to the lower index.
 *    Same limits as mean IDF.  (The pages name entropy and BM25 without
 *    formulas; these are the textbook definitions.)
 *  - PA_SCORE_EVENLY_SPACED does not read ids (may be NULL).
 *  chunk_score_opt  out [L / chunk] int64, or NULL: for PA_SCORE_MEAN_IDF,
 *                   PA_SCORE_ENTROPY and PA_SCORE_BM25 each chunk's rank in
 *                   its block's order (0 = best; the ranks of a block are a
 *                   permutation of 0 .. block/chunk - 1); for
 *                   PA_SCORE_MAX_IDF the min df; not written for
 *                   PA_SCORE_EVENLY_SPACED.
 * Workspace: pa_select_workspace_size.
 */
int pulsar_select_summaries_scored(const int32_t* ids, int64_t L, int32_t vocab, int32_t block,
                                   int32_t chunk, int32_t k_chunks, int method, int32_t* sel,
                                   int64_t* chunk_score_opt, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * Allocation-free variant of pulsar_select_summaries.  The paper has no
 * counterpart to this call: it exists for callers that cannot allocate
 * device memory -- e.g. a plugin inside a host application that owns every
 * device allocation, or a latency-critical serving thread that must never
 * call cudaMalloc (which may synchronise the whole device).  The caller
 * passes inputs and outputs only (same meaning, layout and results as
 * pulsar_select_summaries); the scratch lives in a fixed array inside this
 * library's device memory, which every GPU that loads the library keeps
 * until the process exits.
 *
 * Limits: vocab <= 262144 and L / chunk <= 65536 (PA_ERR_UNSUPPORTED
 * beyond), plus every rule of pulsar_select_summaries.  No cudaMalloc,
 * cudaFree or other allocating routine is called.
 * Set-up: the first call on a device looks up the array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture.  Every call reuses the same array and clears what must
 * start at zero, so calls that may overlap on the GPU (different streams, or
 * different host threads, without ordering between them) race with each
 * other and must be serialised by the caller.  Device-detected invalid ids
 * are skipped as in pulsar_select_summaries, but this call has no workspace
 * whose status could be read back: pass ids in [0, vocab).
 */
int pulsar_select_summaries_noalloc(const int32_t* ids, int64_t L, int32_t vocab, int32_t block,
                                    int32_t chunk, int32_t k_chunks, int32_t* sel, int32_t* df_opt,
                                    int32_t* chunk_mindf_opt, void* stream);

/* ------------------------------------------------------------------------ */
/* (a4-a5) Phase-1 context encoding   [PS] Fase 1; [P] §2, §2.1; [S] summary */
/* ------------------------------------------------------------------------ */

/*
 * Host row layout of Phase 1 (HOST pointer row_off, [N + 1] int64).
 * Host 0 encodes B_0 alone (n_0 = block).  Host i >= 1 encodes
 *   Pulsar (star == 0): [sink tokens || Sigma_0 || .. || Sigma_{i-1} || B_i],
 *                       n_i = sink + i * summary_tokens + block;
 *   Star   (star != 0): [B_0 || B_i], n_i = 2 * block.
 * row_off[i] is the first packed output row of host i, row_off[N] the total.
 * Returns PA_ERR_INVALID for L % block != 0, block <= 0, N < 1, sink > block
 * or summary_tokens > block.
 */
int pa_phase1_layout(int64_t L, int32_t block, int32_t sink, int32_t summary_tokens, int star,
                     int64_t* row_off);

/* Bytes of scratch the Phase-1 calls need (star selects the variant); enough
 * for the call over every host and for any host range. */
size_t pa_phase1_workspace_size(int64_t L, int32_t hq, int32_t hkv, int32_t d, int dtype,
                                int32_t block, int32_t sink, int32_t summary_tokens, int star);

/* Bytes of scratch a call over hosts [host_begin, host_end) needs (the
 * *_phase1_encode_hosts calls).  A range that reads few of the sequence's
 * positions rotates only those: the sink, the summaries of blocks
 * 0 .. host_end - 2 and its own blocks (Star: B_0 and its own blocks), so
 * its scratch scales with them, not with L.  0 for invalid arguments. */
size_t pa_phase1_hosts_workspace_size(int64_t L, int32_t hq, int32_t hkv, int32_t d, int dtype,
                                      int32_t block, int32_t sink, int32_t summary_tokens, int star,
                                      int32_t host_begin, int32_t host_end);

/*
 * Pulsar Phase-1 encoding of every host of one attention layer, all hosts
 * batched on this GPU.  Each row carries its ORIGINAL position id p; Q and
 * K are rotated (RoPE, rotate-half, omega_m = rope_theta^(-2m/d)) at p; host
 * i runs causal softmax attention over its concatenated rows (row r sees
 * rows c <= r); query head h reads kv head h / (hq / hkv).
 *
 *  q              [L][hq][d]  dtype, unrotated.
 *  k, v           [L][hkv][d] dtype, unrotated.
 *  L, block       as in pulsar_select_summaries.
 *  sink, chunk, k_chunks  sink % 16 == 0, chunk % 16 == 0, sink <= block,
 *                 k_chunks * chunk <= block.
 *  sel            [N][k_chunks] int32 device array from
 *                 pulsar_select_summaries (row N-1 is not read).
 *  o              out [row_off[N]][hq][d] dtype: every host row's output,
 *                 hosts packed in order (pa_phase1_layout).
 *  lse_opt        out [row_off[N]][hq] float: natural-log sum of exp of the
 *                 row's scaled scores, or NULL.
 *  k_ret, v_ret   out [N][block][hkv][d] dtype == [L][hkv][d]: the retained
 *                 cache -- only each host's own block survives, K rotated
 *                 at its positions, V unchanged ([P] §2.1, §2.2).  v_ret
 *                 may equal v (then it is not written).
 *
 * d must be 64 or 128, hq % hkv == 0.  For PA_BF16, rotated Q and K are
 * carried in fp16 for the QK^T product; P is rounded to bf16 for the PV
 * product; all sums are fp32.  The first 32 rows of every host (too few
 * visible keys to average the fp16 rounding out of their lse) are computed
 * again in fp32 from the bf16 inputs.  For PA_F32 the whole path is fp32.
 * Limit (bf16): a rotated Q value times log2(e)/sqrt(d), or a rotated K
 * value, beyond 65504 is refused through the device status PA_ERR_RANGE
 * (pa_workspace_status); the outputs are then unspecified.
 */
int pulsar_phase1_encode(const void* q, const void* k, const void* v, int dtype, int64_t L,
                         int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                         int32_t sink, int32_t chunk, int32_t k_chunks, const int32_t* sel,
                         void* o, float* lse_opt, void* k_ret, void* v_ret, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * Star Attention anchor variant of Phase 1 ([S] key_machinery): host i >= 1
 * encodes [B_0 || B_i] with B_0 at its original positions, host 0 encodes
 * B_0 alone.  Arguments and outputs as pulsar_phase1_encode; row layout
 * pa_phase1_layout(.., star = 1).
 */
int star_phase1_encode(const void* q, const void* k, const void* v, int dtype, int64_t L,
                       int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                       void* o, float* lse_opt, void* k_ret, void* v_ret, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * Phase 1 of a contiguous range of hosts, [host_begin, host_end) of the
 * sequence's N = L / block hosts: the unit of work of one GPU when the hosts
 * of one sequence are spread over GPUs ([P] §2.1, §2.2: each host encodes
 * its own input and keeps its own block's KV; no communication in Phase 1).
 * Inputs and arguments as pulsar_phase1_encode / star_phase1_encode (q, k,
 * v hold the whole sequence; only the positions the range's hosts read are
 * read and rotated: the sink, the summary chunks of blocks before host_end - 1
 * and the range's blocks, or B_0 and the range's blocks for Star).
 * Workspace: pa_phase1_hosts_workspace_size (pa_phase1_workspace_size is
 * always enough).  Outputs cover the range only:
 *  o, lse_opt     rows row_off[host_begin] .. row_off[host_end] of the full
 *                 layout (pa_phase1_layout), packed from row 0.
 *  k_ret, v_ret   [host_end - host_begin][block][hkv][d]: the range's blocks.
 * Results are bit-identical to the same rows of a call over every host.
 * 0 <= host_begin <= host_end <= N (PA_ERR_INVALID otherwise); an empty range
 * does nothing.
 */
int pulsar_phase1_encode_hosts(const void* q, const void* k, const void* v, int dtype, int64_t L,
                               int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                               int32_t sink, int32_t chunk, int32_t k_chunks, const int32_t* sel,
                               int32_t host_begin, int32_t host_end, void* o, float* lse_opt,
                               void* k_ret, void* v_ret, void* ws, size_t ws_bytes, void* stream);
int star_phase1_encode_hosts(const void* q, const void* k, const void* v, int dtype, int64_t L,
                             int32_t hq, int32_t hkv, int32_t d, double rope_theta, int32_t block,
                             int32_t host_begin, int32_t host_end, void* o, float* lse_opt,
                             void* k_ret, void* v_ret, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* (a6-a7) Phase-2 split-KV attention + exact LSE merge                     */
/*         [P] §2.2; [PS] Fase 2; [S] key_machinery, Algorithm 2 comment     */
/* ------------------------------------------------------------------------ */

/* Bytes of scratch star_phase2_attend needs. */
size_t pa_phase2_workspace_size(int32_t B, int32_t Tq, int64_t T, int32_t n_shards, int32_t hq,
                                int32_t hkv, int32_t d);

/*
 * Global query attention over a retained cache split into n_shards shards
 * (shard h = keys [h * ceil(T / n_shards), min((h + 1) * ceil(T / n_shards), T))).
 * Each shard yields a partial (A_h, s_h) = (softmax(q K_h^T / sqrt(d)) V_h,
 * ln sum exp(q K_h^T / sqrt(d))); the exact merge is
 * s = ln sum_h exp(s_h), O = sum_h exp(s_h - s) A_h.  Every key is visible.
 *
 *  q              [B][Tq][hq][d] dtype, unrotated; row j is rotated at
 *                 position q_pos0 + j when rope_theta > 0, used as given
 *                 otherwise.
 *  k_ret, v_ret   [B][T][hkv][d] dtype: batch element b has its own cache
 *                 (K already rotated, as written by Phase 1).
 *  o              out [B][Tq][hq][d] dtype.
 *  lse            out [B][Tq][hq] float.
 *  part_o_opt     out [B][n_shards][Tq][hq][d] float (A_h) or NULL.
 *  part_lse_opt   out [B][n_shards][Tq][hq] float (s_h) or NULL.
 *
 * An empty shard has s_h = -inf and A_h = 0; with T == 0, O = 0 and
 * lse = -inf.  d must be 64 or 128, hq % hkv == 0, 1 <= n_shards <= 4096.
 * When neither partial output is asked for and the query has more than 8
 * rows per kv head, or B * n_shards * hkv < 148, the work is cut into equal
 * key ranges regardless of shard boundaries (the merge is exact either way;
 * results differ only in fp32 rounding order).
 * Precision (bf16): on the tensor-core path (at least 64 query rows per kv
 * head, Tq * hq / hkv; hq / hkv dividing 128; 16-byte aligned caches) the
 * scores are computed from the rotated query rounded to fp16 against the
 * keys converted exactly to fp16; a work unit that meets a key beyond fp16
 * range (every unit, if a rotated query value times log2(e)/sqrt(d) is) is
 * recomputed in fp32 (bf16 keys widened exactly, fp32 sums), so every bf16
 * input is computed.  Otherwise
 * the scores come from a bf16 high part plus a bf16 residual of the query
 * (about 16 significant bits of the rotated query) against the stored keys,
 * summed in fp32.  P is rounded to bf16 for P V.
 */
int star_phase2_attend(const void* q, int dtype, int32_t B, int32_t Tq, int64_t q_pos0,
                       double rope_theta, const void* k_ret, const void* v_ret, int64_t T,
                       int32_t n_shards, int32_t hq, int32_t hkv, int32_t d, void* o, float* lse,
                       float* part_o_opt, float* part_lse_opt, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Phase-2 attention with run-time early termination of the key walk (NEXT
 * row; "ART: Attention Run-time Termination" review page: stop fetching
 * further KV blocks once a probe of the running output has been stable in
 * magnitude and direction for a patience window; defaults tau = 1e-5,
 * phi = 1e-3, patience = 5).  An approximation: its result is attention
 * over the keys visited.  For every (batch, kv head) group the cache is
 * walked from the newest key backwards in blocks of block_keys keys; after
 * block t >= 2 the step is stable when, for every query row of the group
 * (Tq tokens x the group's query heads), the normalised running output x_t
 * satisfies | |x_t| - |x_{t-1}| | <= tau |x_{t-1}| and 1 - cos(x_t, x_{t-1})
 * <= phi; the walk stops after `patience` consecutive stable steps.
 *  q              [B][Tq][hq][d] bf16 (rotated at q_pos0 + j when rope_theta > 0).
 *  k_ret, v_ret   [B][T][hkv][d] bf16, K rotated.
 *  o, lse         out: attention over the visited keys.
 *  visited_blocks_opt  out [B][hkv] int32: blocks walked, or NULL.
 * bf16 only; Tq * hq / hkv <= 8 (decode rows); block_keys a multiple of 32;
 * workspace pa_phase2_workspace_size(B, Tq, T, 1, hq, hkv, d).
 */
int star_phase2_attend_art(const void* q, int dtype, int32_t B, int32_t Tq, int64_t q_pos0,
                           double rope_theta, const void* k_ret, const void* v_ret, int64_t T,
                           int32_t hq, int32_t hkv, int32_t d, int32_t block_keys, double tau,
                           double phi, int32_t patience, void* o, float* lse,
                           int32_t* visited_blocks_opt, void* ws, size_t ws_bytes, void* stream);

/*
 * Exact merge of Phase-2 partials ([S] Algorithm 2 as corrected in the
 * referee's comment; [P] §2.2, where the hosts' partial results are
 * all-gathered and combined by an online softmax), for partials gathered
 * from several GPUs:
 * lse = ln sum_h exp(s_h), O = sum_h exp(s_h - lse) A_h.
 *  part_o    [B][S][Tq][hq][d] float (A_h, as star_phase2_attend writes it),
 *            16-byte aligned (PA_ERR_INVALID otherwise)
 *  part_lse  [B][S][Tq][hq] float (s_h; -inf marks an empty shard, whose
 *            A_h is then ignored)
 *  o         out [B][Tq][hq][d] dtype;  lse out [B][Tq][hq] float.
 * All shards empty: O = 0, lse = -inf.  No workspace.
 */
int pa_lse_merge(const float* part_o, const float* part_lse, int32_t B, int32_t S, int32_t Tq,
                 int32_t hq, int32_t d, int dtype, void* o, float* lse, void* stream);

/*
 * One step of the query host (NEXT row: query and generation loop).  The
 * query and the generated tokens attend globally ([S] summary: "only the
 * query and generated tokens attend globally"; [P] §5 --tokens_to_generate):
 * the Tq new tokens' K (rotated at q_pos0 + j) and V are appended to the
 * query host's own cache at rows self_len + j, then row j of q (rotated at
 * q_pos0 + j) attends to every key of the retained shards and, causally, to
 * own-cache rows 0 .. self_len + j; the result is merged exactly with the
 * shards'.  Calling it once with the query (self_len = 0) and then once per
 * generated token (Tq = 1, self_len growing) is the generation loop.
 *
 *  q, k_new, v_new  [B][Tq][hq | hkv | hkv][d] dtype, unrotated.
 *  k_self, v_self   in/out [B][self_cap][hkv][d] dtype, the own cache (K
 *                   rotated); self_len + Tq <= self_cap.
 *  o, lse           out as star_phase2_attend.
 * Other arguments, errors and workspace (pa_phase2_workspace_size) as
 * star_phase2_attend.
 */
int star_phase2_query_step(const void* q, const void* k_new, const void* v_new, int dtype, int32_t B,
                           int32_t Tq, int64_t q_pos0, double rope_theta, const void* k_ret,
                           const void* v_ret, int64_t T, int32_t n_shards, void* k_self, void* v_self,
                           int64_t self_cap, int64_t self_len, int32_t hq, int32_t hkv, int32_t d,
                           void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PULSAR_B200_H */
