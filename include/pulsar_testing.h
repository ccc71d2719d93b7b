/*
 * pulsar_testing.h -- test hooks of libpulsar_b200.so (not part of the
 * computation; used by the test suite to exercise failure detection).
 */
#ifndef PULSAR_B200_TESTING_H
#define PULSAR_B200_TESTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Runs star_phase1_encode on bf16 inputs through the tensor-core kernel
 * with every bounded device wait limited to wait_limit_us microseconds
 * (1 .. 10^7) and one barrier made unsatisfiable: each CTA's Q barrier
 * expects 16 bytes more than its copies deliver.  Every wait that depends
 * on it runs out, the CTA records PA_ERR_TIMEOUT in the workspace status
 * block, drains its copies and MMAs, frees its tensor memory and returns;
 * no memory is accessed out of bounds and the CUDA context stays usable.
 * Arguments as star_phase1_encode (dtype bf16, lse not written); the outputs
 * are unspecified.  Returns PA_ERR_UNSUPPORTED unless hq / hkv is even.
 */
int pa_testing_phase1_stall(const void* q, const void* k, const void* v, int64_t L, int32_t hq,
                            int32_t hkv, int32_t d, int32_t block, void* o, void* k_ret,
                            void* v_ret, void* ws, size_t ws_bytes, int32_t wait_limit_us,
                            void* stream);

/*
 * Runs star_phase2_attend on bf16 inputs (query used as given, no RoPE)
 * through the tensor-core query kernel with every bounded device wait
 * limited to wait_limit_us microseconds (1 .. 10^7) and its Q barrier made
 * unsatisfiable in the same way.  Every CTA records PA_ERR_TIMEOUT, drains
 * its copies and MMAs, frees its tensor memory and returns; the context
 * stays usable.  Arguments as star_phase2_attend (no partials); the outputs
 * are unspecified.  Returns PA_ERR_UNSUPPORTED unless the inputs take the
 * tensor-core path (at least 64 query rows per kv head, hq / hkv dividing
 * 128, 16-byte aligned caches).
 */
int pa_testing_phase2_stall(const void* q, const void* k_ret, const void* v_ret, int32_t B, int32_t Tq,
                            int64_t T, int32_t n_shards, int32_t hq, int32_t hkv, int32_t d, void* o,
                            float* lse, void* ws, size_t ws_bytes, int32_t wait_limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PULSAR_B200_TESTING_H */
