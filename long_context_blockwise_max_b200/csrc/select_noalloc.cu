// Max-IDF summary selection without a caller workspace.
//
// Some callers of this library cannot allocate device memory: a plugin
// living inside a host application that owns every device allocation, or a
// latency-critical serving thread that must never call cudaMalloc (which
// may synchronise the device).  pulsar_select_summaries_noalloc serves
// them: it runs the same selection kernels as pulsar_select_summaries, but
// its scratch (status block, per-token block masks and chunk min-df values)
// lives in a fixed array in this library's own device memory.  That array
// is sized for at most kNoAllocMaxVocab token ids and kNoAllocMaxChunks
// chunks, and every GPU that loads the library holds it until the process
// exits.
#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

constexpr int32_t kNoAllocMaxVocab = 262144;   // 2 MiB of 64-bit block masks
constexpr int64_t kNoAllocMaxChunks = 65536;   // 256 KiB of min-df values
constexpr size_t kNoAllocBytes =
    kStatusBytes + sizeof(unsigned long long) * kNoAllocMaxVocab + sizeof(int32_t) * kNoAllocMaxChunks;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device
// address).  Returns nullptr on failure.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pulsar_select_summaries_noalloc(const int32_t* ids, int64_t L, int32_t vocab,
                                               int32_t block, int32_t chunk, int32_t k_chunks,
                                               int32_t* sel, int32_t* df_opt,
                                               int32_t* chunk_mindf_opt, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L <= 0 || vocab <= 0 || block <= 0 || chunk <= 0) return PA_ERR_INVALID;
  if (L % block != 0 || block % chunk != 0) return PA_ERR_INVALID;
  if (k_chunks < 0 || k_chunks > block / chunk) return PA_ERR_INVALID;
  if (ids == nullptr || (sel == nullptr && k_chunks > 0)) return PA_ERR_INVALID;
  if (L / block > kMaxBlocks) return PA_ERR_UNSUPPORTED;
  if (vocab > kNoAllocMaxVocab || L / chunk > kNoAllocMaxChunks) return PA_ERR_UNSUPPORTED;
  char* w = static_cast<char*>(scratch_on_current_device());
  if (w == nullptr) return PA_ERR_CUDA;
  // The array keeps the previous call's contents: clear the status block
  // (launch_select clears the block masks it uses).
  if (cudaMemsetAsync(w, 0, kStatusBytes, s) != cudaSuccess) return PA_ERR_CUDA;
  SelectArgs a;
  a.ids = ids; a.L = L; a.vocab = vocab; a.block = block; a.chunk = chunk; a.k = k_chunks;
  a.sel = sel; a.df_out = df_opt;
  a.status = reinterpret_cast<DeviceStatus*>(w);
  a.mask = reinterpret_cast<unsigned long long*>(w + kStatusBytes);
  a.mindf = chunk_mindf_opt ? chunk_mindf_opt
                            : reinterpret_cast<int32_t*>(w + kStatusBytes +
                                                         sizeof(unsigned long long) * kNoAllocMaxVocab);
  return launch_select(a, s);
}
