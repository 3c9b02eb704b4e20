// noalloc.cu -- pdn_chunk_fwd_noalloc: the chunked forward's workspace path
// with its scratch in a fixed device array instead of caller-provided memory.
//
// Some callers have no way to obtain device memory for a workspace: code
// running under a framework whose allocator owns every device allocation and
// forbids raw cudaMalloc, latency-critical serving loops where cudaMalloc's
// implicit synchronisation is not acceptable, or plugins that are handed
// input/output buffers but no allocator. This entry point serves them: the
// scratch the tensor-core path needs lives in one file-scope device array,
// reserved by the CUDA driver when the library's device code is loaded on a GPU
// and held until the process exits.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

// Largest workspace the array can stand in for: 64 MiB, i.e. problems with
// B * H * ceil(T / 64) <= 809 (d_k = d_v = 128, bf16, chunk 64).
constexpr size_t kNoallocScratchBytes = 64ull << 20;

// One instance per device that loads the library.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the array on the current device. Host code cannot use
// the array's name as a device pointer (on the host it names a host-side
// stand-in), so the address is looked up once per device, with that device
// current, and cached.
void *scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace pdn

extern "C" pdn_status_t pdn_chunk_fwd_noalloc(const pdn_problem_t *p, const pdn_tensors_t *t,
                                              void *stream) {
  if (!p) return PDN_ERR_INVALID_ARG;
  pdn_problem_t q = *p;
  q.impl = PDN_IMPL_TC;  // the workspace-using tensor-core path
  const size_t need = pdn_chunk_fwd_workspace(&q);
  if (need == (size_t)-1) return PDN_ERR_INVALID_ARG;
  if (pdn_chunk_fwd_impl(&q) != PDN_IMPL_TC) return PDN_ERR_UNSUPPORTED;
  if (need > pdn::kNoallocScratchBytes) return PDN_ERR_WORKSPACE;  // problem too large
  void *scratch = pdn::scratch_on_current_device();
  if (!scratch) return PDN_ERR_CUDA;
  return pdn_chunk_fwd(&q, t, scratch, pdn::kNoallocScratchBytes, stream);
}
