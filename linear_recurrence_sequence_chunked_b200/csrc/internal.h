// internal.h -- host-side launchers shared between the library's .cu files.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace pdn {

// CUDA-core chunk kernel (any supported shape, fp32 math).
int simt_supported(const KParams &P);
cudaError_t launch_chunk_simt(const KParams &P, cudaStream_t stream);

// Tensor-core (tcgen05) chunk kernel: bf16 operands, fp32 state in TMEM.
int tc_supported(const KParams &P);
size_t tc_workspace_bytes(const KParams &P);
cudaError_t launch_chunk_tc(const KParams &P, void *workspace, cudaStream_t stream);

// Tensor-core three-kernel path: intra-chunk work for all chunks at once,
// then the sequential state pass; needs a workspace.
int split_supported(const KParams &P);
size_t split_workspace_bytes(const KParams &P);
cudaError_t launch_chunk_split(const KParams &P, void *workspace, cudaStream_t stream);

// One decode step (state streamed through once).
cudaError_t launch_decode(const KParams &P, cudaStream_t stream);

// Bounded-wait self test.
cudaError_t launch_selftest_wait(long long spin_limit, int *err, cudaStream_t stream);

}  // namespace pdn
