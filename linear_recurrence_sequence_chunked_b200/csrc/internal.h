// internal.h -- host-side launchers shared between the library's .cu files.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace pdn {

// CUDA-core chunk kernel (any supported shape, fp32 math).
int simt_supported(const KParams &P);
cudaError_t launch_chunk_simt(const KParams &P, cudaStream_t stream);

// Tensor-core three-kernel path: intra-chunk work for all chunks at once,
// then the sequential state pass; needs a workspace.
int split_supported(const KParams &P);
size_t split_workspace_bytes(const KParams &P);
// `ev` (optional, four events) is recorded before the key-energy kernels,
// before the intra-chunk kernel, before the state kernel and after it.
cudaError_t launch_chunk_split(const KParams &P, void *workspace, cudaStream_t stream,
                               cudaEvent_t *ev = nullptr);

// Sequence-parallel pieces: AT = A0 + sum_t k.k per (batch, head); and
// S_out = S_in A + B_add per (batch, head) (S_in, B_add may be NULL = zero).
cudaError_t launch_key_energy(const KParams &P, cudaStream_t stream);
cudaError_t launch_compose(int BH, int dv, int dk, const float *S_in, const float *A,
                           const float *Badd, float *S_out, cudaStream_t stream);
cudaError_t launch_accumulate(int n, long long len, const float *parts, const float *base,
                              float *out, cudaStream_t stream);

// One decode step (state streamed through once).
cudaError_t launch_decode(const KParams &P, cudaStream_t stream);

// Multiprocessors of the current device (cached per device).
int num_sms();

// Every check pdn_chunk_fwd makes before it enqueues work (host-only);
// on PDN_OK, *impl_out (if non-NULL) is the path it would run.
pdn_status_t check_chunk_fwd(const pdn_problem_t *p, const pdn_tensors_t *t,
                             const void *workspace, size_t ws_bytes, int *impl_out);

// Backward (gradient of the chunked forward): workspace bytes, and the
// enqueue of every kernel of it (CUDA cores, fp32).
size_t bwd_workspace_bytes(const KParams &P);
cudaError_t launch_chunk_bwd(const KParams &P, const pdn_grads_t *g, void *workspace,
                             cudaStream_t stream);

// Bounded-wait self test.
cudaError_t launch_selftest_wait(long long limit_ns, int *err, cudaStream_t stream);

}  // namespace pdn
