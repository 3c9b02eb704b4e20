// common.cuh -- device helpers shared by the kernels of the gated delta-rule
// library (parameter block, element loads, variant rules, preconditioner).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pdn.h"

namespace pdn {

// Everything a kernel needs, passed by value.
struct KParams {
  int B, T, H, dk, dv, chunk;
  int variant, decay, dtype;
  float q_scale, x, lnx, eps;
  int prologue;       // PDN_PRO_* bits
  float decay_scale;  // PDN_PRO_DECAY_SOFTPLUS
  // Segment transition mode (pdn_chunk_transition): the targets u are zero,
  // the state starts from the identity (d_v = d_k) and no output is written,
  // so the final state is prod_t Diag(alpha_t) (I - r_t w_t^T).
  int transition;
  const void *q, *k, *v, *log_alpha, *beta, *erase, *write;
  const float *S0;
  float *ST;
  const float *A0;
  float *AT;
  void *o;
  // Training mode (tensor-core state pass; NULL = off): every token's delta
  // [B*H][T][d_v] and the state at the start of every chunk, transposed
  // [B*H][ceil(T/64)][d_k][d_v], both fp32, for the backward to reuse.
  float *sv_delta, *sv_ckpt;
  int *err;  // per-device error word (first error wins)
};

// Variants with the diagonal preconditioner (accumulator A, coefficients B).
__host__ __device__ constexpr bool is_precond(int variant) {
  return variant == PDN_VAR_PDN || variant == PDN_VAR_PGDN || variant == PDN_VAR_PKDA ||
         variant == PDN_VAR_PLA;
}
// Variants whose gain beta is one fp32 scalar per (token, head).
__host__ __device__ constexpr bool has_scalar_beta(int variant) {
  return variant != PDN_VAR_FG2_GDN && variant != PDN_VAR_GDN2 && variant != PDN_VAR_FG2_GDN_PLUS;
}

// Element load as fp32 from a tensor of the problem dtype.
template <typename T>
__device__ __forceinline__ float ldf(const void *p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const void *p, size_t i) {
  return __ldg(reinterpret_cast<const float *>(p) + i);
}
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const void *p, size_t i) {
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
}

template <typename T>
__device__ __forceinline__ void stf(void *p, size_t i, float x);
template <>
__device__ __forceinline__ void stf<float>(void *p, size_t i, float x) {
  reinterpret_cast<float *>(p)[i] = x;
}
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(void *p, size_t i, float x) {
  reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
}

// Flat index of token (b, t, h) in a [B,T,H] tensor.
__device__ __forceinline__ size_t tok_index(const KParams &P, int b, int t, int h) {
  return ((size_t)b * P.T + t) * P.H + h;
}

// Stabilised diagonal preconditioner coefficient ("Preconditioned DeltaNet",
// ja §2.2 / fr §2.C): c = log(A + eps) - mean_i log(A_i + eps) is squashed to
// s = c / (1 + |c|) in (-1, 1) and mapped to B = x^(-s) in [1/x, x].
// `logA` is log(A + eps) for this channel, `mu` the per-token channel mean.
__device__ __forceinline__ float precond_coef(float logA, float mu, float lnx) {
  const float c = logA - mu;
  const float s = c / (1.0f + fabsf(c));
  return expf(-s * lnx);
}

// ---- fused prologue (PDN_PRO_* bits) -----------------------------------
// softplus(x) = log(1 + e^x), written as max(x, 0) + log(1 + e^{-|x|}) so
// that neither exponential overflows.
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
// The activations themselves live out of line: the kernels call them per
// element inside fully unrolled loops, and inlined copies of expf / log1pf
// there would multiply the code every block has to fetch even when the
// prologue is off (a uniform branch skips the call).
static __device__ __noinline__ float sigmoid_call(float x) { return 1.f / (1.f + expf(-x)); }
static __device__ __noinline__ float decay_act_call(int prologue, float decay_scale, float x) {
  if (prologue & PDN_PRO_DECAY_SOFTPLUS) return -decay_scale * softplus_f(x);
  return -softplus_f(-x);
}
// A gate or gain as the kernels use it: sigmoid of the input when the
// problem's gates arrive as logits, else the input.
__device__ __forceinline__ float gate_act(int prologue, float x) {
  return (prologue & PDN_PRO_SIGMOID_GATES) ? sigmoid_call(x) : x;
}
// The log decay as the kernels use it.
__device__ __forceinline__ float decay_act(int prologue, float decay_scale, float x) {
  if (prologue & (PDN_PRO_DECAY_SOFTPLUS | PDN_PRO_DECAY_LOGSIGMOID))
    return decay_act_call(prologue, decay_scale, x);
  return x;
}
// 1 / max(||x||, 1e-12) from a sum of squares (L2 normalisation of q, k).
__device__ __forceinline__ float inv_norm(float sumsq) {
  return 1.f / fmaxf(sqrtf(sumsq), 1e-12f);
}

__device__ __forceinline__ void record_error(int *err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Index checks of the debug build (compiled with PDN_DEBUG_BOUNDS, shipped as
// libpdn_debug.so): `in_bounds(err, idx < n)` records PDN_ERR_BOUNDS in the
// device error word when the condition fails, and the caller skips the
// access. In the release build it is the constant true and vanishes.
#ifdef PDN_DEBUG_BOUNDS
__device__ __forceinline__ bool in_bounds(int *err, bool ok) {
  if (!ok) record_error(err, PDN_ERR_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(int *, bool) { return true; }
#endif

}  // namespace pdn
