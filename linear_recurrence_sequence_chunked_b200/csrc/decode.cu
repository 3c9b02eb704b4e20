// decode.cu -- one recurrent decode step of the gated delta rule.
//
// Constant-memory decoding ("Gated DeltaNet-2", ja, problem statement): the
// fixed-size fp32 state S (d_v x d_k per batch and head) is read once and
// written once per token. Per (batch, head), with alpha the decay, r/w/u the
// variant's read key, write key and target ("pdn.h" header table):
//   S' = S Diag(alpha),  y = S' r,  z = S' q,  delta = u - y,
//   S  = S' + delta w^T, o = q_scale (z + delta (w . q))
// Every row of S is independent given (r, w, q), so each warp streams whole
// rows: lane l holds key channels 4l..4l+3 as one float4, two warp
// reductions give y_j and z_j, and the updated row is written back in place.
// The kernel is bound by HBM: 8 d_k d_v bytes of state traffic per
// (token, head) against about 7 d_k d_v flops.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace pdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxD = 128;
constexpr int kRows = kMaxD / kWarps;  // state rows per warp (all in flight at once)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block; every thread gets the result. `red` has kWarps floats.
__device__ __forceinline__ float block_sum(float v, float *red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += red[w];
  return s;
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads) decode_kernel(const KParams P) {
  __shared__ float s_r[kMaxD], s_w[kMaxD], s_q[kMaxD], s_al[kMaxD], s_u[kMaxD];
  __shared__ float s_red[kWarps];

  const int tid = threadIdx.x;
  const int bh = blockIdx.x;
  const int b = bh / P.H, h = bh % P.H;
  const int dk = P.dk, dv = P.dv;
  const size_t tokh = tok_index(P, b, 0, h);
  const bool precond = is_precond(P.variant);

  // Issue every state-row load first: they do not depend on the token, so
  // the per-token prologue below runs while they are in flight.
  const int warp = tid >> 5, lane = tid & 31;
  const int c = lane * 4;
  const bool act = c < dk;
  float *S = P.ST + (size_t)bh * dv * dk;
  float4 s[kRows];
#pragma unroll
  for (int m = 0; m < kRows; ++m) {
    const int j = warp + m * kWarps;
    s[m] = (act && j < dv) ? __ldcs(reinterpret_cast<const float4 *>(S + (size_t)j * dk + c))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // per-token vectors
  float kv = 0.f, qv = 0.f, logA = 0.f;
  const bool chan = tid < dk;
  if (chan) {
    kv = ldf<Tin>(P.k, tokh * dk + tid);
    qv = ldf<Tin>(P.q, tokh * dk + tid);
    if (precond) {
      float a = P.AT[(size_t)bh * dk + tid] + kv * kv;
      P.AT[(size_t)bh * dk + tid] = a;
      logA = logf(a + P.eps);
    }
  }
  float mu = 0.f;
  if (precond) mu = block_sum(chan ? logA : 0.f, s_red) / (float)dk;
  float r = 0.f, w = 0.f;
  if (chan) {
    switch (P.variant) {
      case PDN_VAR_PDN: case PDN_VAR_PGDN: case PDN_VAR_PKDA:
        r = kv;
        w = ldf<float>(P.beta, tokh) * precond_coef(logA, mu, P.lnx) * kv;
        break;
      case PDN_VAR_FG2_GDN:
        r = sqrtf(ldf<Tin>(P.beta, tokh * dk + tid)) * kv;
        w = r;
        break;
      case PDN_VAR_GDN2:
        r = ldf<Tin>(P.erase, tokh * dk + tid) * kv;
        w = kv;
        break;
      default:
        r = kv;
        w = ldf<float>(P.beta, tokh) * kv;
    }
    s_r[tid] = r;
    s_w[tid] = w;
    s_q[tid] = qv;
    float al = 1.f;
    if (P.decay == PDN_DECAY_SCALAR) al = expf(ldf<float>(P.log_alpha, tokh));
    else if (P.decay == PDN_DECAY_CHANNEL) al = expf(ldf<Tin>(P.log_alpha, tokh * dk + tid));
    s_al[tid] = al;
  }
  for (int j = tid; j < dv; j += kThreads) {
    float u = ldf<Tin>(P.v, tokh * dv + j);
    if (P.variant == PDN_VAR_FG2_GDN) u *= sqrtf(ldf<Tin>(P.beta, tokh * dv + j));
    else if (P.variant == PDN_VAR_GDN2) u *= ldf<Tin>(P.write, tokh * dv + j);
    s_u[j] = u;
  }
  const float wq = block_sum(chan ? w * qv : 0.f, s_red);  // ends with __syncthreads

  // update the state rows
  float4 rr = make_float4(0.f, 0.f, 0.f, 0.f), ww = rr, qq = rr, aa = rr;
  if (act) {
    rr = make_float4(s_r[c], s_r[c + 1], s_r[c + 2], s_r[c + 3]);
    ww = make_float4(s_w[c], s_w[c + 1], s_w[c + 2], s_w[c + 3]);
    qq = make_float4(s_q[c], s_q[c + 1], s_q[c + 2], s_q[c + 3]);
    aa = make_float4(s_al[c], s_al[c + 1], s_al[c + 2], s_al[c + 3]);
  }
#pragma unroll
  for (int m = 0; m < kRows; ++m) {
    const int j = warp + m * kWarps;
    float4 x = s[m];
    x.x *= aa.x; x.y *= aa.y; x.z *= aa.z; x.w *= aa.w;
    const float y = warp_sum(x.x * rr.x + x.y * rr.y + x.z * rr.z + x.w * rr.w);
    const float z = warp_sum(x.x * qq.x + x.y * qq.y + x.z * qq.z + x.w * qq.w);
    if (j < dv) {
      const float delta = s_u[j] - y;
      x.x = fmaf(delta, ww.x, x.x);
      x.y = fmaf(delta, ww.y, x.y);
      x.z = fmaf(delta, ww.z, x.z);
      x.w = fmaf(delta, ww.w, x.w);
      if (act) __stcs(reinterpret_cast<float4 *>(S + (size_t)j * dk + c), x);
      if (lane == 0) stf<Tin>(P.o, tokh * dv + j, P.q_scale * fmaf(delta, wq, z));
    }
  }
}

__global__ void selftest_wait_kernel(long long limit, int *err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the phase never completes.
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit)) record_error(err, PDN_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_decode(const KParams &P, cudaStream_t stream) {
  const long long grid = (long long)P.B * P.H;
  if (grid <= 0) return cudaSuccess;
  if (P.dtype == PDN_F32)
    decode_kernel<float><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  else
    decode_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(long long spin_limit, int *err, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(spin_limit, err);
  return cudaGetLastError();
}

}  // namespace pdn
