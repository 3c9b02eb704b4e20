// seqpar.cu -- the pieces a sequence-parallel prefill needs besides the
// chunked forward itself ("FG2-GDN", ja §4, long contexts: the sequence is
// cut into segments, one per GPU, joined by one exchange of states).
//
// Every update acts on the state by right-multiplication, so a segment maps
// its start state affinely: S_end = S_start A_seg + B_seg, with
// A_seg = prod_t Diag(alpha_t) (I - r_t w_t^T) (the chunked forward in
// transition mode) and B_seg the segment's final state from S_start = 0.
// The preconditioner's accumulator needs the key energy of every earlier
// segment before any of that can run (its coefficients depend on it).
//   key_energy_kernel   AT = A0 + sum_t k_t . k_t (optionally of the L2-
//                       normalised keys): one CTA per (batch, head)
//   compose_kernel      S_out = S_in A + B_add per (batch, head), fp32
//   accumulate_kernel   out = base + sum of the first n of the gathered parts
//                       (the accumulator at a segment start)
#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Warp w takes tokens w, w + 8, ...; lane l holds key channels 4l .. 4l + 3.
template <typename Tin>
__global__ void __launch_bounds__(kThreads) key_energy_kernel(const KParams P) {
  __shared__ float part[kWarps][128];
  const int bh = blockIdx.x, b = bh / P.H, h = bh % P.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dk = P.dk;
  const bool norm = P.prologue & PDN_PRO_L2NORM_QK;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int t = warp; t < P.T; t += kWarps) {
    const size_t base = tok_index(P, b, t, h) * dk;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 4 * lane + e;
      x[e] = i < dk ? ldf<Tin>(P.k, base + i) : 0.f;
    }
    float scale = 1.f;
    if (norm) scale = inv_norm(warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k = x[e] * scale;
      acc[e] = fmaf(k, k, acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (4 * lane + e < 128) part[warp][4 * lane + e] = acc[e];
  __syncthreads();
  for (int i = threadIdx.x; i < dk; i += kThreads) {
    float s = P.A0 ? P.A0[(size_t)bh * dk + i] : 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += part[w][i];
    P.AT[(size_t)bh * dk + i] = s;
  }
}

// One CTA per (batch, head, 32 rows of S): out[32 x d_k] accumulates
// S_in[32 x 32-slice] * A[32-slice x d_k] over the d_k / 32 slices.
constexpr int kRowsPerCta = 32;
__global__ void __launch_bounds__(kThreads) compose_kernel(int dv, int dk, const float *S_in,
                                                           const float *A, const float *Badd,
                                                           float *S_out) {
  __shared__ float sS[kRowsPerCta][33];
  __shared__ float sA[32][129];
  const int nblk = (dv + kRowsPerCta - 1) / kRowsPerCta;
  const int bh = blockIdx.x / nblk, j0 = (blockIdx.x % nblk) * kRowsPerCta;
  const int tid = threadIdx.x, jj = tid >> 3, c0 = tid & 7;  // row jj, columns c0 + 8 c
  const size_t sbase = (size_t)bh * dv * dk, abase = (size_t)bh * dk * dk;
  float acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = 0.f;
  if (S_in) {
    for (int m0 = 0; m0 < dk; m0 += 32) {
      for (int e = tid; e < kRowsPerCta * 32; e += kThreads) {
        const int r = e >> 5, m = e & 31;
        sS[r][m] = (j0 + r < dv && m0 + m < dk) ? S_in[sbase + (size_t)(j0 + r) * dk + m0 + m] : 0.f;
      }
      for (int e = tid; e < 32 * 128; e += kThreads) {
        const int m = e >> 7, i = e & 127;
        sA[m][i] = (m0 + m < dk && i < dk) ? A[abase + (size_t)(m0 + m) * dk + i] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int m = 0; m < 32; ++m) {
        const float s = sS[jj][m];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = fmaf(s, sA[m][c0 + 8 * c], acc[c]);
      }
      __syncthreads();
    }
  }
  const int j = j0 + jj;
  if (j < dv) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = c0 + 8 * c;
      if (i < dk) {
        const size_t o = sbase + (size_t)j * dk + i;
        S_out[o] = acc[c] + (Badd ? Badd[o] : 0.f);
      }
    }
  }
}

__global__ void accumulate_kernel(int n, long long len, const float *parts, const float *base,
                                  float *out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < len;
       i += (long long)gridDim.x * blockDim.x) {
    float s = base ? base[i] : 0.f;
    for (int g = 0; g < n; ++g) s += parts[(size_t)g * len + i];
    out[i] = s;
  }
}

}  // namespace

cudaError_t launch_accumulate(int n, long long len, const float *parts, const float *base,
                              float *out, cudaStream_t stream) {
  if (len <= 0) return cudaSuccess;
  const long long blocks = (len + kThreads - 1) / kThreads;
  accumulate_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), kThreads, 0, stream>>>(n, len, parts,
                                                                                    base, out);
  return cudaGetLastError();
}

cudaError_t launch_key_energy(const KParams &P, cudaStream_t stream) {
  const long long grid = (long long)P.B * P.H;
  if (grid <= 0) return cudaSuccess;
  if (P.dtype == PDN_F32)
    key_energy_kernel<float><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  else
    key_energy_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_compose(int BH, int dv, int dk, const float *S_in, const float *A,
                           const float *Badd, float *S_out, cudaStream_t stream) {
  const long long grid = (long long)BH * ((dv + kRowsPerCta - 1) / kRowsPerCta);
  if (grid <= 0) return cudaSuccess;
  compose_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(dv, dk, S_in, A, Badd, S_out);
  return cudaGetLastError();
}

}  // namespace pdn
