// chunk_simt.cu -- chunked forward of the gated delta rule on CUDA cores, fp32.
//
// One CTA owns one (batch, head, block of 32 value rows) and walks the chunks
// of its sequence in order. The rows of the d_v x d_k state are independent
// under every variant (each update multiplies S on the right), so splitting
// d_v across CTAs needs no communication; the d_v-independent chunk products
// are recomputed per block.
//
// Per chunk of C tokens (chunkwise WY/UT form: "Gated DeltaNet-2", ja §3,
// decay absorbed into the erase/write matrices and a lower-triangular
// (I + T)^{-1} solve; "Preconditioned DeltaNet", ja §2.3, prefix-sum
// preconditioner inside the chunk form):
//   G_t    = sum_{s<=t} log alpha_s                 (per key channel)
//   M_ts   = sum_i r_ti w_si e^{G_ti - G_si}  (s < t)
//   P_ts   = q_scale sum_i q_ti w_si e^{G_ti - G_si}  (s <= t)
//   Rh     = e^{G} . r,  Qh = q_scale e^{G} . q,  Wb = e^{G_C - G} . w
//   Delta  = (I + M)^{-1} (U - Rh S0^T)             (forward substitution)
//   O      = Qh S0^T + P Delta
//   S_C    = S0 Diag(e^{G_C}) + Delta^T Wb
// Every decay factor is e^{x} with x <= 0, so no decay strength leaves the
// fp32 range (the factorised form e^{G_t} e^{-G_s} would overflow once a
// channel decays by more than e^{-87} inside a chunk). Channel decay costs
// one exponential per (t, s, i) term of M and P; scalar decay one per (t, s).
#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxC = 64;
constexpr int kMaxD = 128;
constexpr int kLD = kMaxD + 1;  // padded row stride (floats) of token x channel tiles
constexpr int kDVB = 32;        // value rows per CTA
constexpr int kLDU = kDVB + 1;
constexpr int kLDC = kMaxC + 1;

struct Smem {
  float R[kMaxC][kLD];   // raw k, then Rh
  float W[kMaxC][kLD];   // log(A + eps), then w, then Wb
  float Q[kMaxC][kLD];   // raw q, then Qh
  float G[kMaxC][kLD];   // cumulative log decay
  float M[kMaxC][kLDC];  // M (strict lower)
  float Pm[kMaxC][kLDC]; // P (lower)
  float U[kMaxC][kLDU];  // u, then RHS, then Delta
  float S[kDVB][kLD];    // state block (rows j0.., all key channels)
  float A[kMaxD];        // preconditioner accumulator carry
  float GC[kMaxD];       // G at the chunk end
  float EGC[kMaxD];      // e^{G_C}
  float mu[kMaxC];       // per-token channel mean of log(A + eps)
  float beta[kMaxC];     // scalar gain per token
  float la[kMaxC];       // scalar log decay per token
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 1) chunk_simt_kernel(const KParams P) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>(smem_raw);

  const int tid = threadIdx.x;
  const int nblk = (P.dv + kDVB - 1) / kDVB;
  const int blk = blockIdx.x % nblk;
  const int bh = blockIdx.x / nblk;
  const int b = bh / P.H, h = bh % P.H;
  const int j0 = blk * kDVB;
  const int nj = min(kDVB, P.dv - j0);
  const int dk = P.dk, dv = P.dv, C = P.chunk;
  const bool precond = is_precond(P.variant);

  // initial state block and accumulator
  const size_t sbase = (size_t)bh * dv * dk;
  for (int idx = tid; idx < kDVB * dk; idx += kThreads) {
    const int jj = idx / dk, i = idx % dk;
    sm.S[jj][i] = jj >= nj       ? 0.f
                  : P.transition ? (j0 + jj == i ? 1.f : 0.f)  // the identity (d_v = d_k)
                  : P.S0         ? P.S0[sbase + (size_t)(j0 + jj) * dk + i] : 0.f;
  }
  for (int i = tid; i < dk; i += kThreads)
    sm.A[i] = (precond && P.A0) ? P.A0[(size_t)bh * dk + i] : 0.f;
  __syncthreads();

  const int nchunks = (P.T + C - 1) / C;
  for (int c = 0; c < nchunks; ++c) {
    const int c0 = c * C;
    const int Cn = min(C, P.T - c0);

    // (a) raw loads; tokens past the end are zero (they contribute nothing)
    for (int idx = tid; idx < C * dk; idx += kThreads) {
      const int t = idx / dk, i = idx % dk;
      const bool ok = t < Cn;
      const size_t e = tok_index(P, b, c0 + t, h) * dk + i;
      sm.R[t][i] = ok ? ldf<Tin>(P.k, e) : 0.f;
      sm.Q[t][i] = ok ? ldf<Tin>(P.q, e) : 0.f;
      if (P.decay == PDN_DECAY_CHANNEL)
        sm.G[t][i] = ok ? decay_act(P.prologue, P.decay_scale, ldf<Tin>(P.log_alpha, e)) : 0.f;
    }
    for (int idx = tid; idx < C * kDVB; idx += kThreads) {
      const int t = idx / kDVB, jj = idx % kDVB;
      const bool ok = t < Cn && jj < nj && !P.transition;  // transition mode: no targets
      sm.U[t][jj] = ok ? ldf<Tin>(P.v, tok_index(P, b, c0 + t, h) * dv + j0 + jj) : 0.f;
    }
    for (int t = tid; t < C; t += kThreads) {
      const bool ok = t < Cn;
      const size_t e = tok_index(P, b, c0 + t, h);
      sm.beta[t] = (ok && has_scalar_beta(P.variant)) ? gate_act(P.prologue, ldf<float>(P.beta, e)) : 0.f;
      sm.la[t] = (ok && P.decay == PDN_DECAY_SCALAR)
                     ? decay_act(P.prologue, P.decay_scale, ldf<float>(P.log_alpha, e)) : 0.f;
    }
    __syncthreads();
    if (P.prologue & PDN_PRO_L2NORM_QK) {
      // L2 normalisation of each token's k and q (8 lanes per token and tensor)
      const int warp = tid >> 5, lane = tid & 31;
      for (int t = warp * 2 + (lane >> 4); t < C; t += (kThreads / 32) * 2) {
        const int part = lane & 15;  // lanes part and part ^ 8 .. cover the token
        float (*X)[kLD] = part < 8 ? sm.R : sm.Q;
        float ss = 0.f;
        for (int i = part & 7; i < dk; i += 8) ss = fmaf(X[t][i], X[t][i], ss);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        const float inv = inv_norm(ss);
        for (int i = part & 7; i < dk; i += 8) X[t][i] *= inv;
      }
      __syncthreads();
    }

    // (b) per-channel scans: cumulative log decay and the key-energy prefix sum
    for (int i = tid; i < dk; i += kThreads) {
      float g = 0.f, a = sm.A[i];
      for (int t = 0; t < C; ++t) {
        // a log decay below -100 is raised to it: e^{-100} is below the
        // smallest normal fp32 number, so every factor it enters stays zero
        const float la = fmaxf(P.decay == PDN_DECAY_CHANNEL ? sm.G[t][i]
                               : P.decay == PDN_DECAY_SCALAR ? sm.la[t] : 0.f, -100.f);
        g += la;
        sm.G[t][i] = g;
        if (precond) {
          const float kk = sm.R[t][i];
          a += kk * kk;
          sm.W[t][i] = logf(a + P.eps);
        }
      }
      sm.A[i] = a;
      sm.GC[i] = g;
      sm.EGC[i] = expf(g);
    }
    __syncthreads();

    // (c) per-token channel mean of log(A + eps)
    if (precond) {
      for (int t = tid; t < C; t += kThreads) {
        float s = 0.f;
        for (int i = 0; i < dk; ++i) s += sm.W[t][i];
        sm.mu[t] = s / (float)dk;
      }
      __syncthreads();
    }

    // (d) read key r, write key w, scaled query (undecayed)
    for (int idx = tid; idx < C * dk; idx += kThreads) {
      const int t = idx / dk, i = idx % dk;
      const bool ok = t < Cn;
      const float kv = sm.R[t][i];
      float r = kv, w, qf = P.q_scale * sm.Q[t][i];
      switch (P.variant) {
        case PDN_VAR_PDN: case PDN_VAR_PGDN: case PDN_VAR_PKDA:
          w = sm.beta[t] * precond_coef(sm.W[t][i], sm.mu[t], P.lnx) * kv;
          break;
        case PDN_VAR_PLA:  // no erase; the preconditioner acts on the query
          r = 0.f;
          w = sm.beta[t] * kv;
          qf *= precond_coef(sm.W[t][i], sm.mu[t], P.lnx);
          break;
        case PDN_VAR_FG2_GDN: case PDN_VAR_FG2_GDN_PLUS: {
          const float sb =
              ok ? sqrtf(gate_act(P.prologue, ldf<Tin>(P.beta, tok_index(P, b, c0 + t, h) * dk + i))) : 0.f;
          r = sb * kv;
          w = r;
        } break;
        case PDN_VAR_GDN2: {
          const float e = ok ? gate_act(P.prologue, ldf<Tin>(P.erase, tok_index(P, b, c0 + t, h) * dk + i)) : 0.f;
          r = e * kv;
          w = kv;
        } break;
        default:
          w = sm.beta[t] * kv;
      }
      sm.R[t][i] = r;
      sm.W[t][i] = w;
      sm.Q[t][i] = qf;
    }
    if (P.variant == PDN_VAR_FG2_GDN || P.variant == PDN_VAR_GDN2 ||
        P.variant == PDN_VAR_FG2_GDN_PLUS) {
      for (int idx = tid; idx < C * kDVB; idx += kThreads) {
        const int t = idx / kDVB, jj = idx % kDVB;
        if (t < Cn && jj < nj) {
          const size_t e = tok_index(P, b, c0 + t, h) * dv + j0 + jj;
          const float f = P.variant == PDN_VAR_FG2_GDN ? sqrtf(gate_act(P.prologue, ldf<Tin>(P.beta, e)))
                          : P.variant == PDN_VAR_GDN2 ? gate_act(P.prologue, ldf<Tin>(P.write, e))
                                                      : sqrtf(gate_act(P.prologue, ldf<Tin>(P.write, e)));
          sm.U[t][jj] *= f;
        }
      }
    }
    __syncthreads();

    // (e) M and P with their in-chunk decay e^{G_t - G_s} <= 1
    {
      const int t = tid >> 2, p = tid & 3;  // 64 rows x 4 lanes, 16 columns each
      if (t < C) {
        float am[16], ap[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) { am[m] = 0.f; ap[m] = 0.f; }
        if (P.decay == PDN_DECAY_CHANNEL) {
          for (int i = 0; i < dk; ++i) {
            const float rt = sm.R[t][i], qt = sm.Q[t][i], gt = sm.G[t][i];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int s = p + 4 * m;
              if (s <= t) {
                const float x = sm.W[s][i] * expf(gt - sm.G[s][i]);
                am[m] = fmaf(rt, x, am[m]);
                ap[m] = fmaf(qt, x, ap[m]);
              }
            }
          }
        } else {
          for (int i = 0; i < dk; ++i) {
            const float rt = sm.R[t][i], qt = sm.Q[t][i];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int s = p + 4 * m;
              const float ws = s < C ? sm.W[s][i] : 0.f;
              am[m] = fmaf(rt, ws, am[m]);
              ap[m] = fmaf(qt, ws, ap[m]);
            }
          }
          if (P.decay == PDN_DECAY_SCALAR) {
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int s = p + 4 * m;
              if (s <= t) {
                const float f = expf(sm.G[t][0] - sm.G[s][0]);
                am[m] *= f;
                ap[m] *= f;
              }
            }
          }
        }
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int s = p + 4 * m;
          if (s < C) {
            sm.M[t][s] = s < t ? am[m] : 0.f;
            sm.Pm[t][s] = s <= t ? ap[m] : 0.f;
          }
        }
      }
    }
    __syncthreads();
    // decayed operands of the state terms: Rh = e^{G} r, Qh = e^{G} q,
    // Wb = e^{G_C - G} w (all factors <= 1)
    if (P.decay != PDN_DECAY_NONE) {
      for (int idx = tid; idx < C * dk; idx += kThreads) {
        const int t = idx / dk, i = idx % dk;
        const float g = sm.G[t][i];
        const float eg = expf(g);
        sm.R[t][i] *= eg;
        sm.Q[t][i] *= eg;
        sm.W[t][i] *= expf(sm.GC[i] - g);
      }
      __syncthreads();
    }
    // RHS = U - Rh S^T
    for (int idx = tid; idx < C * kDVB; idx += kThreads) {
      const int t = idx / kDVB, jj = idx % kDVB;
      float acc = 0.f;
      for (int i = 0; i < dk; ++i) acc = fmaf(sm.R[t][i], sm.S[jj][i], acc);
      sm.U[t][jj] -= acc;
    }
    __syncthreads();

    // (f) Delta = (I + M)^{-1} RHS by forward substitution; 8 lanes per column
    {
      const int warp = tid >> 5, lane = tid & 31;
      const int jj = warp * 4 + (lane >> 3), part = lane & 7;
      for (int t = 1; t < C; ++t) {
        float acc = 0.f;
        for (int s = part; s < t; s += 8) acc = fmaf(sm.M[t][s], sm.U[s][jj], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (part == 0) sm.U[t][jj] -= acc;
        __syncwarp();
      }
    }
    __syncthreads();

    // (g) O = Qh S^T + P Delta for the valid tokens
    for (int idx = tid; idx < C * kDVB; idx += kThreads) {
      const int t = idx / kDVB, jj = idx % kDVB;
      if (t < Cn && jj < nj && P.o) {
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc = fmaf(sm.Q[t][i], sm.S[jj][i], acc);
        for (int s = 0; s <= t; ++s) acc = fmaf(sm.Pm[t][s], sm.U[s][jj], acc);
        stf<Tin>(P.o, tok_index(P, b, c0 + t, h) * dv + j0 + jj, acc);
      }
    }
    __syncthreads();

    // (h) S <- S Diag(e^{G_C}) + Delta^T Wb
    for (int idx = tid; idx < kDVB * dk; idx += kThreads) {
      const int jj = idx / dk, i = idx % dk;
      float acc = sm.S[jj][i] * sm.EGC[i];
      for (int t = 0; t < C; ++t) acc = fmaf(sm.U[t][jj], sm.W[t][i], acc);
      sm.S[jj][i] = acc;
    }
    __syncthreads();
  }

  if (P.ST) {
    for (int idx = tid; idx < nj * dk; idx += kThreads) {
      const int jj = idx / dk, i = idx % dk;
      P.ST[sbase + (size_t)(j0 + jj) * dk + i] = sm.S[jj][i];
    }
  }
  if (P.AT && precond && blk == 0) {
    for (int i = tid; i < dk; i += kThreads) P.AT[(size_t)bh * dk + i] = sm.A[i];
  }
}

}  // namespace

int simt_supported(const KParams &P) {
  return P.dk <= kMaxD && P.dv <= kMaxD && P.chunk <= kMaxC;
}

cudaError_t launch_chunk_simt(const KParams &P, cudaStream_t stream) {
  const int nblk = (P.dv + kDVB - 1) / kDVB;
  const long long grid = (long long)P.B * P.H * nblk;
  if (grid <= 0) return cudaSuccess;
  const size_t smem = sizeof(Smem);
  cudaError_t e;
  if (P.dtype == PDN_F32) {
    e = cudaFuncSetAttribute(chunk_simt_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<float><<<(unsigned)grid, kThreads, smem, stream>>>(P);
  } else {
    e = cudaFuncSetAttribute(chunk_simt_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, smem, stream>>>(P);
  }
  return cudaGetLastError();
}

}  // namespace pdn
