// backward.cu -- gradient of the chunked forward ("Gated DeltaNet-2", ja §3:
// the gate-aware backward; the erase and write gates enter the gradient
// through the read key, the write key and the target).
//
// Generic token step (every variant; r read key, w write key, u target,
// alpha the decay, q' the read-out query, c = q_scale):
//   P_t = S_{t-1} Diag(alpha_t),  delta_t = u_t - P_t r_t,
//   S_t = P_t + delta_t w_t^T,    o_t = c S_t q'_t.
// Reverse mode, with dS~_t the total cotangent of S_t:
//   dS~_t = dS_t + c dO_t q'_t^T,  dd_t = dS~_t w_t        (= d delta = du)
//   dw_t = dS~_t^T delta_t,        dr_t = -P_t^T dd_t,      dq'_t = c S_t^T dO_t
//   dS_{t-1} = (dS~_t - dd_t r_t^T) Diag(alpha_t).
// Every row of S and of dS evolves on its own; only the read-outs mix rows.
// The work is split so that no per-token state is ever stored:
//   F1  forward, 8 (or 4) state rows per warp: delta_t (a row reduction
//       per token)
//   R1  reverse, likewise: dd_t, dS0 (F1 and R1 share no data and run as
//       one launch)
//   F2  forward, thread per key column, delta given: dq'_t and dr_t
//   R2  reverse, thread per key column, dd given:    dw_t
// F2 and R2 have no reduction and no feedback (a gated linear attention pass
// each), so they run every 64-token chunk in parallel from the states F1 and
// R1 leave at the chunk boundaries; their column sums over a CTA's rows are
// written per row group and added in the epilogue.
//
// The decay gradient needs no state either. With psi_t,i = sum_j P_t[j,i]
// dP_t[j,i] (the cotangent of log alpha_t,i), expanding S_t = P_t + delta_t
// w_t^T and dS~_t gives psi_t = psi_{t+1} + q'_t.dq'_t - w_t.dw_t + r_t.dr_t
// (elementwise), started from psi_T,i = sum_j S_T[j,i] dS_T[j,i]: a suffix
// sum over tokens. A scalar decay takes sum_i psi_t,i.
//
// The preconditioner's coefficients B_t depend on A_t = A_{t-1} + k_t.k_t
// ("Preconditioned DeltaNet", ja §2.2); each token's dB_t gives a dA_t, and
// A_t feeds every later token, so k_t receives 2 k_t (sum_{s>=t} dA_s).
//
// Under a fused prologue the inputs are raw projections: the activations
// are applied where the inputs are read and the gradients are taken back
// through them (to the logits of the gates, through the L2 normalisation of
// q and k, through the decay map).
//
// All arithmetic is fp32; inputs of either dtype are widened on load and
// every gradient is written in fp32.
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace pdn {

// Workspace plan (floats), shared by the size query and the launcher.
struct BwdPlan {
  int GS;          // floats per (token, head) of the generic vectors: q'|r|w|a|u
  int R, G;        // rows per CTA of F2/R2, row groups (d_v / R)
  int nb;          // scan blocks per sequence
  int nck;         // state checkpoints per sequence (one per kCk tokens)
  size_t gen, acc, delta, dd, cdo, st, part, cpsi, sigma, dacc, bsum, phi, ckS, ckD, total;
};

namespace {

constexpr int kScanBlk = 64;     // tokens per scan block
constexpr int kCk = 64;          // tokens per state checkpoint (F2 / R2 run chunk-parallel)
constexpr int kLCC = 8;          // tokens staged per chunk in F2 / R2

size_t up64(size_t n) { return (n + 63) & ~(size_t)63; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace

static BwdPlan bwd_plan(const KParams &P) {
  BwdPlan L;
  memset(&L, 0, sizeof(L));
  const size_t BH = (size_t)P.B * P.H, T = (size_t)P.T;
  const int dk = P.dk, dv = P.dv;
  L.GS = 4 * dk + dv;
  // F2 / R2 are chunk-parallel: wide row groups (fewer partial sums)
  L.R = dv % 64 == 0 ? 64 : dv % 32 == 0 ? 32 : 16;
  L.G = dv / L.R;
  L.nb = (int)((T + kScanBlk - 1) / kScanBlk);
  size_t off = 0;
  auto take = [&](size_t n) { const size_t o = off; off += up64(n); return o; };
  L.gen = take(BH * T * L.GS);
  L.acc = take(is_precond(P.variant) ? BH * T * dk : 0);
  L.delta = take(BH * T * dv);
  L.dd = take(BH * T * dv);
  L.cdo = take(BH * T * dv);
  L.st = take(BH * dv * dk);
  L.part = take((size_t)L.G * BH * T * 3 * dk);
  L.cpsi = take(P.decay == PDN_DECAY_CHANNEL ? BH * T * dk : 0);
  L.sigma = take(P.decay == PDN_DECAY_SCALAR ? BH * T : 0);
  L.dacc = take(is_precond(P.variant) ? BH * T * dk : 0);
  L.bsum = take(BH * (size_t)L.nb * dk);
  L.phi = take(BH * dk + BH);
  L.nck = (int)((T + kCk - 1) / kCk);
  L.ckS = take(BH * (size_t)L.nck * dv * dk);
  L.ckD = take(BH * (size_t)L.nck * dv * dk);
  L.total = off;
  return L;
}

namespace {

// Everything the backward kernels read and write, by value.
struct BParams {
  KParams P;
  const void *dO;     // dtype [B,T,H,dv] or NULL
  const float *dST;   // [B,H,dv,dk] or NULL
  float *dq, *dk, *dv, *dla, *dbeta, *derase, *dwrite, *dS0, *dA0;
  float *gen, *acc, *delta, *dd, *st, *part, *cpsi, *sigma, *dacc, *bsum, *phi;
  // c dO in fp32, [BH][T][d_v] like delta and dd (zeros when dO is not given)
  float *cdo;
  // S before the first token of each kCk-token chunk (F1) and the cotangent
  // entering each chunk's last token (R1): [BH][nck][d_v][d_k]; the states
  // saved by the forward in training mode are transposed, [BH][nck][d_k][d_v]
  // (ck_t)
  float *ckS, *ckD;
  bool ck_t;
  int GS, R, G, nb, nck;
  // element counts of the workspace arrays (index checks of the debug build)
  size_t n_rows, n_part, n_ck;
};

// Generic vectors of one token, in the workspace order q'|r|w|a|u.
__device__ __forceinline__ float *gen_at(const BParams &Q, int bh, int t) {
  return Q.gen + ((size_t)bh * Q.P.T + t) * Q.GS;
}

// ---------------------------------------------------------------------------
// Suffix / prefix sums over tokens, per (batch, head, channel), in three
// passes: block totals, the carry into each block, the sums inside blocks.
// A tensor is addressed either as workspace [BH][T][nch] (tok = false) or as
// a [B,T,H,nch] tensor (tok = true).
struct ScanArr {
  float *p;
  bool tok;
};
__device__ __forceinline__ size_t scan_off(const KParams &P, const ScanArr &a, int nch, int bh,
                                           int t, int c) {
  if (a.tok) return tok_index(P, bh / P.H, t, bh % P.H) * nch + c;
  return ((size_t)bh * P.T + t) * nch + c;
}

__global__ void scan_part_kernel(const KParams P, ScanArr X, int nch, int nb, float *bsum) {
  const long long n = (long long)P.B * P.H * nb * nch;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % nch);
    const long long r = e / nch;
    const int blk = (int)(r % nb), bh = (int)(r / nb);
    const int t0 = blk * kScanBlk, t1 = min(P.T, t0 + kScanBlk);
    float s = 0.f;
#pragma unroll 8
    for (int t = t0; t < t1; ++t) s += X.p[scan_off(P, X, nch, bh, t, c)];
    bsum[e] = s;
  }
}

// Replaces each block total by the sum carried into that block (from the
// sequence start when !rev, from its end when rev), seeded with init
// ([BH][nch], may be NULL). total (may be NULL) gets the full sum + init.
// Eight block totals are loaded at a time, so the walk over the blocks waits
// on memory once per eight.
__global__ void scan_carry_kernel(const KParams P, int nch, int nb, bool rev, float *bsum,
                                  const float *init, float *total) {
  constexpr int kB = 8;
  const long long n = (long long)P.B * P.H * nch;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % nch), bh = (int)(e / nch);
    float carry = init ? init[e] : 0.f;
    float *base = bsum + (size_t)bh * nb * nch + c;
    for (int k0 = 0; k0 < nb; k0 += kB) {
      float v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int blk = rev ? nb - 1 - (k0 + u) : k0 + u;
        v[u] = k0 + u < nb ? base[(size_t)blk * nch] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int blk = rev ? nb - 1 - (k0 + u) : k0 + u;
        if (k0 + u < nb) base[(size_t)blk * nch] = carry;
        carry += v[u];
      }
    }
    if (total) total[e] = carry;
  }
}

// Y_t = carry + inclusive sum of X inside the block (Y may alias X).
__global__ void scan_fill_kernel(const KParams P, ScanArr X, ScanArr Y, int nch, int nb, bool rev,
                                 const float *bsum) {
  const long long n = (long long)P.B * P.H * nb * nch;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % nch);
    const long long r = e / nch;
    const int blk = (int)(r % nb), bh = (int)(r / nb);
    const int t0 = blk * kScanBlk, t1 = min(P.T, t0 + kScanBlk);
    float y = bsum[e];
    if (!rev) {
      for (int t = t0; t < t1; ++t) {
        y += X.p[scan_off(P, X, nch, bh, t, c)];
        Y.p[scan_off(P, Y, nch, bh, t, c)] = y;
      }
    } else {
      for (int t = t1 - 1; t >= t0; --t) {
        y += X.p[scan_off(P, X, nch, bh, t, c)];
        Y.p[scan_off(P, Y, nch, bh, t, c)] = y;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Four consecutive floats from p (16-byte aligned) where `ok`, else zeros.
__device__ __forceinline__ void ld4(const float *p, bool ok, float (&v)[4]) {
  const float4 x = ok ? *reinterpret_cast<const float4 *>(p) : make_float4(0.f, 0.f, 0.f, 0.f);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}

// Four consecutive input elements from element i (8- or 16-byte aligned),
// widened to fp32.
template <typename Tin>
__device__ __forceinline__ void ld4_in(const void *p, size_t i, float (&v)[4]) {
  if constexpr (sizeof(Tin) == 4) {
    const float4 x = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const uint2 x = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + i);
    v[0] = __uint_as_float(x.x << 16); v[1] = __uint_as_float(x.x & 0xffff0000u);
    v[2] = __uint_as_float(x.y << 16); v[3] = __uint_as_float(x.y & 0xffff0000u);
  }
}

// The same where `ok`, else four copies of `fill`.
template <typename Tin>
__device__ __forceinline__ void ld4_opt(const void *p, size_t i, bool ok, float (&v)[4],
                                        float fill = 0.f) {
  if (ok) {
    ld4_in<Tin>(p, i, v);
  } else {
    v[0] = v[1] = v[2] = v[3] = fill;
  }
}

// q and k as the recurrence uses them: under PDN_PRO_L2NORM_QK they arrive
// raw and are divided by their norm over the head dimension (lane l holds
// channels 4l..4l+3; every lane of the warp takes part). Returns the
// inverse norm (1 without the prologue bit).
__device__ __forceinline__ float l2norm_fwd(int prologue, float (&x)[4]) {
  if (!(prologue & PDN_PRO_L2NORM_QK)) return 1.f;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) s = fmaf(x[e], x[e], s);
  const float inv = inv_norm(warp_sum(s));
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] *= inv;
  return inv;
}

// The gradient through y = x / max(||x||, 1e-12): dy (this lane's 4
// channels) becomes dx = (dy - y (y . dy)) / ||x||, or dy / 1e-12 where the
// floor applies. inv = 1 / max(||x||, 1e-12), y the normalised vector.
__device__ __forceinline__ void l2norm_bwd(const float (&y)[4], float (&dy)[4], float inv) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) s = fmaf(y[e], dy[e], s);
  s = warp_sum(s);
  const bool floored = !(inv < 1e12f);
#pragma unroll
  for (int e = 0; e < 4; ++e) dy[e] = (floored ? dy[e] : dy[e] - y[e] * s) * inv;
}

// d gate / d logit of a sigmoid gate g = sigmoid(x), from g.
__device__ __forceinline__ float sigmoid_grad(float g) { return g * (1.f - g); }
// Four gate or gain values as the recurrence uses them (sigmoid of logits
// under PDN_PRO_SIGMOID_GATES).
__device__ __forceinline__ void gate4(int prologue, float (&x)[4]) {
  if (prologue & PDN_PRO_SIGMOID_GATES) {
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = sigmoid_call(x[e]);
  }
}

// Prep (preconditioned variants): the block totals of k_{t,i}^2 over each
// kScanBlk-token block, into bsum[bh][block][i], for the carry pass; the
// generic-vector pass then accumulates A_t = A_0 + sum_{s<=t} k_s^2 inside
// each block in the same order as the sums here. One warp per (head,
// block), lane l on key channels 4l .. 4l + 3 (k normalised first under the
// prologue, as in the generic-vector pass).
template <typename Tin>
__global__ void ksq_part_kernel(const BParams Q) {
  const KParams &P = Q.P;
  const int lane = threadIdx.x & 31, dk = P.dk, c = 4 * lane;
  const bool ak = c < dk;
  const long long nblk = (long long)P.B * P.H * Q.nb;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < nblk; wid += nw) {
    const int bh = (int)(wid / Q.nb), blk = (int)(wid % Q.nb);
    const int t_begin = blk * kScanBlk, t_end = min(P.T, t_begin + kScanBlk);
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t = t_begin; t < t_end; ++t) {
      float k[4];
      ld4_opt<Tin>(P.k, tok_index(P, bh / P.H, t, bh % P.H) * dk + c, ak, k);
      l2norm_fwd(P.prologue, k);
#pragma unroll
      for (int e = 0; e < 4; ++e) s[e] += k[e] * k[e];
    }
    if (ak)
      *reinterpret_cast<float4 *>(Q.bsum + ((size_t)bh * Q.nb + blk) * dk + c) =
          make_float4(s[0], s[1], s[2], s[3]);
  }
}

// The variant's (q', r, w, alpha, u) of every token, one warp per (head,
// kScanBlk-token block) walking its tokens in order; lane l holds channels
// 4l..4l+3 of the key side and of the value side. For the preconditioned
// variants the warp carries A_t from the block's carry-in (bsum) and writes
// it to acc for the chain rules.
// Variant table: DN/GDN/KDA r = k, w = beta k, u = v; PDN/PGDN/PKDA w = beta
// (B_t . k); FG2-GDN r = w = sqrt(beta) . k, u = sqrt(beta) . v; GDN-2 r = e . k,
// w = k, u = g . v; PLA r = 0, w = beta k, q' = B_t . q; FG2-GDN+ r = w =
// sqrt(beta_k) . k, u = sqrt(beta_v) . v.
template <typename Tin>
__global__ void prep_gen_kernel(const BParams Q) {
  const KParams &P = Q.P;
  const int lane = threadIdx.x & 31, dk = P.dk, dv = P.dv;
  const long long nblk = (long long)P.B * P.H * Q.nb;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const bool pre = is_precond(P.variant);
  const int c = 4 * lane;
  const bool ak = c < dk, av = c < dv;
  for (long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < nblk; wid += nw) {
    const int bh = (int)(wid / Q.nb), blk = (int)(wid % Q.nb);
    const int t_begin = blk * kScanBlk, t_end = min(P.T, t_begin + kScanBlk);
    float Arun[4];  // A before the current token (the block's carry-in first)
    ld4(pre ? Q.bsum + ((size_t)bh * Q.nb + blk) * dk + c : nullptr, pre && ak, Arun);
    for (int t = t_begin; t < t_end; ++t) {
      const size_t tk = tok_index(P, bh / P.H, t, bh % P.H);
      float k[4], q[4], v[4], Bc[4], a[4];
      ld4_opt<Tin>(P.k, tk * dk + c, ak, k);
      ld4_opt<Tin>(P.q, tk * dk + c, ak, q);
      ld4_opt<Tin>(P.v, tk * dv + c, av, v);
      l2norm_fwd(P.prologue, k);
      l2norm_fwd(P.prologue, q);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Bc[e] = 1.f;
        a[e] = 1.f;
      }
      if (pre) {
        float L[4], s = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) Arun[e] += k[e] * k[e];
        if (ak)
          *reinterpret_cast<float4 *>(Q.acc + ((size_t)bh * P.T + t) * dk + c) =
              make_float4(Arun[0], Arun[1], Arun[2], Arun[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          L[e] = ak ? logf(Arun[e] + P.eps) : 0.f;
          s += L[e];
        }
        const float mu = warp_sum(s) / (float)dk;
#pragma unroll
        for (int e = 0; e < 4; ++e) Bc[e] = precond_coef(L[e], mu, P.lnx);
      }
      if (P.decay == PDN_DECAY_SCALAR) {
        const float ea = expf(decay_act(P.prologue, P.decay_scale,
                                        reinterpret_cast<const float *>(P.log_alpha)[tk]));
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = ea;
      } else if (P.decay == PDN_DECAY_CHANNEL) {
        float la[4];
        ld4_opt<Tin>(P.log_alpha, tk * dk + c, ak, la);
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = ak ? expf(decay_act(P.prologue, P.decay_scale, la[e])) : 1.f;
      }
      float r[4], w[4], u[4], qq[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        r[e] = k[e];
        w[e] = k[e];
        u[e] = v[e];
        qq[e] = q[e];
      }
      switch (P.variant) {
        case PDN_VAR_DN: case PDN_VAR_GDN: case PDN_VAR_KDA: {
          const float be = gate_act(P.prologue, reinterpret_cast<const float *>(P.beta)[tk]);
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = be * k[e];
        } break;
        case PDN_VAR_PDN: case PDN_VAR_PGDN: case PDN_VAR_PKDA: {
          const float be = gate_act(P.prologue, reinterpret_cast<const float *>(P.beta)[tk]);
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = be * Bc[e] * k[e];
        } break;
        case PDN_VAR_PLA: {
          const float be = gate_act(P.prologue, reinterpret_cast<const float *>(P.beta)[tk]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            r[e] = 0.f;
            w[e] = be * k[e];
            qq[e] = Bc[e] * q[e];
          }
        } break;
        case PDN_VAR_FG2_GDN: case PDN_VAR_FG2_GDN_PLUS: {
          const bool plus = P.variant == PDN_VAR_FG2_GDN_PLUS;
          float bk[4], bv[4];
          ld4_opt<Tin>(P.beta, tk * dk + c, ak, bk);
          gate4(P.prologue, bk);
          if (plus) {
            ld4_opt<Tin>(P.write, tk * dv + c, av, bv);
            gate4(P.prologue, bv);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float sb = ak ? sqrtf(bk[e]) : 0.f;
            r[e] = sb * k[e];
            w[e] = sb * k[e];
            // (FG2-GDN: one gain for both sides, d_k = d_v)
            const float g = av ? (plus ? bv[e] : bk[e]) : 0.f;
            u[e] = sqrtf(g) * v[e];
          }
        } break;
        case PDN_VAR_GDN2: {
          float er[4], gw[4];
          ld4_opt<Tin>(P.erase, tk * dk + c, ak, er);
          ld4_opt<Tin>(P.write, tk * dv + c, av, gw);
          gate4(P.prologue, er);
          gate4(P.prologue, gw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            r[e] = er[e] * k[e];
            u[e] = gw[e] * v[e];
          }
        } break;
        default: break;
      }
      float *g = gen_at(Q, bh, t);
      if (ak) {
        *reinterpret_cast<float4 *>(g + c) = make_float4(qq[0], qq[1], qq[2], qq[3]);
        *reinterpret_cast<float4 *>(g + dk + c) = make_float4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<float4 *>(g + 2 * dk + c) = make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<float4 *>(g + 3 * dk + c) = make_float4(a[0], a[1], a[2], a[3]);
      }
      if (av) *reinterpret_cast<float4 *>(g + 4 * dk + c) = make_float4(u[0], u[1], u[2], u[3]);
      if (av) {  // c dO of the token (zeros without dO), once, for the three sweeps that read it
        float o[4];
        ld4_opt<Tin>(Q.dO, tk * dv + c, Q.dO != nullptr, o);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] *= P.q_scale;
        *reinterpret_cast<float4 *>(Q.cdo + ((size_t)bh * P.T + t) * dv + c) = make_float4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Row sweeps F1 / R1, blocked over rows in registers. A warp owns RW = 8
// consecutive state rows of one (batch, head) -- a CTA, 4 warps, owns 32
// rows -- and lane l holds key channels C l .. C l + C - 1 (C = 1, 2 or 4 by
// d_k) of all of them, so every per-token vector a lane reads from shared
// memory serves RW rows and the 32 lanes of one load read 32 distinct
// pieces. (With lanes of different rows reading the same vector, a 16-byte
// load is served a quarter-warp at a time and every row-token costs the whole
// vector in shared-memory wavefronts: at the headline sizes that pipe, not the
// arithmetic, bounds the sweeps.) The RW row reductions over key channels
// share one transposed butterfly (rows_sum) and the finished row values
// return to every lane by its reverse (rows_spread); a lane-dependent order
// of the rows in registers spares both every select. The arithmetic stays
// scalar fp32: packed pair instructions would need a register pair for every
// broadcast operand, and the moves that builds cost as much as the pairs
// save (measured). The per-token vectors are staged
// through shared memory kLCR tokens at a time with cp.async (double
// buffered), each padded to 32 C floats with zeros, and every full chunk of
// kLCR tokens runs unrolled (constant shared-memory offsets).
//
// F1 and R1 share no data (F1 reads S0 and the generic vectors, R1 dS_T, c dO
// and the generic vectors), so they run as one launch, R1's CTAs first (the
// longer sweep), both resident at once.
constexpr int kLCR = 8;  // tokens staged per chunk in F1 / R1

// C consecutive floats (16-, 8- or 4-byte aligned) to registers and back;
// a NULL source reads zeros.
template <int C>
__device__ __forceinline__ void ld_c(const float *p, float (&v)[C]) {
  if constexpr (C == 4) {
    const float4 x = p ? *reinterpret_cast<const float4 *>(p) : make_float4(0.f, 0.f, 0.f, 0.f);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else if constexpr (C == 2) {
    const float2 x = p ? *reinterpret_cast<const float2 *>(p) : make_float2(0.f, 0.f);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = p ? *p : 0.f;
  }
}
template <int C>
__device__ __forceinline__ void st_c(float *p, const float (&v)[C]) {
  if constexpr (C == 4)
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  else if constexpr (C == 2)
    *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
  else
    *p = v[0];
}

// Packed fp32 pairs (one instruction for two lanes' worth of FMA or MUL; each
// element rounds exactly as fmaf / a single multiply).
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// Row sums of a warp's RW rows. Lane l keeps its rows in a lane-dependent
// order: register slot s holds row s ^ jl, jl = l / (32 / RW). p[s] is this
// lane's partial sum of the row in slot s. Each of the first log2(RW)
// exchanges (across lane bits 4, 3, ...) adds the upper half of the slots a
// lane still carries to the lower half of its partner's -- with the xor
// order the two hold the same rows there, so no lane selects -- and the
// remaining xor levels finish the sum. Returns the full sum of row jl.
template <int RW>
__device__ __forceinline__ float rows_sum(const float (&p)[RW]) {
  float c[RW];
#pragma unroll
  for (int s = 0; s < RW; ++s) c[s] = p[s];
#pragma unroll
  for (int n = RW, m = 16; n > 1; n >>= 1, m >>= 1)
#pragma unroll
    for (int k = 0; k < n / 2; ++k) c[k] += __shfl_xor_sync(0xffffffffu, c[k + n / 2], m);
  float v = c[0];
#pragma unroll
  for (int m = 16 / RW; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// The reverse: v is a value of row jl (the same on the lanes of a row);
// o[s] receives the value of row s ^ jl, slot order as above.
template <int RW>
__device__ __forceinline__ void rows_spread(float v, float (&o)[RW]) {
  o[0] = v;
#pragma unroll
  for (int n = 1, m = 32 / RW; n < RW; n <<= 1, m <<= 1)
#pragma unroll
    for (int k = 0; k < n; ++k) o[k + n] = __shfl_xor_sync(0xffffffffu, o[k], m);
}

// State rows held in slot order: X[s][e] is row jw + (s ^ jl) at key channel
// c0 + e (base: row 0, channel c0 of the (batch, head) block).
template <int C, int RW>
__device__ __forceinline__ void ld_state(const float *base, int dv, int dk, int jw, int jl,
                                         bool cok, float (&X)[RW][C]) {
#pragma unroll
  for (int s = 0; s < RW; ++s) {
    const int j = jw + (s ^ jl);
    ld_c<C>(base && cok && j < dv ? base + (size_t)j * dk : nullptr, X[s]);
  }
}
template <int C, int RW>
__device__ __forceinline__ void st_state(float *base, int dv, int dk, int jw, int jl,
                                         const float (&X)[RW][C], int *err, size_t limit,
                                         size_t base_off) {
#pragma unroll
  for (int s = 0; s < RW; ++s) {
    const int j = jw + (s ^ jl);
    if (j < dv && in_bounds(err, base_off + (size_t)j * dk + C <= limit)) st_c<C>(base + (size_t)j * dk, X[s]);
  }
}

// F1: the forward recurrence, writing delta_t of every row, the state
// checkpoints and S_T; `blk` numbers the CTA among F1's.
template <int C, int RW, bool UNR>
__device__ __forceinline__ void f1_body(const BParams &Q, int blk, float *sm) {
  constexpr int VW = 32 * C;            // staged floats per vector
  constexpr int NR = 4 * RW;            // rows per CTA
  constexpr int TS = 3 * VW + NR;       // r | w | alpha | u of the CTA's rows
  const KParams &P = Q.P;
  const int dk = P.dk, dv = P.dv, T = P.T;
  const int nrg = (dv + NR - 1) / NR;
  const int bh = blk / nrg, j0 = (blk % nrg) * NR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jw = j0 + RW * warp;        // the warp's first row
  const int jl = lane / (32 / RW);      // slot s of this lane holds row jw + (s ^ jl)
  const int c0 = C * lane;              // this lane's first key channel
  const bool cok = c0 < dk;
  const int nc = (T + kLCR - 1) / kLCR;
  // This thread's 16-byte piece of every staged token (at most one: 24 C +
  // RW <= 104 pieces for 128 threads), fixed for the whole sweep: r | w |
  // alpha, then the u of the CTA's rows.
  int src_off = 0, dst_off = 0;
  bool piece = false, valid = false;
  {
    const int k = threadIdx.x;
    if (k < 24 * C) {
      const int v = k / (8 * C), col = 4 * (k % (8 * C));
      piece = true;
      valid = col < dk;
      src_off = (v + 1) * dk + (valid ? col : 0);
      dst_off = v * VW + col;
    } else if (k < 24 * C + NR / 4) {
      const int r4 = 4 * (k - 24 * C);
      piece = true;
      valid = j0 + r4 < dv;
      src_off = 4 * dk + (valid ? j0 + r4 : 0);
      dst_off = 3 * VW + r4;
    }
  }
  auto issue = [&](int ch) {
    float *buf = sm + (ch & 1) * kLCR * TS;
    const int t0 = ch * kLCR, n = min(kLCR, T - t0);
    if (!piece || !in_bounds(P.err, t0 + n <= T)) return;
    const float *g = gen_at(Q, bh, t0) + src_off;
    const uint32_t d = smem_u32(buf + dst_off);
    for (int tt = 0; tt < n; ++tt)
      cp_async16(d + tt * TS * 4, g + (size_t)tt * Q.GS, valid);
  };
  float S[RW][C];
  ld_state<C, RW>(P.S0 ? P.S0 + (size_t)bh * dv * dk + c0 : nullptr, dv, dk, jw, jl, cok, S);
  issue(0);
  cp_async_commit();
  for (int ch = 0; ch < nc; ++ch) {
    if (ch + 1 < nc) issue(ch + 1);
    cp_async_commit();
    cp_async_wait_group<1>();
    __syncthreads();
    const float *buf = sm + (ch & 1) * kLCR * TS;
    const int t0 = ch * kLCR, n = min(kLCR, T - t0);
    if (t0 % kCk == 0 && cok) {  // the state before chunk t0 / kCk
      const size_t off = ((size_t)bh * Q.nck + t0 / kCk) * dv * dk + c0;
      st_state<C, RW>(Q.ckS + off, dv, dk, jw, jl, S, P.err, Q.n_ck, off);
    }
    // one token (with UNR, unrolled over a full chunk: constant shared-memory
    // offsets)
    auto step = [&](int tt) {
      const float *sv = buf + tt * TS + c0;
      float rr[C], ww[C], al[C];
      ld_c<C>(sv, rr);
      ld_c<C>(sv + VW, ww);
      ld_c<C>(sv + 2 * VW, al);
      float y[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < C; ++e) {
          S[r][e] *= al[e];
          acc = fmaf(S[r][e], rr[e], acc);
        }
        y[r] = acc;
      }
      // delta of row jw + jl, then every row's delta to every lane
      const float d = buf[tt * TS + 3 * VW + RW * warp + jl] - rows_sum<RW>(y);
      const size_t di = ((size_t)bh * T + t0 + tt) * dv + jw + jl;
      if (lane % (32 / RW) == 0 && jw + jl < dv && in_bounds(P.err, di < Q.n_rows)) Q.delta[di] = d;
      float ds[RW];
      rows_spread<RW>(d, ds);
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int e = 0; e < C; ++e) S[r][e] = fmaf(ds[r], ww[e], S[r][e]);
    };
    if (UNR && n == kLCR) {
#pragma unroll
      for (int tt = 0; tt < kLCR; ++tt) step(tt);
    } else {
      for (int tt = 0; tt < n; ++tt) step(tt);
    }
    __syncthreads();  // the buffer is refilled two chunks on
  }
  if (cok) st_state<C, RW>(Q.st + (size_t)bh * dv * dk + c0, dv, dk, jw, jl, S, P.err, ~(size_t)0, 0);
}

// R1: the reverse recurrence of the cotangent, writing dd_t of every row, the
// cotangent checkpoints and dS0; `blk` numbers the CTA among R1's.
template <int C, int RW, bool UNR>
__device__ __forceinline__ void r1_body(const BParams &Q, int blk, float *sm) {
  constexpr int VW = 32 * C;
  constexpr int NR = 4 * RW;
  constexpr int TS = 4 * VW + NR;  // q' | r | w | alpha | c dO of the CTA's rows
  constexpr int ND = NR / 4;       // c dO pieces per token
  const KParams &P = Q.P;
  const int dk = P.dk, dv = P.dv, T = P.T;
  const int nrg = (dv + NR - 1) / NR;
  const int bh = blk / nrg, j0 = (blk % nrg) * NR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jw = j0 + RW * warp, jl = lane / (32 / RW);
  const int c0 = C * lane;
  const bool cok = c0 < dk;
  constexpr int nd = ND;
  const int nc = (T + kLCR - 1) / kLCR;
  // This thread's 16-byte pieces of every staged token (up to two: 32 C + ND
  // <= 136 pieces for 128 threads), fixed for the whole sweep: q' | r | w |
  // alpha (source: the token's generic vectors), then c dO of the CTA's rows
  // (source: the token's row of cdo).
  int src_off[2] = {0, 0}, dst_off[2] = {0, 0};
  bool piece[2] = {false, false}, valid[2] = {false, false}, is_do[2] = {false, false};
#pragma unroll
  for (int p2 = 0; p2 < 2; ++p2) {
    const int k = threadIdx.x + p2 * (int)blockDim.x;
    if (k < 32 * C) {
      const int v = k / (8 * C), col = 4 * (k % (8 * C));
      piece[p2] = true;
      valid[p2] = col < dk;
      src_off[p2] = v * dk + (valid[p2] ? col : 0);
      dst_off[p2] = v * VW + col;
    } else if (k < 32 * C + nd) {
      const int part = k - 32 * C;
      piece[p2] = true;
      is_do[p2] = true;
      valid[p2] = j0 + 4 * part < dv;
      src_off[p2] = valid[p2] ? j0 + 4 * part : 0;  // floats into the token's cdo row
      dst_off[p2] = 4 * VW + 4 * part;
    }
  }
  auto issue = [&](int ch) {
    float *buf = sm + (ch & 1) * kLCR * TS;
    const int t0 = ch * kLCR, n = min(kLCR, T - t0);
    if (!in_bounds(P.err, ((size_t)bh * T + t0 + n) * dv <= Q.n_rows)) return;
    const float *g = gen_at(Q, bh, t0);
    const float *o0 = Q.cdo + ((size_t)bh * T + t0) * dv;
#pragma unroll
    for (int p2 = 0; p2 < 2; ++p2) {
      if (!piece[p2]) continue;
      const uint32_t d = smem_u32(buf + dst_off[p2]);
      if (is_do[p2]) {
        const float *src = o0 + src_off[p2];
        for (int tt = 0; tt < n; ++tt) cp_async16(d + tt * TS * 4, src + (size_t)tt * dv, valid[p2]);
      } else {
        const float *src = g + src_off[p2];
        for (int tt = 0; tt < n; ++tt) cp_async16(d + tt * TS * 4, src + (size_t)tt * Q.GS, valid[p2]);
      }
    }
  };
  float D[RW][C];
  ld_state<C, RW>(Q.dST ? Q.dST + (size_t)bh * dv * dk + c0 : nullptr, dv, dk, jw, jl, cok, D);
  if (nc > 0) issue(nc - 1);
  cp_async_commit();
  for (int ch = nc - 1; ch >= 0; --ch) {
    if (ch > 0) issue(ch - 1);
    cp_async_commit();
    cp_async_wait_group<1>();
    __syncthreads();
    const float *buf = sm + (ch & 1) * kLCR * TS;
    const int t0 = ch * kLCR, n = min(kLCR, T - t0);
    if (((t0 + n) % kCk == 0 || t0 + n == T) && cok) {  // entering chunk (t0 + n - 1) / kCk
      const size_t off = ((size_t)bh * Q.nck + (t0 + n - 1) / kCk) * dv * dk + c0;
      st_state<C, RW>(Q.ckD + off, dv, dk, jw, jl, D, P.err, Q.n_ck, off);
    }
    auto step = [&](int tt) {
      const float *sv = buf + tt * TS + c0;
      float qq[C], rr[C], ww[C], al[C];
      ld_c<C>(sv, qq);
      ld_c<C>(sv + VW, rr);
      ld_c<C>(sv + 2 * VW, ww);
      ld_c<C>(sv + 3 * VW, al);
      const float *slot = buf + tt * TS + 4 * VW;
      float pr[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        // c dO of the row in slot r
        const float cg = slot[RW * warp + (r ^ jl)];
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < C; ++e) {
          D[r][e] = fmaf(cg, qq[e], D[r][e]);
          acc = fmaf(D[r][e], ww[e], acc);
        }
        pr[r] = acc;
      }
      const float dd = rows_sum<RW>(pr);  // dd of row jw + jl
      const size_t di = ((size_t)bh * T + t0 + tt) * dv + jw + jl;
      if (lane % (32 / RW) == 0 && jw + jl < dv && in_bounds(P.err, di < Q.n_rows)) Q.dd[di] = dd;
      float dds[RW];
      rows_spread<RW>(dd, dds);
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int e = 0; e < C; ++e) D[r][e] = fmaf(-dds[r], rr[e], D[r][e]) * al[e];
    };
    if (UNR && n == kLCR) {
#pragma unroll
      for (int tt = kLCR - 1; tt >= 0; --tt) step(tt);
    } else {
      for (int tt = n - 1; tt >= 0; --tt) step(tt);
    }
    __syncthreads();
  }
  if (cok && Q.dS0) st_state<C, RW>(Q.dS0 + (size_t)bh * dv * dk + c0, dv, dk, jw, jl, D, P.err, ~(size_t)0, 0);
}

// The two row sweeps in one launch: CTAs [0, n_r1) run R1, the rest F1.
template <int C, int RW, bool UNR>
__global__ void __launch_bounds__(128) fr1_kernel(const BParams Q, int n_r1) {
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  if ((int)blockIdx.x < n_r1)
    r1_body<C, RW, UNR>(Q, blockIdx.x, sm);
  else
    f1_body<C, RW, UNR>(Q, blockIdx.x - n_r1, sm);
}

// ---------------------------------------------------------------------------
// Column sweeps F2 / R2. CTA = d_k threads, thread i = key channel i, holding
// rows j0 .. j0 + R - 1 of that column; with delta (F2) or dd (R2) known the
// rows need no reduction, and the column sums over the CTA's rows are
// per-thread. With no feedback left, every kCk-token chunk runs on its own
// CTA from the checkpoint F1 (state) or R1 (cotangent) left at its boundary. Per token the CTA writes its row group's partial sums to
// part[g][bh][t][3][d_k] (slots: c S^T dO, -P^T dd, dS~^T delta).

// Offset of rows j0 .. j0 + R - 1 of token t in a [BH][T][d_v] workspace
// vector (0, after recording the error, when the debug build finds it out of
// range).
__device__ __forceinline__ size_t row_base(const BParams &Q, int bh, int t, int j0, int R) {
  const size_t e = ((size_t)bh * Q.P.T + t) * Q.P.dv + j0;
  return in_bounds(Q.P.err, e + R <= Q.n_rows) ? e : 0;
}

// Stages R floats of a per-row workspace vector (delta, dd or c dO) of token t.
__device__ __forceinline__ void stage_rows(const float *src, int part, float *dst) {
  cp_async16(smem_u32(dst + 4 * part), src + 4 * part, true);
}

// One 16-byte piece of a staged token in F2 / R2: from the token's generic
// vectors (kind 0) or its delta, dd or c dO rows (1, 2, 3); src counts floats
// from that row's start (or, kind 0, from the token's vectors), dst floats
// from the staged token's start. kind -1: no piece. (R divides d_v: every
// row piece is in range.)
struct ColPiece {
  int kind, src, dst;
};
__device__ __forceinline__ ColPiece col_piece(int k, int gen_off, int nv, int rows_dst, int R,
                                              int nd, int j0) {
  const int nr = R / 4;
  if (k < nv) return ColPiece{0, gen_off + 4 * k, 4 * k};
  if (k < nv + 2 * nr + nd) {
    const int q = (k - nv) / nr, part = (k - nv) % nr;  // row vector, piece within it
    return ColPiece{1 + q, j0 + 4 * part, rows_dst + q * R + 4 * part};
  }
  return ColPiece{-1, 0, 0};
}

// Issues the pieces pc of tokens t0 .. t0 + n - 1 into buf (TS floats per
// token); per token each source advances by one row.
__device__ __forceinline__ void col_issue(const BParams &Q, const ColPiece (&pc)[4], int bh, int t0,
                                          int n, float *buf, int TS) {
  const KParams &P = Q.P;
  const int dv = P.dv;
  if (!in_bounds(P.err, ((size_t)bh * P.T + t0 + n) * dv <= Q.n_rows)) return;
  const float *g0 = gen_at(Q, bh, t0);
  const size_t r0 = ((size_t)bh * P.T + t0) * dv;
#pragma unroll
  for (int p2 = 0; p2 < 4; ++p2) {
    const ColPiece c = pc[p2];
    if (c.kind < 0) continue;
    const uint32_t d = smem_u32(buf + c.dst);
    if (c.kind == 0) {
      for (int tt = 0; tt < n; ++tt) cp_async16(d + tt * TS * 4, g0 + (size_t)tt * Q.GS + c.src, true);
    } else {
      const float *src = (c.kind == 1 ? Q.delta : c.kind == 2 ? Q.dd : Q.cdo) + r0 + c.src;
      for (int tt = 0; tt < n; ++tt) cp_async16(d + tt * TS * 4, src + (size_t)tt * dv, true);
    }
  }
}

// F2: forward, S_t = S_{t-1} Diag(alpha_t) + delta_t w_t^T;
// dq'_t = c S_t^T dO_t and dr_t = -P_t^T dd_t. (F2 and R2: at most 128
// registers, four CTAs per SM -- a few spilled bytes, but more warps to wait
// on shared-memory loads with; measured 1.5 % faster than three CTAs.)
// CKT: the chunk-start states are the forward's transposed checkpoint
// (training mode).
template <int R, bool CKT>
__global__ void __launch_bounds__(128, 4) f2_kernel(const BParams Q) {
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  const KParams &P = Q.P;
  const int dk = P.dk, dv = P.dv, T = P.T, BH = P.B * P.H;
  // one CTA per (batch-head, kCk-token chunk, row group)
  const int bh = blockIdx.x / (Q.nck * Q.G), ck = (blockIdx.x / Q.G) % Q.nck;
  const int g = blockIdx.x % Q.G, j0 = g * R;
  const int tb = ck * kCk, te = min(T, tb + kCk);  // this CTA's tokens
  const int i = threadIdx.x;
  const int TS = 2 * dk + 3 * R;  // w | alpha | delta | dd | c dO
  const int nv = dk / 2, nr = R / 4, nd = nr;
  const int nc = (te - tb + kLCC - 1) / kLCC;
  // this thread's pieces of every staged token (w | alpha, delta, dd, c dO)
  ColPiece pc[4];
#pragma unroll
  for (int p2 = 0; p2 < 4; ++p2)
    pc[p2] = col_piece(threadIdx.x + p2 * (int)blockDim.x, 2 * dk, nv, 2 * dk, R, nd, j0);
  auto issue = [&](int ch) {
    float *buf = sm + (ch & 1) * kLCC * TS;
    const int t0 = tb + ch * kLCC, n = min(kLCC, te - t0), per = nv + 2 * nr + nd;
    col_issue(Q, pc, bh, t0, n, buf, TS);
    // (pieces past four per thread: no shape with d_k >= 16 and R <= 64 has any)
    for (int tt = 0; tt < n; ++tt)
    for (int k = threadIdx.x + 4 * (int)blockDim.x; k < per; k += blockDim.x) {
      const int t = t0 + tt;
      float *d = buf + tt * TS;
      if (k < nv)
        cp_async16(smem_u32(d + 4 * k), gen_at(Q, bh, t) + 2 * dk + 4 * k, true);
      else if (k < nv + nr)
        stage_rows(Q.delta + row_base(Q, bh, t, j0, R), k - nv, d + 2 * dk);
      else if (k < nv + 2 * nr)
        stage_rows(Q.dd + row_base(Q, bh, t, j0, R), k - nv - nr, d + 2 * dk + R);
      else
        stage_rows(Q.cdo + row_base(Q, bh, t, j0, R), k - nv - 2 * nr, d + 2 * dk + 2 * R);
    }
  };
  float2 S[R / 2];  // rows (2h, 2h + 1) of this column
  if (CKT && R % 32 == 0 && j0 + R <= dv) {
    // the forward's transposed checkpoint, 32 rows at a time through shared
    // memory (the staging buffer is not in use yet): read straight, each
    // thread's rows are one 128-byte run and a warp load spans 32 lines
#pragma unroll
    for (int h = 0; h < R / 32; ++h) {
      for (int k = threadIdx.x; k < dk * 8; k += blockDim.x) {
        const int c = k >> 3, q4 = k & 7;  // column, float4 of its 32 rows
        const size_t e = (((size_t)bh * Q.nck + ck) * dk + c) * dv + j0 + 32 * h + 4 * q4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (in_bounds(P.err, e + 4 <= Q.n_ck)) x = *reinterpret_cast<const float4 *>(Q.ckS + e);
        float *d = sm + c * 33 + 4 * q4;  // padded rows: no bank conflicts either way
        d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
      }
      __syncthreads();
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int j = 32 * h + jj;
        if (j & 1) S[j / 2].y = sm[i * 33 + jj];
        else S[j / 2].x = sm[i * 33 + jj];
      }
      __syncthreads();
    }
  } else {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const size_t e = CKT ? (((size_t)bh * Q.nck + ck) * dk + i) * dv + j0 + j
                           : (((size_t)bh * Q.nck + ck) * dv + j0 + j) * dk + i;
      const float x = in_bounds(P.err, e < Q.n_ck) ? Q.ckS[e] : 0.f;
      if (j & 1) S[j / 2].y = x;
      else S[j / 2].x = x;
    }
  }
  issue(0);
  cp_async_commit();
  for (int ch = 0; ch < nc; ++ch) {
    if (ch + 1 < nc) issue(ch + 1);
    cp_async_commit();
    cp_async_wait_group<1>();
    __syncthreads();
    const float *buf = sm + (ch & 1) * kLCC * TS;
    const int t0 = tb + ch * kLCC, n = min(kLCC, te - t0);
    for (int tt = 0; tt < n; ++tt) {
      const float *sv = buf + tt * TS;
      const float2 w = dup2(sv[i]), a = dup2(sv[dk + i]);
      float2 accq = make_float2(0.f, 0.f), accr = make_float2(0.f, 0.f);  // even | odd rows
#pragma unroll
      for (int j = 0; j < R; j += 4) {
        float de[4], dd[4], go[4];
        ld4(sv + 2 * dk + j, true, de);
        ld4(sv + 2 * dk + R + j, true, dd);
        ld4(sv + 2 * dk + 2 * R + j, true, go);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 &s2 = S[j / 2 + h];
          const float2 p = mul2(s2, a);
          accr = fma2(p, make_float2(dd[2 * h], dd[2 * h + 1]), accr);
          s2 = fma2(make_float2(de[2 * h], de[2 * h + 1]), w, p);
          accq = fma2(s2, make_float2(go[2 * h], go[2 * h + 1]), accq);
        }
      }
      const size_t po = (((size_t)g * BH + bh) * T + t0 + tt) * 3 * dk;
      if (in_bounds(P.err, po + 3 * dk <= Q.n_part)) {
        Q.part[po + i] = accq.x + accq.y;
        Q.part[po + dk + i] = -(accr.x + accr.y);
      }
    }
    __syncthreads();
  }
}

// R2: reverse, dS~_t = dS_t + c dO_t q'_t^T, dS_{t-1} = (dS~_t - dd_t r_t^T)
// Diag(alpha_t); dw_t = dS~_t^T delta_t.
template <int R>
__global__ void __launch_bounds__(128, 4) r2_kernel(const BParams Q) {
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  const KParams &P = Q.P;
  const int dk = P.dk, dv = P.dv, T = P.T, BH = P.B * P.H;
  // one CTA per (batch-head, kCk-token chunk, row group)
  const int bh = blockIdx.x / (Q.nck * Q.G), ck = (blockIdx.x / Q.G) % Q.nck;
  const int g = blockIdx.x % Q.G, j0 = g * R;
  const int tb = ck * kCk, te = min(T, tb + kCk);  // this CTA's tokens
  const int i = threadIdx.x;
  const int TS = 4 * dk + 3 * R;  // q' | r | w | alpha | delta | dd | c dO
  const int nv = dk, nr = R / 4, nd = nr;
  const int nc = (te - tb + kLCC - 1) / kLCC;
  // this thread's pieces of every staged token (q' | r | w | alpha, delta, dd, c dO)
  ColPiece pc[4];
#pragma unroll
  for (int p2 = 0; p2 < 4; ++p2)
    pc[p2] = col_piece(threadIdx.x + p2 * (int)blockDim.x, 0, nv, 4 * dk, R, nd, j0);
  auto issue = [&](int ch) {
    float *buf = sm + (ch & 1) * kLCC * TS;
    const int t0 = tb + ch * kLCC, n = min(kLCC, te - t0), per = nv + 2 * nr + nd;
    col_issue(Q, pc, bh, t0, n, buf, TS);
    // (pieces past four per thread: no shape with d_k >= 16 and R <= 64 has any)
    for (int tt = 0; tt < n; ++tt)
    for (int k = threadIdx.x + 4 * (int)blockDim.x; k < per; k += blockDim.x) {
      const int t = t0 + tt;
      float *d = buf + tt * TS;
      if (k < nv)
        cp_async16(smem_u32(d + 4 * k), gen_at(Q, bh, t) + 4 * k, true);
      else if (k < nv + nr)
        stage_rows(Q.delta + row_base(Q, bh, t, j0, R), k - nv, d + 4 * dk);
      else if (k < nv + 2 * nr)
        stage_rows(Q.dd + row_base(Q, bh, t, j0, R), k - nv - nr, d + 4 * dk + R);
      else
        stage_rows(Q.cdo + row_base(Q, bh, t, j0, R), k - nv - 2 * nr, d + 4 * dk + 2 * R);
    }
  };
  float2 D[R / 2];  // rows (2h, 2h + 1) of this column
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const size_t e = (((size_t)bh * Q.nck + ck) * dv + j0 + j) * dk + i;
    const float x = in_bounds(P.err, e < Q.n_ck) ? Q.ckD[e] : 0.f;
    if (j & 1) D[j / 2].y = x;
    else D[j / 2].x = x;
  }
  if (nc > 0) issue(nc - 1);
  cp_async_commit();
  for (int ch = nc - 1; ch >= 0; --ch) {
    if (ch > 0) issue(ch - 1);
    cp_async_commit();
    cp_async_wait_group<1>();
    __syncthreads();
    const float *buf = sm + (ch & 1) * kLCC * TS;
    const int t0 = tb + ch * kLCC, n = min(kLCC, te - t0);
    for (int tt = n - 1; tt >= 0; --tt) {
      const float *sv = buf + tt * TS;
      const float2 q2 = dup2(sv[i]), nr2 = dup2(-sv[dk + i]), a = dup2(sv[3 * dk + i]);
      float2 accw = make_float2(0.f, 0.f);  // even | odd rows
#pragma unroll
      for (int j = 0; j < R; j += 4) {
        float de[4], dd[4], go[4];
        ld4(sv + 4 * dk + j, true, de);
        ld4(sv + 4 * dk + R + j, true, dd);
        ld4(sv + 4 * dk + 2 * R + j, true, go);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 &d2 = D[j / 2 + h];
          const float2 dt = fma2(q2, make_float2(go[2 * h], go[2 * h + 1]), d2);
          accw = fma2(dt, make_float2(de[2 * h], de[2 * h + 1]), accw);
          d2 = mul2(fma2(make_float2(dd[2 * h], dd[2 * h + 1]), nr2, dt), a);
        }
      }
      const size_t po = (((size_t)g * BH + bh) * T + t0 + tt) * 3 * dk;
      if (in_bounds(P.err, po + 3 * dk <= Q.n_part)) Q.part[po + 2 * dk + i] = accw.x + accw.y;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// E1: per (token, head), one warp: the row groups' partial sums are added,
// then each variant's map from (q', r, w, u) to its inputs is differentiated
// ("Gated DeltaNet-2" ja §3: the gates' own gradients, derase = k . dr and
// dwrite = v . du). Also the token's term of the decay suffix sum and, for
// the preconditioner, the dA_t of its own coefficients:
//   B = x^-s, s = c / (1 + |c|), c = L - mean(L), L = log(A + eps)
//   => dA = (dc - mean(dc)) / (A + eps), dc = -ln x B dB / (1 + |c|)^2.
// (At most 64 registers: four 256-thread blocks per SM keep enough loads in
// flight; with the compiler's 85, two blocks left it waiting on memory.)
template <typename Tin>
__global__ void __launch_bounds__(256, 4) e1_kernel(const BParams Q) {
  const KParams &P = Q.P;
  const int lane = threadIdx.x & 31, dk = P.dk, dv = P.dv, T = P.T, BH = P.B * P.H;
  const long long n = (long long)BH * T;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < n; wid += nw) {
    const int bh = (int)(wid / T), t = (int)(wid % T);
    const size_t tk = tok_index(P, bh / P.H, t, bh % P.H);
    const int c = 4 * lane;
    const bool ak = c < dk, av = c < dv;
    float dq[4], dr[4], dw[4], du[4], qq[4], r[4], w[4], k[4], v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[e] = dr[e] = dw[e] = 0.f;
    for (int g = 0; g < Q.G; ++g) {
      size_t po = (((size_t)g * BH + bh) * T + t) * 3 * dk;
      if (!in_bounds(P.err, po + 3 * dk <= Q.n_part)) po = 0;
      const float *pp = Q.part + po + c;
      float x[4], y[4], z[4];
      ld4(pp, ak, x);
      ld4(pp + dk, ak, y);
      ld4(pp + 2 * dk, ak, z);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dq[e] += x[e];
        dr[e] += y[e];
        dw[e] += z[e];
      }
    }
    const float *gv = gen_at(Q, bh, t);
    ld4(gv + c, ak, qq);
    ld4(gv + dk + c, ak, r);
    ld4(gv + 2 * dk + c, ak, w);
    ld4(Q.dd + ((size_t)bh * T + t) * dv + c, av, du);
    ld4_opt<Tin>(P.k, tk * dk + c, ak, k);
    ld4_opt<Tin>(P.v, tk * dv + c, av, v);
    // q and k as the recurrence used them (normalised under the prologue)
    const bool l2 = P.prologue & PDN_PRO_L2NORM_QK;
    float qn[4] = {0.f, 0.f, 0.f, 0.f}, iq = 1.f;
    const float ik = l2norm_fwd(P.prologue, k);
    if (l2 || P.variant == PDN_VAR_PLA) {
      ld4_opt<Tin>(P.q, tk * dk + c, ak, qn);
      iq = l2norm_fwd(P.prologue, qn);
    }
    // decay: this token's term q'.dq' - w.dw + r.dr
    if (P.decay != PDN_DECAY_NONE) {
      float cp[4], s = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cp[e] = qq[e] * dq[e] - w[e] * dw[e] + r[e] * dr[e];
        s += cp[e];
      }
      if (P.decay == PDN_DECAY_CHANNEL) {
        if (ak)
          *reinterpret_cast<float4 *>(Q.cpsi + ((size_t)bh * T + t) * dk + c) =
              make_float4(cp[0], cp[1], cp[2], cp[3]);
      } else {
        s = warp_sum(s);
        if (lane == 0) Q.sigma[(size_t)bh * T + t] = s;
      }
    }
    float gq[4], gk[4], gvv[4], dB[4], Bc[4], A[4], L[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gq[e] = dq[e];
      gk[e] = dr[e] + dw[e];
      gvv[e] = du[e];
      dB[e] = 0.f;
      Bc[e] = 1.f;
    }
    const bool pre = is_precond(P.variant);
    float mu = 0.f;
    if (pre) {
      float s = 0.f;
      ld4(Q.acc + ((size_t)bh * T + t) * dk + c, ak, A);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        L[e] = ak ? logf(A[e] + P.eps) : 0.f;
        s += L[e];
      }
      mu = warp_sum(s) / (float)dk;
#pragma unroll
      for (int e = 0; e < 4; ++e) Bc[e] = precond_coef(L[e], mu, P.lnx);
    }
    switch (P.variant) {
      case PDN_VAR_DN: case PDN_VAR_GDN: case PDN_VAR_KDA:
      case PDN_VAR_PDN: case PDN_VAR_PGDN: case PDN_VAR_PKDA: {
        const float be = gate_act(P.prologue, reinterpret_cast<const float *>(P.beta)[tk]);
        float db = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          gk[e] = dr[e] + be * Bc[e] * dw[e];
          db = fmaf(Bc[e] * k[e], dw[e], db);
          dB[e] = be * k[e] * dw[e];
        }
        db = warp_sum(db);
        if (P.prologue & PDN_PRO_SIGMOID_GATES) db *= sigmoid_grad(be);
        if (lane == 0 && Q.dbeta) Q.dbeta[tk] = db;
      } break;
      case PDN_VAR_PLA: {
        const float be = gate_act(P.prologue, reinterpret_cast<const float *>(P.beta)[tk]);
        float db = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          gk[e] = be * dw[e];
          db = fmaf(k[e], dw[e], db);
          dB[e] = qn[e] * dq[e];
          gq[e] = Bc[e] * dq[e];
        }
        db = warp_sum(db);
        if (P.prologue & PDN_PRO_SIGMOID_GATES) db *= sigmoid_grad(be);
        if (lane == 0 && Q.dbeta) Q.dbeta[tk] = db;
      } break;
      case PDN_VAR_FG2_GDN: case PDN_VAR_FG2_GDN_PLUS: {
        const bool plus = P.variant == PDN_VAR_FG2_GDN_PLUS;
        float dbk[4], dwr[4], bkv[4], bvv[4];
        ld4_opt<Tin>(P.beta, tk * dk + c, ak, bkv, 1.f);
        if (plus) ld4_opt<Tin>(P.write, tk * dv + c, av, bvv, 1.f);
        if (P.prologue & PDN_PRO_SIGMOID_GATES) {  // gains as used, sigmoid of the logits (lanes in range)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (ak) bkv[e] = sigmoid_call(bkv[e]);
            if (plus && av) bvv[e] = sigmoid_call(bvv[e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float bk = bkv[e];
          const float sb = sqrtf(bk);
          gk[e] = sb * (dr[e] + dw[e]);
          dbk[e] = k[e] * (dr[e] + dw[e]) / (2.f * sb);
          const float bv = av ? (plus ? bvv[e] : bk) : 1.f;
          const float sv = sqrtf(bv);
          gvv[e] = sv * du[e];
          dwr[e] = v[e] * du[e] / (2.f * sv);
          if (!plus) dbk[e] += dwr[e];
          if (P.prologue & PDN_PRO_SIGMOID_GATES) {  // back to the logits
            dbk[e] *= sigmoid_grad(bk);
            if (plus) dwr[e] *= sigmoid_grad(bv);
          }
        }
        if (Q.dbeta && ak)
          *reinterpret_cast<float4 *>(Q.dbeta + tk * dk + c) = make_float4(dbk[0], dbk[1], dbk[2], dbk[3]);
        if (plus && Q.dwrite && av)
          *reinterpret_cast<float4 *>(Q.dwrite + tk * dv + c) = make_float4(dwr[0], dwr[1], dwr[2], dwr[3]);
      } break;
      case PDN_VAR_GDN2: {
        float de[4], dg[4], erv[4], gwv[4];
        ld4_opt<Tin>(P.erase, tk * dk + c, ak, erv);
        ld4_opt<Tin>(P.write, tk * dv + c, av, gwv);
        gate4(P.prologue, erv);
        gate4(P.prologue, gwv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float er = erv[e];
          const float gw = gwv[e];
          gk[e] = er * dr[e] + dw[e];
          de[e] = k[e] * dr[e];
          gvv[e] = gw * du[e];
          dg[e] = v[e] * du[e];
          if (P.prologue & PDN_PRO_SIGMOID_GATES) {  // back to the logits
            de[e] *= sigmoid_grad(er);
            dg[e] *= sigmoid_grad(gw);
          }
        }
        if (Q.derase && ak)
          *reinterpret_cast<float4 *>(Q.derase + tk * dk + c) = make_float4(de[0], de[1], de[2], de[3]);
        if (Q.dwrite && av)
          *reinterpret_cast<float4 *>(Q.dwrite + tk * dv + c) = make_float4(dg[0], dg[1], dg[2], dg[3]);
      } break;
      default: break;
    }
    if (pre) {
      // dA of this token's own coefficients
      float dc[4], s = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float cc = L[e] - mu;
        const float den = 1.f + fabsf(cc);
        dc[e] = ak ? -P.lnx * Bc[e] * dB[e] / (den * den) : 0.f;
        s += dc[e];
      }
      const float mdc = warp_sum(s) / (float)dk;
      if (ak) {
        float da[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) da[e] = (dc[e] - mdc) / (A[e] + P.eps);
        *reinterpret_cast<float4 *>(Q.dacc + ((size_t)bh * T + t) * dk + c) =
            make_float4(da[0], da[1], da[2], da[3]);
      }
    }
    // back through the normalisation of q, and of k unless the
    // preconditioner's term is still to come (then E3 does it)
    if (l2) {
      l2norm_bwd(qn, gq, iq);
      if (!pre) l2norm_bwd(k, gk, ik);
    }
    if (Q.dq && ak) *reinterpret_cast<float4 *>(Q.dq + tk * dk + c) = make_float4(gq[0], gq[1], gq[2], gq[3]);
    if (Q.dk && ak) *reinterpret_cast<float4 *>(Q.dk + tk * dk + c) = make_float4(gk[0], gk[1], gk[2], gk[3]);
    if (Q.dv && av)
      *reinterpret_cast<float4 *>(Q.dv + tk * dv + c) = make_float4(gvv[0], gvv[1], gvv[2], gvv[3]);
  }
}

// E3 (preconditioned variants): k_t feeds A_s for every s >= t, so
// dk_t += 2 k_t . (sum_{s>=t} dA_s). One warp per (head, kScanBlk-token
// block) walks its tokens from the last, the suffix sum starting from the
// block's carry (the sum over all later blocks, in bsum). Under the L2
// prologue the whole gradient of the normalised k is then taken back
// through the normalisation here.
template <typename Tin>
__global__ void e3_kernel(const BParams Q) {
  const KParams &P = Q.P;
  const int lane = threadIdx.x & 31, dk = P.dk, c = 4 * lane;
  const bool ak = c < dk;
  const long long nblk = (long long)P.B * P.H * Q.nb;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < nblk; wid += nw) {
    const int bh = (int)(wid / Q.nb), blk = (int)(wid % Q.nb);
    const int t_begin = blk * kScanBlk, t_end = min(P.T, t_begin + kScanBlk);
    float y[4];
    ld4(Q.bsum + ((size_t)bh * Q.nb + blk) * dk + c, ak, y);
    for (int t = t_end - 1; t >= t_begin; --t) {
      const size_t o = tok_index(P, bh / P.H, t, bh % P.H) * dk + c;
      float k[4], da[4], g[4];
      ld4_opt<Tin>(P.k, o, ak, k);
      const float ik = l2norm_fwd(P.prologue, k);
      ld4(Q.dacc + ((size_t)bh * P.T + t) * dk + c, ak, da);
      ld4(Q.dk + o, ak, g);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        y[e] += da[e];
        g[e] += 2.f * k[e] * y[e];
      }
      if (P.prologue & PDN_PRO_L2NORM_QK) l2norm_bwd(k, g, ik);
      if (ak) *reinterpret_cast<float4 *>(Q.dk + o) = make_float4(g[0], g[1], g[2], g[3]);
    }
  }
}

// dlog_alpha with respect to the raw decay input x under the decay prologue:
// log alpha = -s softplus(x) gives -s sigmoid(x); log alpha = log sigmoid(x)
// gives sigmoid(-x). Same layout as the input ([B,T,H] or [B,T,H,d_k]).
template <typename Tin>
__global__ void decay_pro_kernel(const BParams Q, long long n) {
  const KParams &P = Q.P;
  const bool ch = P.decay == PDN_DECAY_CHANNEL;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const float x = ch ? ldf<Tin>(P.log_alpha, (size_t)e) : reinterpret_cast<const float *>(P.log_alpha)[e];
    const float d = (P.prologue & PDN_PRO_DECAY_SOFTPLUS) ? -P.decay_scale / (1.f + expf(-x))
                                                          : 1.f / (1.f + expf(x));
    Q.dla[e] *= d;
  }
}

// psi_T,i = sum_j S_T[j,i] dS_T[j,i] per (batch, head), and its sum over i
// (the start of the scalar decay's suffix sum) at phi[BH * d_k + bh].
__global__ void __launch_bounds__(128) phi_kernel(const BParams Q) {
  __shared__ float red[4];
  const KParams &P = Q.P;
  const int bh = blockIdx.x, i = threadIdx.x, dk = P.dk, dv = P.dv;
  float s = 0.f;
  if (i < dk) {
    const size_t base = (size_t)bh * dv * dk + i;
    for (int j = 0; j < dv; ++j) s = fmaf(Q.st[base + (size_t)j * dk], Q.dST[base + (size_t)j * dk], s);
    Q.phi[(size_t)bh * dk + i] = s;
  }
  s = warp_sum(s);
  if ((i & 31) == 0) red[i >> 5] = s;
  __syncthreads();
  if (i == 0) Q.phi[(size_t)P.B * P.H * dk + bh] = red[0] + red[1] + red[2] + red[3];
}

unsigned grid_for(long long n, int threads) {
  const long long b = (n + threads - 1) / threads;
  return (unsigned)(b < 1 ? 1 : (b > 148 * 16 ? 148 * 16 : b));
}

void run_scan(const KParams &P, ScanArr X, ScanArr Y, int nch, int nb, bool rev, const float *init,
              float *total, float *bsum, cudaStream_t st) {
  const long long BH = (long long)P.B * P.H;
  scan_part_kernel<<<grid_for(BH * nb * nch, 256), 256, 0, st>>>(P, X, nch, nb, bsum);
  scan_carry_kernel<<<grid_for(BH * nch, 128), 128, 0, st>>>(P, nch, nb, rev, bsum, init, total);
  scan_fill_kernel<<<grid_for(BH * nb * nch, 256), 256, 0, st>>>(P, X, Y, nch, nb, rev, bsum);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// The merged row sweeps for C key channels per lane and RW rows per warp.
template <int C, int RW, bool UNR>
cudaError_t launch_fr1_t(const BParams &Q, unsigned n, bool r1_only, cudaStream_t st) {
  const size_t smem = 2 * kLCR * (4 * 32 * C + 4 * RW) * sizeof(float);  // R1's (> F1's)
  const cudaError_t err = set_smem(fr1_kernel<C, RW, UNR>, smem);
  if (err != cudaSuccess) return err;
  fr1_kernel<C, RW, UNR><<<r1_only ? n : 2 * n, 128, smem, st>>>(Q, (int)n);
  return cudaSuccess;
}

// Key channels per lane: 32 lanes cover d_k. Rows per warp: 8 (each staged
// vector serves more rows) when that still gives each sweep at least one CTA
// per SM, else 4 (twice the CTAs). The unrolled chunk loop issues fewer
// instructions but schedules worse when too few warps hide its latency, so
// it runs only from one CTA per SM per sweep on. Measured on B200 (ms per
// backward): headline layer (512 CTAs at 8 rows) 5.31 with 8 rows against
// 5.62 with 4; 32 (batch, head) pairs of 32k tokens 24.3 with 8 rows (rolled)
// against 22.6 with 4 (unrolled); unrolled against rolled at 8 rows there:
// 28.7 against 26.1. The same rules hold for R1 launched alone (training
// mode, ms per training-mode backward): headline layer (256 CTAs at 8 rows)
// 4.23 with 8 rows against 4.37 with 4, and 4.25 unrolled against 4.53
// rolled; 32 pairs of 32k tokens (128 CTAs at 8 rows) 19.25 with 4 rows
// against 20.79 with 8, and 19.3 unrolled against 20.3 rolled.
template <int C>
cudaError_t launch_fr1_c(const BParams &Q, unsigned n, bool rw8, bool unr, bool r1_only,
                         cudaStream_t st) {
  if (rw8)
    return unr ? launch_fr1_t<C, 8, true>(Q, n, r1_only, st) : launch_fr1_t<C, 8, false>(Q, n, r1_only, st);
  return unr ? launch_fr1_t<C, 4, true>(Q, n, r1_only, st) : launch_fr1_t<C, 4, false>(Q, n, r1_only, st);
}
cudaError_t launch_fr1(const BParams &Q, cudaStream_t st) {
  const KParams &P = Q.P;
  const bool r1_only = P.sv_delta && P.sv_ckpt;  // training mode: F1's outputs are saved
  const long long BH = (long long)P.B * P.H, sms = num_sms();
  const long long n8 = BH * ((P.dv + 31) / 32);  // CTAs per sweep at 8 rows per warp
  const bool rw8 = n8 >= sms;  // >= 1 CTA per SM per sweep
  const unsigned n = (unsigned)(rw8 ? n8 : BH * ((P.dv + 15) / 16));
  const bool unr = (long long)n >= sms;
  if (P.dk > 64) return launch_fr1_c<4>(Q, n, rw8, unr, r1_only, st);
  if (P.dk > 32) return launch_fr1_c<2>(Q, n, rw8, unr, r1_only, st);
  return launch_fr1_c<1>(Q, n, rw8, unr, r1_only, st);
}

template <typename Tin, int R>
cudaError_t launch_bwd_t(const BParams &Q, cudaStream_t st) {
  const KParams &P = Q.P;
  const int dk = P.dk;
  const long long BH = (long long)P.B * P.H, BHT = BH * P.T;
  cudaError_t err;
  if (is_precond(P.variant)) {
    ksq_part_kernel<Tin><<<grid_for(BH * Q.nb * 32, 256), 256, 0, st>>>(Q);
    scan_carry_kernel<<<grid_for(BH * dk, 128), 128, 0, st>>>(P, dk, Q.nb, false, Q.bsum, P.A0,
                                                             nullptr);
  }
  prep_gen_kernel<Tin><<<grid_for(BH * Q.nb * 32, 256), 256, 0, st>>>(Q);

  const size_t sm_f2 = 2 * kLCC * (2 * dk + 3 * R) * sizeof(float);
  const size_t sm_r2 = 2 * kLCC * (4 * dk + 3 * R) * sizeof(float);
  if ((err = set_smem(Q.ck_t ? f2_kernel<R, true> : f2_kernel<R, false>, sm_f2)) != cudaSuccess)
    return err;
  if ((err = set_smem(r2_kernel<R>, sm_r2)) != cudaSuccess) return err;
  const unsigned grid_cols = (unsigned)(BH * Q.nck * Q.G);
  if ((err = launch_fr1(Q, st)) != cudaSuccess) return err;
  if (Q.ck_t) f2_kernel<R, true><<<grid_cols, dk, sm_f2, st>>>(Q);
  else f2_kernel<R, false><<<grid_cols, dk, sm_f2, st>>>(Q);
  r2_kernel<R><<<grid_cols, dk, sm_r2, st>>>(Q);
  e1_kernel<Tin><<<grid_for(BHT * 32, 256), 256, 0, st>>>(Q);

  if (P.decay != PDN_DECAY_NONE && Q.dla) {
    if (Q.dST) phi_kernel<<<(unsigned)BH, 128, 0, st>>>(Q);
    if (P.decay == PDN_DECAY_CHANNEL)
      run_scan(P, ScanArr{Q.cpsi, false}, ScanArr{Q.dla, true}, dk, Q.nb, true,
               Q.dST ? Q.phi : nullptr, nullptr, Q.bsum, st);
    else
      run_scan(P, ScanArr{Q.sigma, false}, ScanArr{Q.dla, true}, 1, Q.nb, true,
               Q.dST ? Q.phi + BH * dk : nullptr, nullptr, Q.bsum, st);
    if (P.prologue & (PDN_PRO_DECAY_SOFTPLUS | PDN_PRO_DECAY_LOGSIGMOID)) {
      const long long n = BHT * (P.decay == PDN_DECAY_CHANNEL ? dk : 1);
      decay_pro_kernel<Tin><<<grid_for(n, 256), 256, 0, st>>>(Q, n);
    }
  }
  if (is_precond(P.variant) && (Q.dk || Q.dA0)) {
    // block totals of dA and the carries from the sequence end (dA0 gets
    // the full sum); E3 finishes the suffix sums inside the blocks
    scan_part_kernel<<<grid_for(BH * Q.nb * dk, 256), 256, 0, st>>>(P, ScanArr{Q.dacc, false}, dk,
                                                                    Q.nb, Q.bsum);
    scan_carry_kernel<<<grid_for(BH * dk, 128), 128, 0, st>>>(P, dk, Q.nb, true, Q.bsum, nullptr,
                                                             Q.dA0);
    if (Q.dk) e3_kernel<Tin><<<grid_for(BH * Q.nb * 32, 256), 256, 0, st>>>(Q);
  }
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_bwd_d(const BParams &Q, int R, cudaStream_t st) {
  if (R == 64) return launch_bwd_t<Tin, 64>(Q, st);
  if (R == 32) return launch_bwd_t<Tin, 32>(Q, st);
  return launch_bwd_t<Tin, 16>(Q, st);
}

}  // namespace

size_t bwd_workspace_bytes(const KParams &P) { return bwd_plan(P).total * sizeof(float); }

cudaError_t launch_chunk_bwd(const KParams &P, const pdn_grads_t *g, void *workspace,
                             cudaStream_t stream) {
  const long long BH = (long long)P.B * P.H;
  if (P.T == 0) {
    // no token: the initial state is the final state, A0 reaches nothing
    cudaError_t err = cudaSuccess;
    if (g->dS0) {
      const size_t bytes = (size_t)BH * P.dv * P.dk * sizeof(float);
      err = g->dST ? cudaMemcpyAsync(g->dS0, g->dST, bytes, cudaMemcpyDeviceToDevice, stream)
                   : cudaMemsetAsync(g->dS0, 0, bytes, stream);
      if (err != cudaSuccess) return err;
    }
    if (g->dA0 && is_precond(P.variant))
      err = cudaMemsetAsync(g->dA0, 0, (size_t)BH * P.dk * sizeof(float), stream);
    return err;
  }
  const BwdPlan L = bwd_plan(P);
  float *ws = static_cast<float *>(workspace);
  BParams Q;
  memset(&Q, 0, sizeof(Q));
  Q.P = P;
  Q.dO = g->dO; Q.dST = g->dST;
  Q.dq = g->dq; Q.dk = g->dk; Q.dv = g->dv; Q.dla = g->dlog_alpha; Q.dbeta = g->dbeta;
  Q.derase = g->derase; Q.dwrite = g->dwrite; Q.dS0 = g->dS0; Q.dA0 = g->dA0;
  Q.gen = ws + L.gen; Q.acc = ws + L.acc; Q.delta = ws + L.delta; Q.dd = ws + L.dd;
  Q.cdo = ws + L.cdo;
  Q.st = ws + L.st; Q.part = ws + L.part; Q.cpsi = ws + L.cpsi; Q.sigma = ws + L.sigma;
  Q.dacc = ws + L.dacc; Q.bsum = ws + L.bsum; Q.phi = ws + L.phi;
  Q.ckS = ws + L.ckS; Q.ckD = ws + L.ckD;
  if (P.sv_delta && P.sv_ckpt) {
    // training mode: delta, the chunk-start states and S_T come from the
    // forward (pdn_chunk_fwd_save); the forward row sweep F1 is skipped
    Q.delta = P.sv_delta;
    Q.ckS = P.sv_ckpt;
    Q.ck_t = true;
    Q.st = P.ST;
  }
  Q.GS = L.GS; Q.R = L.R; Q.G = L.G; Q.nb = L.nb; Q.nck = L.nck;
  Q.n_rows = (size_t)BH * P.T * P.dv;
  Q.n_part = (size_t)L.G * BH * P.T * 3 * P.dk;
  Q.n_ck = (size_t)BH * L.nck * P.dv * P.dk;
  if (P.dtype == PDN_BF16) return launch_bwd_d<__nv_bfloat16>(Q, L.R, stream);
  return launch_bwd_d<float>(Q, L.R, stream);
}

}  // namespace pdn
