// chunk_tc.cu -- chunked forward of the gated delta rule on the sm_100a tensor
// cores (tcgen05.mma, bf16 operands, fp32 accumulators in tensor memory).
//
// One CTA owns one (batch, head) chain, d_k = d_v = 128, and walks its chunks
// of C = 64 tokens in order. The fp32 master state S (d_v x d_k) lives in
// tensor memory for the whole sequence; a bf16 copy in shared memory is the
// MMA operand. Per chunk (the chunkwise WY/UT form: "Gated DeltaNet-2", ja §3,
// decay absorbed into the erase/write matrices, lower-triangular (I+T)^{-1}
// solve for the erase-side auxiliary Y and the write-side auxiliary U;
// "Preconditioned DeltaNet", ja §2.3, prefix-sum preconditioner in the chunk
// form; "FG2-GDN", ja §2.3, same diagonal-plus-low-rank chunk algorithm):
//
//   prep (CUDA cores): G = in-chunk cumulative log decay, preconditioner
//     A_t = A_{t-1} + k.k, B_t = x^{-s}, write key w per variant, then
//     Rh = e^G.r, Qh = q_scale e^G.q, Wh = e^{-G}.w, Wb = e^{G_C-G}.w  (bf16)
//   MMA1  [Rh;Qh] Wh^T                -> M (strict lower) and P (lower)
//   solve T = (I + M)^{-1}            (blocked 16x16 substitution, fp32)
//   MMA2  Y^T  = Rh^T T^T
//   MMA3  U^T  = U^T T^T
//   MMA5  D^T  = U^T - S Y^T          (negated-A accumulate, in place)
//   MMA6  O^T  = S Qh^T
//   MMA7  O^T += D^T P^T
//   MMA8  S   += D^T Wb               (S pre-scaled by Diag(e^{G_C}))
//
// Every MMA is M = 128 (d_v or d_k rows on the 128 TMEM lanes), N = 64 or
// 128, K = 16 per instruction, operands in the no-swizzle canonical layout:
// "TL" tiles of 8-row x 16-byte core matrices, row-groups major. A TL tile
// with rows = tokens serves both as a K-major operand (K = channels) and as
// an MN-major operand (K = tokens), so no operand is transposed in memory.
//
// The exponent factorisation needs the in-chunk cumulative log decay of each
// channel to stay above about -80 (fp32 range of e^{-G}).
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tiles.cuh"

// Phase boundary hook for out-of-tree timing harnesses; empty in the library.
#ifndef PDN_PHASE_MARK
#define PDN_PHASE_MARK(k)
#endif

namespace pdn {
namespace {

constexpr int kThreads = 256;
constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // d_k = d_v

// ---- shared memory map (bytes) -------------------------------------------
constexpr uint32_t OFF_RQ = 0;          // TL 128 x 128: rows 0-63 Rh, 64-127 Qh
constexpr uint32_t OFF_WH = 32768;      // TL  64 x 128
constexpr uint32_t OFF_WB = 49152;      // TL  64 x 128
constexpr uint32_t OFF_U = 65536;       // TL  64 x 128 (v staged here)
constexpr uint32_t OFF_SB = 81920;      // TL 128 x 128 bf16 copy of S (rows = d_v); between
                                        // the S-products and the next state epilogue it
                                        // stages the next chunk's channel log-decay
constexpr uint32_t KS_LD = 272;         // staged row stride (bytes), padded
constexpr uint32_t OFF_KS = 114688;     // raw k, row-major [64][128] bf16
constexpr uint32_t OFF_QS = OFF_KS + 64 * KS_LD;
constexpr uint32_t OFF_RA = OFF_QS + 64 * KS_LD;  // region A (phase-dependent)
constexpr int LB_LD = 132;              // floats per row of the fp32 prep buffers
constexpr uint32_t OFF_LBUF = OFF_RA;                    // prep: log2(A + eps)
constexpr uint32_t OFF_GBUF = OFF_RA + 64 * LB_LD * 4;   // prep: cumulative log decay
constexpr int MS_LD = 68, TS_LD = 68, YS_LD = 34;        // fp32 solve scratch strides
constexpr uint32_t OFF_TM = OFF_RA;                      // TL 64 x 64: T
constexpr uint32_t OFF_PM = OFF_RA + 8192;               // TL 64 x 64: P
constexpr uint32_t OFF_MS = OFF_RA + 16384;              // fp32 [64][68]: M
constexpr uint32_t OFF_TS = OFF_MS + 64 * MS_LD * 4;     // fp32 [64][68]: T
constexpr uint32_t OFF_YS = OFF_TS + 64 * TS_LD * 4;     // fp32 [32][34]: merge scratch
constexpr uint32_t OFF_YT = OFF_RA + 16384;              // TL 128 x 64: Y^T (rows d_k)
constexpr uint32_t OFF_DT = OFF_RA + 32768;              // TL 128 x 64: D^T (rows d_v)
constexpr uint32_t RA_BYTES = 2 * 64 * LB_LD * 4;
constexpr uint32_t OFF_SMALL = OFF_RA + RA_BYTES;
constexpr uint32_t OFF_ACAR = OFF_SMALL;          // float[128] accumulator carry
constexpr uint32_t OFF_GC = OFF_SMALL + 512;      // float[128] G at chunk end
constexpr uint32_t OFF_EGC = OFF_SMALL + 1024;    // float[128] e^{G_C}
constexpr uint32_t OFF_PARTK = OFF_SMALL + 1536;  // float[128] first-half key energy
constexpr uint32_t OFF_PARTG = OFF_SMALL + 2048;  // float[128] first-half log decay
constexpr uint32_t OFF_MU = OFF_SMALL + 2560;     // float[64] mean log2(A + eps)
constexpr uint32_t OFF_BETA = OFF_SMALL + 2816;   // float[64] scalar gain (staged)
constexpr uint32_t OFF_GS = OFF_SMALL + 3072;     // float[64] scalar cumulative decay
constexpr uint32_t OFF_LAS = OFF_SMALL + 3328;    // float[64] scalar log decay (staged)
constexpr uint32_t OFF_BAR = OFF_SMALL + 3584;    // uint64[kNumBars] mbarriers
constexpr int kNumBars = 6;                       // one per MMA group, see below
constexpr uint32_t OFF_TBASE = OFF_BAR + 8 * kNumBars;  // uint32 TMEM base
constexpr uint32_t SMEM_BYTES = OFF_TBASE + 16;
static_assert(OFF_YS + 32 * YS_LD * 4 <= OFF_RA + RA_BYTES, "region A overflow");
static_assert(OFF_DT + 16384 <= OFF_RA + RA_BYTES, "region A overflow");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- TMEM columns ---------------------------------------------------------
constexpr uint32_t TM_D1 = 0;    // [Rh;Qh] Wh^T    (128 x 64)
constexpr uint32_t TM_YT = 64;   // Y^T             (128 x 64)
constexpr uint32_t TM_UD = 128;  // U^T, then D^T   (128 x 64)
constexpr uint32_t TM_OT = 192;  // O^T, even chunks (128 x 64)
constexpr uint32_t TM_S = 256;   // S               (128 x 128)
constexpr uint32_t TM_OT1 = 384; // O^T, odd chunks  (128 x 64)
constexpr uint32_t TM_COLS = 512;

constexpr long long kSpinLimit = 1LL << 22;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kMinG = -80.f;  // floor of the in-chunk cumulative log decay (fp32 range)

// ---- staging of the next chunk's raw inputs (cp.async, zero-filled tail) ----
template <int kVariant, int kDecay>
__device__ __forceinline__ void stage_kq(const KParams &P, uint32_t sb, int b, int h, int c0,
                                         int Cn, int tid) {
  const __nv_bfloat16 *k = reinterpret_cast<const __nv_bfloat16 *>(P.k);
  const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(P.q);
  const size_t tstride = (size_t)P.H * kD;
  const size_t base = tok_index(P, b, c0, h) * kD + (tid & 15) * 8;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
    const bool ok = t < Cn;
    const size_t e = ok ? base + t * tstride : 0;
    cp_async16(sb + OFF_KS + t * KS_LD + c8 * 16, k + e, ok);
    cp_async16(sb + OFF_QS + t * KS_LD + c8 * 16, q + e, ok);
  }
  if (tid < kC) {
    const bool ok = tid < Cn;
    const size_t e = ok ? tok_index(P, b, c0 + tid, h) : 0;
    if (kVariant != PDN_VAR_FG2_GDN && kVariant != PDN_VAR_GDN2)
      cp_async4(sb + OFF_BETA + 4 * tid, reinterpret_cast<const float *>(P.beta) + e, ok);
    if (kDecay == PDN_DECAY_SCALAR)
      cp_async4(sb + OFF_LAS + 4 * tid, reinterpret_cast<const float *>(P.log_alpha) + e, ok);
  }
  cp_async_commit();
}

// v into its TL operand tile (or the channel log-decay, row-major, into SB).
__device__ __forceinline__ void stage_rows(const KParams &P, const void *src_t, uint32_t dst,
                                           bool tl, int b, int h, int c0, int Cn, int tid) {
  const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(src_t);
  const size_t tstride = (size_t)P.H * kD;
  const size_t base = tok_index(P, b, c0, h) * kD + (tid & 15) * 8;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
    const bool ok = t < Cn;
    const size_t e = ok ? base + t * tstride : 0;
    cp_async16(dst + (tl ? tl128(t, c8) : (uint32_t)(t * 256 + c8 * 16)), src + e, ok);
  }
  cp_async_commit();
}

__device__ __forceinline__ uint32_t ot_col(int n) { return (n & 1) ? TM_OT1 : TM_OT; }

// Writes the 64 x 128 output tile of chunk starting at token pc0 (rows of
// O^T in TMEM lanes, tokens in columns) to HBM. Warp-collective; the warp
// covers its TMEM lane quarter (32 value channels) and all 64 tokens.
__device__ __forceinline__ void store_o_tile(const KParams &P, uint32_t taddr, int b, int h,
                                             int pc0, int Cn, int lane, int quarter) {
  const size_t tstride = (size_t)P.H * kD;
  const int j = 32 * quarter + lane;
  __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(P.o) + tok_index(P, b, pc0, h) * kD + (j & ~1);
  const bool odd = lane & 1;
#pragma unroll
  for (int hc = 0; hc < 2; ++hc) {
    float ov[2][16];
    tmem_ld16(taddr + 32 * hc, ov[0]);
    tmem_ld16(taddr + 32 * hc + 16, ov[1]);
    tmem_wait_ld();
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const float *v = ov[cc];
      // lane pairs (j, j^1) exchange values so each stores two adjacent columns
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        const float send = odd ? v[2 * e2] : v[2 * e2 + 1];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
        const int t = 32 * hc + 16 * cc + 2 * e2 + (odd ? 1 : 0);
        const float lo = odd ? recv : v[2 * e2];
        const float hi = odd ? v[2 * e2 + 1] : recv;
        if (t < Cn) *reinterpret_cast<uint32_t *>(orow + t * tstride) = pack_bf16(lo, hi);
      }
    }
  }
}

// Same for the 32 tokens [t0, t0 + 32) of the tile (taddr points at column t0).
__device__ __forceinline__ void store_o_half(const KParams &P, uint32_t taddr, int b, int h,
                                             int pc0, int Cn, int t0, int lane, int quarter) {
  const size_t tstride = (size_t)P.H * kD;
  const int j = 32 * quarter + lane;
  __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(P.o) + tok_index(P, b, pc0, h) * kD + (j & ~1);
  const bool odd = lane & 1;
  float ov[2][16];
  tmem_ld16(taddr, ov[0]);
  tmem_ld16(taddr + 16, ov[1]);
  tmem_wait_ld();
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const float *v = ov[cc];
#pragma unroll
    for (int e2 = 0; e2 < 8; ++e2) {
      const float send = odd ? v[2 * e2] : v[2 * e2 + 1];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      const int t = t0 + 16 * cc + 2 * e2 + (odd ? 1 : 0);
      const float lo = odd ? recv : v[2 * e2];
      const float hi = odd ? v[2 * e2 + 1] : recv;
      if (t < Cn) *reinterpret_cast<uint32_t *>(orow + t * tstride) = pack_bf16(lo, hi);
    }
  }
}

__device__ __forceinline__ void mma_sync_point() {
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

template <int kVariant, int kDecay>
__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(const KParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  float *Acar = reinterpret_cast<float *>(smem + OFF_ACAR);
  float *GC = reinterpret_cast<float *>(smem + OFF_GC);
  float *EGC = reinterpret_cast<float *>(smem + OFF_EGC);
  float *PARTK = reinterpret_cast<float *>(smem + OFF_PARTK);
  float *PARTG = reinterpret_cast<float *>(smem + OFF_PARTG);
  float *MU = reinterpret_cast<float *>(smem + OFF_MU);
  float *BETA = reinterpret_cast<float *>(smem + OFF_BETA);
  float *GS = reinterpret_cast<float *>(smem + OFF_GS);
  float *LAS = reinterpret_cast<float *>(smem + OFF_LAS);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tbase_p = reinterpret_cast<uint32_t *>(smem + OFF_TBASE);
  float *LBUF = reinterpret_cast<float *>(smem + OFF_LBUF);
  float *GBUF = reinterpret_cast<float *>(smem + OFF_GBUF);
  float *MS = reinterpret_cast<float *>(smem + OFF_MS);
  float *TS = reinterpret_cast<float *>(smem + OFF_TS);
  float *YS = reinterpret_cast<float *>(smem + OFF_YS);

  constexpr bool kPre = kVariant == PDN_VAR_PDN || kVariant == PDN_VAR_PGDN ||
                        kVariant == PDN_VAR_PKDA;
  constexpr bool kScalarBeta = kVariant != PDN_VAR_FG2_GDN && kVariant != PDN_VAR_GDN2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int b = bh / P.H, h = bh % P.H;
  const int nchunks = (P.T + kC - 1) / kC;
  const float log2x = P.lnx * kLog2e;
  const uint32_t lane_q = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter
  const int half = warp >> 2;

  // ---- set-up: TMEM, barrier, accumulator, first chunk in flight ----
  if (warp == 0) {
    tmem_alloc(tbase_p, TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar + i, 1);
    fence_mbarrier_init();
  }
  if (tid < kD) Acar[tid] = (kPre && P.A0) ? P.A0[(size_t)bh * kD + tid] : 0.f;
  {
    const int Cn0 = min(kC, P.T);
    stage_kq<kVariant, kDecay>(P, sb, b, h, 0, Cn0, tid);
    stage_rows(P, P.v, sb + OFF_U, true, b, h, 0, Cn0, tid);
    if (kDecay == PDN_DECAY_CHANNEL) stage_rows(P, P.log_alpha, sb + OFF_SB, false, b, h, 0, Cn0, tid);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tbase_p;
  bool aborted = false;
  // MMA groups, each committed to its own mbarrier once per chunk (so the
  // wait parity is the chunk index mod 2):
  uint64_t *bar_m1 = bar + 0;  // MMA1  [Rh;Qh] Wh^T
  uint64_t *bar_m6 = bar + 1;  // MMA6  O^T = S Qh^T
  uint64_t *bar_m2 = bar + 2;  // MMA2  Y^T
  uint64_t *bar_m3 = bar + 3;  // MMA3  U^T
  uint64_t *bar_m5 = bar + 4;  // MMA5  D^T -= S Y^T
  uint64_t *bar_m7 = bar + 5;  // MMA7/8

  // Only warp 0 polls; the other warps park at the block barrier, leaving
  // the issue slots and the shared-memory pipe to warps with work.
  auto wait_mma = [&](uint64_t *b_, int n_) -> bool {
    bool ok = true;
    if (warp == 0) ok = mbar_wait_bounded(b_, (uint32_t)(n_ & 1), kSpinLimit);
    const bool any_fail = __syncthreads_or(!ok);
    tc_fence_after();
    if (any_fail && tid == 0) record_error(P.err, PDN_ERR_TIMEOUT);
    return !any_fail;
  };

  for (int n = 0; n < nchunks && !aborted; ++n) {
    const int c0 = n * kC;
    const int Cn = min(kC, P.T - c0);
    const int Cn_next = min(kC, P.T - c0 - kC);  // <= 0 past the last chunk
    PDN_PHASE_MARK(0);
    cp_async_wait_all();
    __syncthreads();
    PDN_PHASE_MARK(1);

    // ---- prep P1: per-channel scans; thread = (channel, half of the chunk) ----
    {
      const int i = tid & 127, hf = tid >> 7, t0 = 32 * hf;
      float kk[32], la[32];
      float ks = 0.f, gs = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        kk[e] = 0.f;
        la[e] = 0.f;
        if (kPre) {
          kk[e] = __bfloat162float(
              *reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_KS + (t0 + e) * KS_LD + i * 2));
          ks = fmaf(kk[e], kk[e], ks);
        }
        if (kDecay == PDN_DECAY_CHANNEL)
          la[e] = __bfloat162float(
              *reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_SB + (t0 + e) * 256 + i * 2));
        else if (kDecay == PDN_DECAY_SCALAR)
          la[e] = LAS[t0 + e];
        gs += la[e];
      }
      if (hf == 0) {
        PARTK[i] = ks;
        PARTG[i] = gs;
      }
      __syncthreads();
      PDN_PHASE_MARK(16);
      float a = Acar[i] + (hf ? PARTK[i] : 0.f);
      float g = hf ? PARTG[i] : 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int t = t0 + e;
        if (kPre) {
          a = fmaf(kk[e], kk[e], a);
          LBUF[t * LB_LD + i] = lg2_approx(a + P.eps);
        }
        g += la[e];
        if (kDecay == PDN_DECAY_CHANNEL) GBUF[t * LB_LD + i] = g;
        else if (kDecay == PDN_DECAY_SCALAR && i == 0) GS[t] = g;
      }
      if (hf) {
        Acar[i] = a;
        GC[i] = g;
        EGC[i] = ex2_approx(fmaxf(g, kMinG) * kLog2e);
      }
    }
    __syncthreads();
    PDN_PHASE_MARK(2);
    PDN_PHASE_MARK(3);

    // ---- prep P2: per-token channel mean of log2(A + eps) ----
    if (kPre) {
      const int t = tid >> 2, qd = tid & 3;
      float s = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        const float4 x = *reinterpret_cast<const float4 *>(LBUF + t * LB_LD + qd * 32 + 4 * k4);
        s += (x.x + x.y) + (x.z + x.w);
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (qd == 0) MU[t] = s * (1.f / kD);
      __syncthreads();
    }
    PDN_PHASE_MARK(4);

    // ---- prep P3: operand tiles, (token, 8-channel) units ----
    {
      const int t = 8 * warp + (lane & 7);
      const bool ok = t < Cn;
      const size_t etok = ok ? tok_index(P, b, c0 + t, h) * kD : 0;
      float eg_s = 1.f, emg_s = 1.f, ewb_s = 1.f;
      if (kDecay == PDN_DECAY_SCALAR) {
        eg_s = ex2_approx(fmaxf(GS[t], kMinG) * kLog2e);
        emg_s = rcp_approx(eg_s);
        ewb_s = EGC[0] * emg_s;
      }
      const float be = kScalarBeta ? BETA[t] : 0.f;
      const float mu = kPre ? MU[t] : 0.f;
      const float qs = P.q_scale;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c8 = 4 * m + (lane >> 3);
        const int i0 = 8 * c8;
        float kf[8], qf[8], r[8], w[8];
        unpack8(*reinterpret_cast<const uint4 *>(smem + OFF_KS + t * KS_LD + c8 * 16), kf);
        unpack8(*reinterpret_cast<const uint4 *>(smem + OFF_QS + t * KS_LD + c8 * 16), qf);
        if (kPre) {
          float L[8];
          ld8f(LBUF + t * LB_LD + i0, L);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float cc = (L[c] - mu) * kLn2;
            const float s = cc * rcp_approx(1.f + fabsf(cc));
            r[c] = kf[c];
            w[c] = be * ex2_approx(-s * log2x) * kf[c];
          }
        } else if (kVariant == PDN_VAR_FG2_GDN) {
          float gb[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) gb[c] = 0.f;
          if (ok)
            unpack8(__ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(P.beta) + etok + i0)), gb);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[c] = sqrtf(gb[c]) * kf[c];
            w[c] = r[c];
          }
        } else if (kVariant == PDN_VAR_GDN2) {
          float ge[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) ge[c] = 0.f;
          if (ok)
            unpack8(__ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(P.erase) + etok + i0)), ge);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[c] = ge[c] * kf[c];
            w[c] = kf[c];
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            r[c] = kf[c];
            w[c] = be * kf[c];
          }
        }
        float rh[8], qh[8], wh[8], wb[8];
        if (kDecay == PDN_DECAY_CHANNEL) {
          float G[8], E[8];
          ld8f(GBUF + t * LB_LD + i0, G);
          ld8f(EGC + i0, E);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float eg = ex2_approx(fmaxf(G[c], kMinG) * kLog2e);
            const float emg = rcp_approx(eg);
            rh[c] = r[c] * eg;
            qh[c] = qs * qf[c] * eg;
            wh[c] = w[c] * emg;
            wb[c] = w[c] * (E[c] * emg);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            rh[c] = r[c] * eg_s;
            qh[c] = (qs * eg_s) * qf[c];
            wh[c] = w[c] * emg_s;
            wb[c] = w[c] * ewb_s;
          }
        }
        *reinterpret_cast<uint4 *>(smem + OFF_RQ + tl128(t, c8)) = pack8(rh);
        *reinterpret_cast<uint4 *>(smem + OFF_RQ + tl128(64 + t, c8)) = pack8(qh);
        *reinterpret_cast<uint4 *>(smem + OFF_WH + tl128(t, c8)) = pack8(wh);
        *reinterpret_cast<uint4 *>(smem + OFF_WB + tl128(t, c8)) = pack8(wb);
        if (kVariant == PDN_VAR_FG2_GDN || kVariant == PDN_VAR_GDN2) {
          // u = sqrt(beta) . v (FG2) or write-gate . v (GDN-2), in the staged tile
          float uf[8], gt[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) gt[c] = 0.f;
          uint4 *up = reinterpret_cast<uint4 *>(smem + OFF_U + tl128(t, c8));
          unpack8(*up, uf);
          if (ok) {
            const void *gp = kVariant == PDN_VAR_FG2_GDN ? P.beta : P.write;
            unpack8(__ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(gp) + etok + i0)), gt);
          }
#pragma unroll
          for (int c = 0; c < 8; ++c)
            uf[c] *= (kVariant == PDN_VAR_FG2_GDN ? sqrtf(gt[c]) : gt[c]);
          *up = pack8(uf);
        }
      }
    }
    __syncthreads();
    PDN_PHASE_MARK(5);

    // k, q and the scalar gates of the next chunk fly during the rest of this one
    if (Cn_next > 0) stage_kq<kVariant, kDecay>(P, sb, b, h, c0 + kC, Cn_next, tid);

    // ---- MMA1: D1 = [Rh;Qh] Wh^T  (runs under the state epilogue) ----
    mma_sync_point();
    if (tid == 0) {
      const uint32_t id = make_idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TM_D1, make_sdesc(sb + OFF_RQ + 256 * kk, 128, 2048),
                    make_sdesc(sb + OFF_WH + 256 * kk, 128, 2048), id, kk > 0);
      mma_commit(bar_m1);
    }

    // ---- state epilogue of the previous chunk (or the initial state) ----
    // O of the previous chunk -> HBM; S (TMEM, fp32) -> bf16 operand copy;
    // TMEM S <- S Diag(e^{G_C}) for this chunk.
    {
      const int j = 32 * (warp & 3) + lane;
      if (n > 0) store_o_half(P, tm + lane_q + ot_col(n - 1) + 32 * half, b, h, c0 - kC, kC,
                              32 * half, lane, warp & 3);
#pragma unroll
      for (int cp = 0; cp < 2; ++cp) {
        float sv[2][16];
        if (n == 0) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 64 * half + 32 * cp + 16 * u;
            if (P.S0) {
              const float4 *src = reinterpret_cast<const float4 *>(
                  P.S0 + ((size_t)bh * kD + j) * kD + col);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float4 x = __ldg(src + e);
                sv[u][4 * e] = x.x; sv[u][4 * e + 1] = x.y;
                sv[u][4 * e + 2] = x.z; sv[u][4 * e + 3] = x.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) sv[u][e] = 0.f;
            }
          }
        } else {
          tmem_ld16(tm + lane_q + TM_S + 64 * half + 32 * cp, sv[0]);
          tmem_ld16(tm + lane_q + TM_S + 64 * half + 32 * cp + 16, sv[1]);
          tmem_wait_ld();
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
        const int col = 64 * half + 32 * cp + 16 * u;
        float *v = sv[u];
        float lo[8], hi[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo[e] = v[e]; hi[e] = v[8 + e]; }
        *reinterpret_cast<uint4 *>(smem + OFF_SB + tl128(j, col / 8)) = pack8(lo);
        *reinterpret_cast<uint4 *>(smem + OFF_SB + tl128(j, col / 8 + 1)) = pack8(hi);
        float E[8];
        ld8f(EGC + col, E);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= E[e];
        ld8f(EGC + col + 8, E);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 + e] *= E[e];
        tmem_st16(tm + lane_q + TM_S + col, *reinterpret_cast<float(*)[16]>(v));
        }
      }
      tmem_wait_st();
    }
    mma_sync_point();
    PDN_PHASE_MARK(6);

    // ---- MMA6: O^T = S Qh^T  (runs under the solve) ----
    if (tid == 0) {
      const uint32_t id6 = make_idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + ot_col(n), make_sdesc(sb + OFF_SB + 256 * kk, 128, 2048),
                    make_sdesc(sb + OFF_RQ + 16384 + 256 * kk, 128, 2048), id6, kk > 0);
      mma_commit(bar_m6);
    }
    if (!wait_mma(bar_m1, n)) { aborted = true; break; }
    PDN_PHASE_MARK(7);

    // ---- solve: M, P from TMEM; T = (I + M)^{-1} ----
    {
      const int row = 32 * (warp & 3) + lane;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[16];
        tmem_ld16(tm + lane_q + TM_D1 + 32 * half + 16 * cc, v);
        tmem_wait_ld();
        const int s0 = 32 * half + 16 * cc;
        if (row < kC) {
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            float4 x;
            x.x = (s0 + 4 * e4 + 0 < row) ? v[4 * e4 + 0] : 0.f;
            x.y = (s0 + 4 * e4 + 1 < row) ? v[4 * e4 + 1] : 0.f;
            x.z = (s0 + 4 * e4 + 2 < row) ? v[4 * e4 + 2] : 0.f;
            x.w = (s0 + 4 * e4 + 3 < row) ? v[4 * e4 + 3] : 0.f;
            *reinterpret_cast<float4 *>(MS + row * MS_LD + s0 + 4 * e4) = x;
          }
        } else {
          const int t = row - kC;
          float lo[8], hi[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            lo[e] = (s0 + e <= t) ? v[e] : 0.f;
            hi[e] = (s0 + 8 + e <= t) ? v[8 + e] : 0.f;
          }
          *reinterpret_cast<uint4 *>(smem + OFF_PM + tl64(t, s0 / 8)) = pack8(lo);
          *reinterpret_cast<uint4 *>(smem + OFF_PM + tl64(t, s0 / 8 + 1)) = pack8(hi);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    PDN_PHASE_MARK(8);
    // L0: the four 16x16 diagonal blocks by forward substitution (one column
    // per thread); the other threads zero the upper off-diagonal blocks that
    // the merges below read.
    if (tid < 64) {
      const int base = 16 * (tid >> 4), c = tid & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc0 = (r == c) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
        for (int s = 0; s < r; s += 2) {
          acc0 = fmaf(-MS[(base + r) * MS_LD + base + s], x[s], acc0);
          if (s + 1 < r) acc1 = fmaf(-MS[(base + r) * MS_LD + base + s + 1], x[s + 1], acc1);
        }
        x[r] = acc0 + acc1;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) TS[(base + r) * TS_LD + base + c] = x[r];
    } else {
      // rows 0-15 x cols 16-31 and rows 32-47 x cols 48-63 (512 entries, 192 threads)
      for (int e = tid - 64; e < 512; e += kThreads - 64) {
        const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
        TS[(32 * blk + r) * TS_LD + 32 * blk + 16 + c] = 0.f;
      }
    }
    __syncthreads();
    PDN_PHASE_MARK(9);
    // L1: merge 16 -> 32 within rows/cols [32p, 32p+32): lower-left block
    //   X = -T_D (M_CA T_A), 2x2 outputs per thread (128 threads).
    if (tid < 128) {
      const int p = tid >> 6, rb = (tid >> 3) & 7, cb = tid & 7;
      const int o = 32 * p, r0 = 2 * rb, c0b = 2 * cb;
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll
      for (int s4 = 0; s4 < 16; s4 += 4) {
        const float4 m0 = *reinterpret_cast<const float4 *>(MS + (o + 16 + r0) * MS_LD + o + s4);
        const float4 m1 = *reinterpret_cast<const float4 *>(MS + (o + 16 + r0 + 1) * MS_LD + o + s4);
        const float mv0[4] = {m0.x, m0.y, m0.z, m0.w}, mv1[4] = {m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 tv = *reinterpret_cast<const float2 *>(TS + (o + s4 + k) * TS_LD + o + c0b);
          a00 = fmaf(mv0[k], tv.x, a00); a01 = fmaf(mv0[k], tv.y, a01);
          a10 = fmaf(mv1[k], tv.x, a10); a11 = fmaf(mv1[k], tv.y, a11);
        }
      }
      float *y = YS + p * 16 * YS_LD;
      *reinterpret_cast<float2 *>(y + r0 * YS_LD + c0b) = make_float2(a00, a01);
      *reinterpret_cast<float2 *>(y + (r0 + 1) * YS_LD + c0b) = make_float2(a10, a11);
    }
    __syncthreads();
    if (tid < 128) {
      const int p = tid >> 6, rb = (tid >> 3) & 7, cb = tid & 7;
      const int o = 32 * p, r0 = 2 * rb, c0b = 2 * cb;
      const float *y = YS + p * 16 * YS_LD;
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll
      for (int s4 = 0; s4 < 16; s4 += 4) {
        const float4 t0 = *reinterpret_cast<const float4 *>(TS + (o + 16 + r0) * TS_LD + o + 16 + s4);
        const float4 t1 = *reinterpret_cast<const float4 *>(TS + (o + 16 + r0 + 1) * TS_LD + o + 16 + s4);
        const float tv0[4] = {t0.x, t0.y, t0.z, t0.w}, tv1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 yv = *reinterpret_cast<const float2 *>(y + (s4 + k) * YS_LD + c0b);
          a00 = fmaf(tv0[k], yv.x, a00); a01 = fmaf(tv0[k], yv.y, a01);
          a10 = fmaf(tv1[k], yv.x, a10); a11 = fmaf(tv1[k], yv.y, a11);
        }
      }
      *reinterpret_cast<float2 *>(TS + (o + 16 + r0) * TS_LD + o + c0b) = make_float2(-a00, -a01);
      *reinterpret_cast<float2 *>(TS + (o + 16 + r0 + 1) * TS_LD + o + c0b) =
          make_float2(-a10, -a11);
    }
    __syncthreads();
    // L2: merge 32 -> 64: X = -T_D (M[32:64, 0:32] T_A), 2x2 outputs per thread.
    {
      const int r0 = 2 * (tid >> 4), c0b = 2 * (tid & 15);
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll 4
      for (int s4 = 0; s4 < 32; s4 += 4) {
        const float4 m0 = *reinterpret_cast<const float4 *>(MS + (32 + r0) * MS_LD + s4);
        const float4 m1 = *reinterpret_cast<const float4 *>(MS + (32 + r0 + 1) * MS_LD + s4);
        const float mv0[4] = {m0.x, m0.y, m0.z, m0.w}, mv1[4] = {m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 tv = *reinterpret_cast<const float2 *>(TS + (s4 + k) * TS_LD + c0b);
          a00 = fmaf(mv0[k], tv.x, a00); a01 = fmaf(mv0[k], tv.y, a01);
          a10 = fmaf(mv1[k], tv.x, a10); a11 = fmaf(mv1[k], tv.y, a11);
        }
      }
      *reinterpret_cast<float2 *>(YS + r0 * YS_LD + c0b) = make_float2(a00, a01);
      *reinterpret_cast<float2 *>(YS + (r0 + 1) * YS_LD + c0b) = make_float2(a10, a11);
    }
    __syncthreads();
    {
      const int r0 = 2 * (tid >> 4), c0b = 2 * (tid & 15);
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
#pragma unroll 4
      for (int s4 = 0; s4 < 32; s4 += 4) {
        const float4 t0 = *reinterpret_cast<const float4 *>(TS + (32 + r0) * TS_LD + 32 + s4);
        const float4 t1 = *reinterpret_cast<const float4 *>(TS + (32 + r0 + 1) * TS_LD + 32 + s4);
        const float tv0[4] = {t0.x, t0.y, t0.z, t0.w}, tv1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 yv = *reinterpret_cast<const float2 *>(YS + (s4 + k) * YS_LD + c0b);
          a00 = fmaf(tv0[k], yv.x, a00); a01 = fmaf(tv0[k], yv.y, a01);
          a10 = fmaf(tv1[k], yv.x, a10); a11 = fmaf(tv1[k], yv.y, a11);
        }
      }
      *reinterpret_cast<float2 *>(TS + (32 + r0) * TS_LD + c0b) = make_float2(-a00, -a01);
      *reinterpret_cast<float2 *>(TS + (32 + r0 + 1) * TS_LD + c0b) = make_float2(-a10, -a11);
    }
    __syncthreads();
    // T (lower triangle incl. diagonal) -> bf16 TL tile
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int t = 8 * warp + (lane & 7), s8 = 4 * m + (lane >> 3);
      float v[8];
      ld8f(TS + t * TS_LD + 8 * s8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = (8 * s8 + e <= t) ? v[e] : 0.f;
      *reinterpret_cast<uint4 *>(smem + OFF_TM + tl64(t, s8)) = pack8(v);
    }
    mma_sync_point();
    PDN_PHASE_MARK(10);

    // ---- MMA2: Y^T = Rh^T T^T ; MMA3: U^T = U^T T^T ----
    if (tid == 0) {
      const uint32_t id = make_idesc_bf16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = make_sdesc(sb + OFF_TM + 256 * kk, 128, 1024);
        mma_bf16_ss(tm + TM_YT, make_sdesc(sb + OFF_RQ + 4096 * kk, 2048, 128), bd, id, kk > 0);
      }
      mma_commit(bar_m2);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = make_sdesc(sb + OFF_TM + 256 * kk, 128, 1024);
        mma_bf16_ss(tm + TM_UD, make_sdesc(sb + OFF_U + 4096 * kk, 2048, 128), bd, id, kk > 0);
      }
      mma_commit(bar_m3);
    }
    if (!wait_mma(bar_m2, n)) { aborted = true; break; }
    PDN_PHASE_MARK(11);

    // ---- Y^T -> bf16 operand (rows d_k, columns tokens) ----
    {
      const int i = 32 * (warp & 3) + lane;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[16];
        tmem_ld16(tm + lane_q + TM_YT + 32 * half + 16 * cc, v);
        tmem_wait_ld();
        float lo[8], hi[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo[e] = v[e]; hi[e] = v[8 + e]; }
        const int t8 = 4 * half + 2 * cc;
        *reinterpret_cast<uint4 *>(smem + OFF_YT + tl64(i, t8)) = pack8(lo);
        *reinterpret_cast<uint4 *>(smem + OFF_YT + tl64(i, t8 + 1)) = pack8(hi);
      }
    }
    mma_sync_point();
    PDN_PHASE_MARK(12);

    // ---- MMA5: D^T = U^T - S Y^T (accumulates onto MMA3's U^T, issued after it) ----
    if (tid == 0) {
      const uint32_t id5 = make_idesc_bf16(128, 64, false, true, true);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TM_UD, make_sdesc(sb + OFF_SB + 256 * kk, 128, 2048),
                    make_sdesc(sb + OFF_YT + 2048 * kk, 1024, 128), id5, 1);
      mma_commit(bar_m5);
    }
    // the next chunk's v flies while MMA5 runs (MMA3 has finished reading U)
    if (!wait_mma(bar_m3, n)) { aborted = true; break; }
    if (Cn_next > 0) stage_rows(P, P.v, sb + OFF_U, true, b, h, c0 + kC, Cn_next, tid);
    if (!wait_mma(bar_m6, n)) { aborted = true; break; }
    if (!wait_mma(bar_m5, n)) { aborted = true; break; }
    PDN_PHASE_MARK(13);

    // SB is free until the next state epilogue: stage the next chunk's channel decay there
    if (kDecay == PDN_DECAY_CHANNEL && Cn_next > 0)
      stage_rows(P, P.log_alpha, sb + OFF_SB, false, b, h, c0 + kC, Cn_next, tid);

    // ---- D^T -> bf16 operand (rows d_v, columns tokens) ----
    {
      const int j = 32 * (warp & 3) + lane;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[16];
        tmem_ld16(tm + lane_q + TM_UD + 32 * half + 16 * cc, v);
        tmem_wait_ld();
        float lo[8], hi[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo[e] = v[e]; hi[e] = v[8 + e]; }
        const int t8 = 4 * half + 2 * cc;
        *reinterpret_cast<uint4 *>(smem + OFF_DT + tl64(j, t8)) = pack8(lo);
        *reinterpret_cast<uint4 *>(smem + OFF_DT + tl64(j, t8 + 1)) = pack8(hi);
      }
    }
    mma_sync_point();
    PDN_PHASE_MARK(14);

    // ---- MMA7: O^T += D^T P^T ; MMA8: S += D^T Wb ----
    if (tid == 0) {
      const uint32_t id7 = make_idesc_bf16(128, 64, false, false);
      const uint32_t id8 = make_idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = make_sdesc(sb + OFF_DT + 256 * kk, 128, 1024);
        mma_bf16_ss(tm + ot_col(n), ad, make_sdesc(sb + OFF_PM + 256 * kk, 128, 1024), id7, 1);
        mma_bf16_ss(tm + TM_S, ad, make_sdesc(sb + OFF_WB + 4096 * kk, 2048, 128), id8, 1);
      }
      mma_commit(bar_m7);
    }
    if (!wait_mma(bar_m7, n)) { aborted = true; break; }
    PDN_PHASE_MARK(15);
  }

  // ---- final: O of the last chunk, S_T, A_T ----
  if (!aborted && nchunks > 0) {
    const int j = 32 * (warp & 3) + lane;
    const int pc0 = (nchunks - 1) * kC;
    if (warp < 4) store_o_tile(P, tm + lane_q + ot_col(nchunks - 1), b, h, pc0, P.T - pc0, lane, warp);
    if (P.ST) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int col = 64 * half + 16 * cc;
        float v[16];
        tmem_ld16(tm + lane_q + TM_S + col, v);
        tmem_wait_ld();
        float4 *dst = reinterpret_cast<float4 *>(P.ST + ((size_t)bh * kD + j) * kD + col);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
      }
    }
    if (kPre && P.AT && tid < kD) P.AT[(size_t)bh * kD + tid] = Acar[tid];
  }
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, TM_COLS);
}

template <int V, int Dc>
cudaError_t launch_one(const KParams &P, cudaStream_t stream) {
  auto kern = chunk_tc_kernel<V, Dc>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(P.B * P.H), kThreads, SMEM_BYTES, stream>>>(P);
  return cudaGetLastError();
}

template <int V>
cudaError_t launch_decay(const KParams &P, cudaStream_t stream) {
  switch (P.decay) {
    case PDN_DECAY_NONE: return launch_one<V, PDN_DECAY_NONE>(P, stream);
    case PDN_DECAY_SCALAR: return launch_one<V, PDN_DECAY_SCALAR>(P, stream);
    default: return launch_one<V, PDN_DECAY_CHANNEL>(P, stream);
  }
}

}  // namespace

int tc_supported(const KParams &P) {
  return P.dtype == PDN_BF16 && P.dk == kD && P.dv == kD && P.chunk == kC && P.T > 0 &&
         (long long)P.B * P.H <= 0x7fffffffLL;
}

size_t tc_workspace_bytes(const KParams &) { return 0; }

cudaError_t launch_chunk_tc(const KParams &P, void *, cudaStream_t stream) {
  switch (P.variant) {
    case PDN_VAR_DN: return launch_decay<PDN_VAR_DN>(P, stream);
    case PDN_VAR_GDN: return launch_decay<PDN_VAR_GDN>(P, stream);
    case PDN_VAR_KDA: return launch_decay<PDN_VAR_KDA>(P, stream);
    case PDN_VAR_PDN: return launch_decay<PDN_VAR_PDN>(P, stream);
    case PDN_VAR_PGDN: return launch_decay<PDN_VAR_PGDN>(P, stream);
    case PDN_VAR_PKDA: return launch_decay<PDN_VAR_PKDA>(P, stream);
    case PDN_VAR_FG2_GDN: return launch_decay<PDN_VAR_FG2_GDN>(P, stream);
    default: return launch_decay<PDN_VAR_GDN2>(P, stream);
  }
}

}  // namespace pdn
