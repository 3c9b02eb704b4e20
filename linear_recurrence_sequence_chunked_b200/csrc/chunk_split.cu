// chunk_split.cu -- chunked forward in three kernels: the intra-chunk work,
// which does not depend on the state, runs for every chunk at once; only the
// state pass stays sequential per (batch, head).
//
//   K0  key-energy prefix: A at the start of every chunk (preconditioned
//       variants; "Preconditioned DeltaNet", fr §2.B: A_t = A_{t-1} + k.k)
//   K1  persistent over the (chunk, batch, head) blocks (two CTAs per SM,
//       one for channel decay): gates and preconditioner, M and P (MMA),
//       T = (I + M)^{-1}, Y^T = R^T T^T (MMA); writes the chunk's bf16
//       operand tiles to the workspace, straight from registers, in the
//       shared-memory image the state kernel's MMAs consume
//   K2  one CTA per (batch, head): per chunk, bulk-loads those tiles ahead,
//       U^T = U^T T^T, D^T = U^T - S Y^T, O^T = S Qh^T + D^T P^T,
//       S <- S Diag(e^{G_C}) + D^T Wb; fp32 state in tensor memory
//
// The chunk algebra is the chunkwise WY/UT form ("Gated DeltaNet-2", ja §3:
// decay absorbed into the erase/write matrices, (I+T)^{-1} solve for the
// auxiliaries Y and U). Splitting it trades extra HBM traffic (about 80 KiB of
// operand tiles per chunk and head, written once and read once) for running
// the intra-chunk work with thousands of CTAs instead of one per chain.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tiles.cuh"

namespace pdn {
namespace {

constexpr int kC = 64;
constexpr int kD = 128;

// ---- workspace: one block per (batch, head, chunk) -------------------------
constexpr uint32_t WS_Q = 0;        // TL 64 x 128: Qh (rows tokens)
constexpr uint32_t WS_Y = 16384;    // TL 128 x 64: Y^T (rows d_k, columns tokens)
constexpr uint32_t WS_U = 32768;    // TL 64 x 128: u (rows tokens)
constexpr uint32_t WS_WB = 49152;   // TL 64 x 128: Wb (rows tokens)
constexpr uint32_t WS_T = 65536;    // TL 64 x 64: T = (I + M)^{-1}
constexpr uint32_t WS_P = 73728;    // TL 64 x 64: P
constexpr uint32_t WS_E = 81920;    // float[128]: e^{G_C}
constexpr uint32_t WS_SET = 82432;  // bytes the state kernel loads per chunk
constexpr uint32_t WS_A = 82432;    // float[128]: accumulator A at the chunk start
constexpr size_t WS_CH = 82944;     // bytes per block (256-aligned)

// Chunk-major: the blocks of one chunk index, over all (batch, head), are
// adjacent, so the state pass's concurrent loads stream one contiguous range.
// A chunk index as the kernels use it; the debug build checks it against the
// problem's chunk count (recording PDN_ERR_BOUNDS and taking chunk 0, so
// that no copy another warp waits for is skipped).
__device__ __forceinline__ int chunk_ok(const KParams &P, int c) {
  return in_bounds(P.err, c >= 0 && c < (P.T + kC - 1) / kC) ? c : 0;
}

__device__ __forceinline__ uint8_t *ws_block(void *ws, int bh, int BH, int c) {
  return reinterpret_cast<uint8_t *>(ws) + ((size_t)c * BH + bh) * WS_CH;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ===========================================================================
// K0: per-chunk key energy, then the exclusive prefix over chunks
// ===========================================================================
// One CTA per (batch, head, chunk): thread (8-channel group, token lane)
// loads 16-byte rows and squares them; the 16 token lanes are summed in
// shared memory.
__global__ void __launch_bounds__(256) k0_chunk_energy(const KParams P, void *ws, int N) {
  __shared__ float part[16][kD + 4];
  const int tid = threadIdx.x, c8 = tid & 15, tl = tid >> 4;
  const int BH = P.B * P.H;
  const long long total = (long long)N * BH;
  // chunk blocks in the workspace's chunk-major order; one per CTA up to the
  // grid cap, so each CTA keeps only one block's rows in flight and more
  // CTAs fit per SM
  for (long long it = blockIdx.x; it < total; it += gridDim.x) {
  const int c = (int)(it / BH), bh = (int)(it % BH);
  const int c0 = c * kC, Cn = min(kC, P.T - c0);
  const size_t tstride = (size_t)P.H * kD;
  const __nv_bfloat16 *kp = reinterpret_cast<const __nv_bfloat16 *>(P.k) +
                            tok_index(P, bh / P.H, c0, bh % P.H) * kD + c8 * 8;
  // thread (c8, tl): 8 channels of tokens tl, tl + 16, tl + 32, tl + 48
  uint4 r[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int t = tl + 16 * m;
    r[m] = t < Cn ? __ldg(reinterpret_cast<const uint4 *>(kp + t * tstride)) : make_uint4(0u, 0u, 0u, 0u);
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float kf[8];
    unpack8(r[m], kf);
    if (P.prologue & PDN_PRO_L2NORM_QK) {
      // the token's 128 channels sit in the 16 lanes of this half-warp
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(kf[e], kf[e], ss);
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = inv_norm(ss);
#pragma unroll
      for (int e = 0; e < 8; ++e) kf[e] *= inv;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(kf[e], kf[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[tl][c8 * 8 + e] = acc[e];
  __syncthreads();
  if (tid < kD) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) sum += part[q][tid];
    reinterpret_cast<float *>(ws_block(ws, bh, BH, c) + WS_A)[tid] = sum;
  }
  __syncthreads();  // part is rewritten by the next block
  }
}

// A at every chunk start: per (batch, head), an exclusive prefix over the
// chunk sums, seeded with A0. Four groups of 128 threads take a quarter of the
// chunks each: their totals first, then the prefixes.
constexpr int kK0Groups = 4;
__global__ void __launch_bounds__(kD * kK0Groups) k0_prefix(const KParams P, void *ws, int N) {
  __shared__ float tot[kK0Groups][kD];
  const int bh = blockIdx.x, i = threadIdx.x & (kD - 1), g = threadIdx.x / kD;
  const int BH = P.B * P.H;
  const int L = (N + kK0Groups - 1) / kK0Groups;
  const int c_begin = min(N, g * L), c_end = min(N, c_begin + L);
  float t = 0.f;
  for (int c0 = c_begin; c0 < c_end; c0 += 8) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = (c0 + e < c_end) ? reinterpret_cast<const float *>(ws_block(ws, bh, BH, c0 + e) + WS_A)[i]
                              : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) t += v[e];
  }
  tot[g][i] = t;
  __syncthreads();
  float a = P.A0 ? P.A0[(size_t)bh * kD + i] : 0.f;
  for (int g2 = 0; g2 < g; ++g2) a += tot[g2][i];
  for (int c0 = c_begin; c0 < c_end; c0 += 8) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = (c0 + e < c_end) ? reinterpret_cast<const float *>(ws_block(ws, bh, BH, c0 + e) + WS_A)[i]
                              : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (c0 + e < c_end) reinterpret_cast<float *>(ws_block(ws, bh, BH, c0 + e) + WS_A)[i] = a;
      a += v[e];
    }
  }
  if (g == kK0Groups - 1 && P.AT) P.AT[(size_t)bh * kD + i] = a;
}

// ===========================================================================
// K1: intra-chunk work, persistent over the (chunk, batch, head) blocks
// ===========================================================================
constexpr int kK1Threads = 256;
constexpr int LB_LD = 132;                        // floats per row of the fp32 prep buffer
constexpr int MS_LD = 68, TS_LD = 68, YS_LD = 34; // fp32 solve scratch strides
constexpr uint32_t KS_LD = 272;                   // staged row stride (bytes), padded

// In-chunk decay without range limits. G_t is the cumulative log decay from
// the chunk start (inclusive); every product the chunk form needs is
// e^{G_t - G_s} with s <= t, at most 1, but its two factors e^{G_t} and
// e^{-G_s} leave the fp32 range once a channel decays by more than e^{-87}
// inside the chunk. So:
//   * scalar decay: MMA1 multiplies the undecayed operands and the epilogue
//     applies e^{G_t - G_s} per element;
//   * channel decay: the chunk is cut into four 16-token sub-chunks with
//     boundary values B_a = G_{16a-1} (B_0 = 0). Row t of sub-chunk a is
//     scaled by rho_t = e^{G_t - B_a} <= 1 and its columns s by
//     e^{B_a - G_s}, which is <= 1 for s in an earlier sub-chunk and at most
//     e^{kSubRange} inside sub-chunk a unless that sub-chunk is flagged; a
//     flagged sub-chunk's diagonal block is summed pairwise instead. MMA1's
//     B operand holds one column group per sub-chunk a (the columns
//     s < 16(a+1), scaled for reference B_a), starting at column grp_off(a).
// The state-side factors e^{G_t}, e^{G_C - G_s} and e^{G_C} are at most 1
// and are formed directly. A log decay below kMinLogAlpha per token is
// raised to it: e^{-100} is below the smallest normal fp32 number, so every
// factor such a token enters is zero in fp32 either way.
constexpr float kSubRange = 64.f;
constexpr float kMinLogAlpha = -100.f;
__host__ __device__ constexpr int grp_off(int a) { return 8 * a * (a + 1); }

template <int kVariant, int kDecay>
struct K1Layout {
  static constexpr bool kPre = kVariant == PDN_VAR_PDN || kVariant == PDN_VAR_PGDN ||
                               kVariant == PDN_VAR_PKDA || kVariant == PDN_VAR_PLA;
  static constexpr bool kCh = kDecay == PDN_DECAY_CHANNEL;
  static constexpr int kN1 = kCh ? 160 : 64;                // columns of MMA1
  static constexpr uint32_t kRQ = 0;                        // TL 128 x 128: R rows 0-63, Q rows 64-127
  static constexpr uint32_t kWH = 32768;                    // TL kN1 x 128: MMA1's B operand
  static constexpr uint32_t kRA = kWH + kN1 * 256;          // region A
  // region A during the prep: staged k and q, the bf16 preconditioner
  // coefficients, the fp32 cumulative log decay and the staged channel log
  // decay (channel decay)
  static constexpr uint32_t kKS = kRA;
  static constexpr uint32_t kQS = kKS + 64 * KS_LD;
  static constexpr uint32_t kBC = kQS + 64 * KS_LD;
  static constexpr uint32_t kGBUF = kBC + 64 * KS_LD;
  static constexpr uint32_t kLasStage = kGBUF + 64 * LB_LD * 4;
  // channel decay: FG2's gain vector, GDN-2's erase and write gates, or
  // FG2+'s key-side and value-side gains, staged by cp.async with q (read in P3)
  static constexpr int kGates = !kCh ? 0
                                : kVariant == PDN_VAR_FG2_GDN ? 1
                                : (kVariant == PDN_VAR_GDN2 || kVariant == PDN_VAR_FG2_GDN_PLUS) ? 2 : 0;
  static constexpr uint32_t kGateStage = kLasStage + 64 * 256;
  static constexpr uint32_t kPrepEnd = kCh ? kGateStage + kGates * 16384 : kGBUF;
  // region A from the epilogue of MMA1 on: MMA2's T tile and the fp32 solve
  // scratch
  static constexpr uint32_t kTM = kRA;                      // TL 64 x 64
  static constexpr uint32_t kMS = kRA + 16384;              // fp32 [64][68]
  static constexpr uint32_t kTS = kMS + 64 * MS_LD * 4;     // fp32 [64][68]
  static constexpr uint32_t kYS = kTS + 64 * TS_LD * 4;     // fp32 [32][34]
  static constexpr uint32_t kSolveEnd = kYS + 32 * YS_LD * 4;
  static constexpr uint32_t kSmall = (kPrepEnd > kSolveEnd ? kPrepEnd : kSolveEnd);
  static constexpr uint32_t kAcar = kSmall, kGC = kSmall + 512;
  // float[3][128]: sums over token quarters 0..2 of k.k and of the log decay
  static constexpr uint32_t kPartK = kSmall + 1536, kPartG = kSmall + 3072;
  static constexpr uint32_t kMup = kSmall + 4608;  // float[2][64] per channel-half partial means
  static constexpr uint32_t kMu = kSmall + 5120, kBeta = kSmall + 5376, kGS = kSmall + 5632;
  static constexpr uint32_t kLas = kSmall + 5888;
  static constexpr uint32_t kEGS = kSmall + 6144;  // float[64] e^{G_t}, scalar decay
  // channel decay, float[13][128]: e^{B_1}, e^{B_2}, e^{B_3}, e^{B_2 - B_1},
  // e^{B_3 - B_1}, e^{B_3 - B_2}, e^{G_C - B_1}, e^{G_C - B_2}, e^{G_C - B_3},
  // then e^{B_a - B_{a+1}} for a = 0..3 (B_4 = G_C; read only for sub-chunks
  // that are not flagged, where it is at most e^{kSubRange})
  static constexpr uint32_t kTab = kSmall + 6400;
  static constexpr uint32_t kFlags = kTab + (kCh ? 13 * 512 : 0);  // bit a: sub-chunk a flagged
  static constexpr uint32_t kBar = kFlags + 16;
  static constexpr uint32_t kTbase = kBar + 16;
  static constexpr uint32_t kBytes = kTbase + 16;
  static constexpr uint32_t kTmemCols = kCh ? 256 : 128;
  static constexpr uint32_t kTmY = kN1;  // TMEM column of Y^T (after MMA1's columns)
};
static_assert(K1Layout<PDN_VAR_GDN2, PDN_DECAY_CHANNEL>::kBytes <= 232448 &&
                  K1Layout<PDN_VAR_FG2_GDN_PLUS, PDN_DECAY_CHANNEL>::kBytes <= 232448 &&
                  K1Layout<PDN_VAR_PKDA, PDN_DECAY_CHANNEL>::kBytes <= 232448 &&
                  K1Layout<PDN_VAR_FG2_GDN, PDN_DECAY_CHANNEL>::kBytes <= 232448,
              "intra-chunk kernel shared memory budget");
static_assert(2 * (K1Layout<PDN_VAR_PGDN, PDN_DECAY_SCALAR>::kBytes + 1024) <= 233472,
              "two intra-chunk CTAs per SM for scalar decay");

// sqrt of a gain in [0, 1] as x * x^(-1/2) (rsqrtf, a couple of ulp): short
// straight-line code for the per-element gains of FG2-GDN(+); 0 stays 0.
__device__ __forceinline__ float sqrt_gain(float x) { return x > 0.f ? x * rsqrtf(x) : 0.f; }

__device__ __forceinline__ void sync_for_mma() {
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// Exact diagonal-block entries of row t against columns s0 .. s0 + 15 of a
// flagged sub-chunk: sum_c x_tc w_sc e^{G_tc - G_sc} for s <= t (s < t when
// `strict`), from the undecayed bf16 rows x (row t) and w (rows s) and the
// fp32 cumulative log decay. Out of line: only flagged sub-chunks (very
// strong decay) take it, and inlined copies would sit in the hot epilogue.
__device__ __noinline__ void diag_exact(const uint8_t *xrow, const uint8_t *wbase,
                                           const float *gbuf, int t, int s0, bool strict,
                                           float (&out)[16]) {
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  const float *gt = gbuf + t * LB_LD;
  for (int c8 = 0; c8 < 16; ++c8) {
    float xf[8], gtv[8];
    unpack8(*reinterpret_cast<const uint4 *>(xrow + 16 * c8), xf);
    ld8f(gt + 8 * c8, gtv);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int s = s0 + e;
      if (s <= t) {
        float wf[8], gs[8];
        unpack8(*reinterpret_cast<const uint4 *>(wbase + s * KS_LD + 16 * c8), wf);
        ld8f(gbuf + s * LB_LD + 8 * c8, gs);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          acc[e] = fmaf(xf[k] * wf[k], ex2_approx((gtv[k] - gs[k]) * kLog2e), acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int s = s0 + e;
    out[e] = (s < t || (!strict && s == t)) ? acc[e] : 0.f;
  }
}

template <int kVariant, int kDecay>
__global__ void __launch_bounds__(kK1Threads, kDecay == PDN_DECAY_CHANNEL ? 1 : 2) k1_intra(const KParams P, void *ws, int N,
                                                                         int it_begin, int it_end) {
  using L = K1Layout<kVariant, kDecay>;
  constexpr bool kPre = L::kPre;
  constexpr bool kCh = L::kCh;
  constexpr bool kSc = kDecay == PDN_DECAY_SCALAR;
  constexpr bool kScalarBeta = has_scalar_beta(kVariant);
  constexpr bool kFG2 = kVariant == PDN_VAR_FG2_GDN || kVariant == PDN_VAR_FG2_GDN_PLUS;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  float *Acar = reinterpret_cast<float *>(smem + L::kAcar);
  float *GC = reinterpret_cast<float *>(smem + L::kGC);
  float *PARTK = reinterpret_cast<float *>(smem + L::kPartK);
  float *PARTG = reinterpret_cast<float *>(smem + L::kPartG);
  float *MUP = reinterpret_cast<float *>(smem + L::kMup);
  float *MU = reinterpret_cast<float *>(smem + L::kMu);
  float *BETA = reinterpret_cast<float *>(smem + L::kBeta);
  float *GS = reinterpret_cast<float *>(smem + L::kGS);
  float *LAS = reinterpret_cast<float *>(smem + L::kLas);
  float *EGS = reinterpret_cast<float *>(smem + L::kEGS);
  float *TAB = reinterpret_cast<float *>(smem + L::kTab);
  uint32_t *flags = reinterpret_cast<uint32_t *>(smem + L::kFlags);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L::kBar);
  uint32_t *tbase_p = reinterpret_cast<uint32_t *>(smem + L::kTbase);
  float *GBUF = reinterpret_cast<float *>(smem + L::kGBUF);
  float *MS = reinterpret_cast<float *>(smem + L::kMS);
  float *TS = reinterpret_cast<float *>(smem + L::kTS);
  float *YS = reinterpret_cast<float *>(smem + L::kYS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t tstride = (size_t)P.H * kD;
  const float log2x = P.lnx * kLog2e;
  const uint32_t lane_q = (uint32_t)(32 * (warp & 3)) << 16;
  const int half = warp >> 2;
  const int BH = P.B * P.H;
  // chunk blocks, chunk-major: block index = c * BH + bh; this launch takes
  // blocks it_begin .. it_end - 1 (a range of whole chunks)
  const int total = it_end;
  const int first = it_begin + (int)blockIdx.x;

  if (warp == 0) {
    tmem_alloc(tbase_p, L::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar + 0, 1);
    mbar_init(bar + 1, 1);
    fence_mbarrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tbase_p;

  // Per-token and per-channel scalars of a chunk block, loaded one block
  // ahead into registers. k and q are staged by cp.async at the start of the
  // block; v one block ahead through shared memory (see stage_v).
  struct Raw {
    float beta, las, acar;
  };
  auto load_raw = [&](int it) {
    Raw r;
    const int c_ = it / BH, bh_ = it % BH;
    const int b_ = bh_ / P.H, h_ = bh_ % P.H;
    const int c0_ = c_ * kC, Cn_ = min(kC, P.T - c0_);
    r.beta = 0.f;
    r.las = 0.f;
    if (tid < kC && tid < Cn_) {
      const size_t e = tok_index(P, b_, c0_ + tid, h_);
      if (kScalarBeta) r.beta = gate_act(P.prologue, __ldg(reinterpret_cast<const float *>(P.beta) + e));
      if (kSc)
        r.las = fmaxf(decay_act(P.prologue, P.decay_scale,
                                __ldg(reinterpret_cast<const float *>(P.log_alpha) + e)),
                      kMinLogAlpha);
    }
    r.acar = (kPre && tid < kD) ? reinterpret_cast<const float *>(ws_block(ws, bh_, P.B * P.H, c_) + WS_A)[tid] : 0.f;
    return r;
  };
  // v of a chunk block into the first 16 KiB of the B-operand space, rows of
  // 256 bytes with the 16-byte groups XOR-swizzled by (token & 7); issued
  // while the previous block is in its solve (the B operand is dead once
  // MMA1 has completed).
  auto stage_v = [&](int it) {
    const int c_ = it / BH, bh_ = it % BH;
    const int b_ = bh_ / P.H, h_ = bh_ % P.H;
    const int c0_ = c_ * kC, Cn_ = min(kC, P.T - c0_);
    const size_t tok0_ = tok_index(P, b_, c0_, h_) * kD;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
      const bool ok = t < Cn_;
      const size_t e = ok ? tok0_ + (size_t)t * tstride + c8 * 8 : 0;
      // (transition mode: no targets; the zero fill reads nothing from k)
      const bool use_v = !P.transition && P.v;
      cp_async16(sb + L::kWH + t * 256 + ((c8 ^ (t & 7)) << 4),
                 reinterpret_cast<const __nv_bfloat16 *>(use_v ? P.v : P.k) + e, ok && use_v);
    }
    cp_async_commit();
  };
  // k of a chunk block, rows of 256 bytes swizzled like v: channel decay into
  // rows 64.. of the B operand (dead once MMA1 has completed, and its 40 KiB
  // leave room after v), issued right after MMA1; otherwise into the R half
  // of the [R; Q] tile's space, issued once MMA2 of the previous block has
  // read R.
  constexpr uint32_t kKStage = kCh ? L::kWH + 16384 : L::kRQ;
  auto stage_k = [&](int it) {
    const int c_ = it / BH, bh_ = it % BH;
    const int b_ = bh_ / P.H, h_ = bh_ % P.H;
    const int c0_ = c_ * kC, Cn_ = min(kC, P.T - c0_);
    const size_t tok0_ = tok_index(P, b_, c0_, h_) * kD;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
      const bool ok = t < Cn_;
      const size_t e = ok ? tok0_ + (size_t)t * tstride + c8 * 8 : 0;
      cp_async16(sb + kKStage + t * 256 + ((c8 ^ (t & 7)) << 4),
                 reinterpret_cast<const __nv_bfloat16 *>(P.k) + e, ok);
    }
    cp_async_commit();
  };
  Raw pf = load_raw(first < total ? first : 0);
  if (first < total) {
    stage_v(first);
    stage_k(first);
  }

  int iter = 0;
  for (int it = first; it < total; it += gridDim.x, ++iter) {
  const int c = it / BH, bh = it % BH;
  const int b = bh / P.H, h = bh % P.H;
  const int c0 = c * kC, Cn = min(kC, P.T - c0);
  const size_t tok0 = tok_index(P, b, c0, h) * kD;  // element offset of token c0
  uint8_t *blk = ws_block(ws, bh, P.B * P.H, chunk_ok(P, c));
  const uint32_t par = (uint32_t)(iter & 1);  // mbarrier parity of this block's MMAs

  // ---- P0: k (staged a block ahead) into its padded rows; q (and the
  // channel log decay) by cp.async, q awaited only before P3; the prefetched
  // scalars into shared memory; then start loading the next block's ----
  uint4 vcur[4];
  cp_async_wait_all();  // this block's k and v
  __syncthreads();
  {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
      uint4 kr = *reinterpret_cast<const uint4 *>(smem + kKStage + t * 256 + ((c8 ^ (t & 7)) << 4));
      if (P.prologue & PDN_PRO_L2NORM_QK) {
        // the token's 128 channels sit in the 16 lanes of this half-warp
        float kf[8], ss = 0.f;
        unpack8(kr, kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(kf[e], kf[e], ss);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = inv_norm(ss);
#pragma unroll
        for (int e = 0; e < 8; ++e) kf[e] *= inv;
        kr = pack8(kf);
      }
      *reinterpret_cast<uint4 *>(smem + L::kKS + t * KS_LD + c8 * 16) = kr;
      if (kCh) {
        const bool ok = t < Cn;
        const size_t e = ok ? tok0 + (size_t)t * tstride + c8 * 8 : 0;
        cp_async16(sb + L::kLasStage + t * 256 + c8 * 16,
                   reinterpret_cast<const __nv_bfloat16 *>(P.log_alpha) + e, ok);
      }
    }
    cp_async_commit();  // group: channel log decay (P1)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = (tid >> 4) + 16 * m, c8 = tid & 15;
      const bool ok = t < Cn;
      const size_t e = ok ? tok0 + (size_t)t * tstride + c8 * 8 : 0;
      cp_async16(sb + L::kQS + t * KS_LD + c8 * 16, reinterpret_cast<const __nv_bfloat16 *>(P.q) + e, ok);
      // gates, rows of 256 bytes with the 16-byte groups swizzled by (token & 7)
      const uint32_t gs = sb + L::kGateStage + t * 256 + ((c8 ^ (t & 7)) << 4);
      if (L::kGates >= 1)
        cp_async16(gs, reinterpret_cast<const __nv_bfloat16 *>(
                           kFG2 ? P.beta : P.erase) + e, ok);
      if (L::kGates == 2)
        cp_async16(gs + 16384, reinterpret_cast<const __nv_bfloat16 *>(P.write) + e, ok);
    }
    cp_async_commit();  // group: q and the gates (P3)
    if (tid < kC) {
      BETA[tid] = pf.beta;
      LAS[tid] = pf.las;
    }
    if (tid < kD) Acar[tid] = pf.acar;
    if (kCh && tid == 0) *flags = 0u;
  }
  if (it + (int)gridDim.x < total) pf = load_raw(it + gridDim.x);
  if (kCh) cp_async_wait_group<1>();  // P1 scans the channel log decay
  __syncthreads();

  // ---- P1: per-channel scans; thread = (channel pair, quarter of the chunk) ----
  // Prefix sums of k.k (accumulator) and of the log decay over the chunk's
  // tokens, then (preconditioned variants) the per-token channel mean of
  // log2(A + eps) by a warp transpose-reduce, and B = x^(-s) per element.
  {
    const int p = tid & 63, q4 = tid >> 6, t0 = 16 * q4;  // channels 2p, 2p + 1; tokens t0 ..
    const int i0 = 2 * p;
    float k0[16], k1[16], l0[16], l1[16];
    float ks0 = 0.f, ks1 = 0.f, gs0 = 0.f, gs1 = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int t = t0 + e;
      if (kPre) {
        const float2 kv = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162 *>(smem + L::kKS + t * KS_LD + i0 * 2));
        k0[e] = kv.x;
        k1[e] = kv.y;
      } else {
        k0[e] = 0.f;
        k1[e] = 0.f;
      }
      if (kCh) {
        const float2 lv = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162 *>(smem + L::kLasStage + t * 256 + i0 * 2));
        // (past the sequence end the staged zeros stay zero: no decay)
        const bool in_seq = t < Cn;
        l0[e] = in_seq ? fmaxf(decay_act(P.prologue, P.decay_scale, lv.x), kMinLogAlpha) : 0.f;
        l1[e] = in_seq ? fmaxf(decay_act(P.prologue, P.decay_scale, lv.y), kMinLogAlpha) : 0.f;
      } else if (kSc) {
        l0[e] = LAS[t];
        l1[e] = l0[e];
      } else {
        l0[e] = 0.f;
        l1[e] = 0.f;
      }
      ks0 = fmaf(k0[e], k0[e], ks0);
      ks1 = fmaf(k1[e], k1[e], ks1);
      gs0 += l0[e];
      gs1 += l1[e];
    }
    if (q4 < 3) {
      *reinterpret_cast<float2 *>(PARTK + q4 * kD + i0) = make_float2(ks0, ks1);
      *reinterpret_cast<float2 *>(PARTG + q4 * kD + i0) = make_float2(gs0, gs1);
    }
    __syncthreads();
    float a0 = Acar[i0], a1 = Acar[i0 + 1], g0 = 0.f, g1 = 0.f;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      if (r < q4) {
        const float2 pk = *reinterpret_cast<const float2 *>(PARTK + r * kD + i0);
        const float2 pg = *reinterpret_cast<const float2 *>(PARTG + r * kD + i0);
        a0 += pk.x;
        a1 += pk.y;
        g0 += pg.x;
        g1 += pg.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int t = t0 + e;
      a0 = fmaf(k0[e], k0[e], a0);
      a1 = fmaf(k1[e], k1[e], a1);
      if (kPre) {  // k0, k1 now hold log2(A_t + eps)
        k0[e] = lg2_approx(a0 + P.eps);
        k1[e] = lg2_approx(a1 + P.eps);
      }
      g0 += l0[e];
      g1 += l1[e];
      if (kCh)
        *reinterpret_cast<float2 *>(GBUF + t * LB_LD + i0) = make_float2(g0, g1);
      else if (kSc && p == 0)
        GS[t] = g0;
    }
    if (q4 == 3) {
      GC[i0] = g0;
      GC[i0 + 1] = g1;
      const float e0 = ex2_approx(g0 * kLog2e);
      const float e1 = ex2_approx(g1 * kLog2e);
      *reinterpret_cast<float2 *>(reinterpret_cast<float *>(blk + WS_E) + i0) = make_float2(e0, e1);
    }
    if (kPre) {
      // transpose-reduce over the warp's 64 channels: four butterfly steps
      // leave lanes l and l ^ 1 with halves of the sum for token t0 + (l >> 1)
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = k0[e] + k1[e];
#pragma unroll
      for (int off = 16, len = 8; off >= 2; off >>= 1, len >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int e = 0; e < len; ++e) {
          const float send = upper ? v[e] : v[e + len];
          const float keep = upper ? v[e + len] : v[e];
          v[e] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
      if ((lane & 1) == 0) MUP[(warp & 1) * 64 + t0 + (lane >> 1)] = v[0];
      __syncthreads();
      if (tid < kC) MU[tid] = (MUP[tid] + MUP[64 + tid]) * (1.f / kD);
      __syncthreads();
      const float log2x_ = log2x;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int t = t0 + e;
        const float mu = MU[t];
        const float c0 = (k0[e] - mu) * kLn2, c1 = (k1[e] - mu) * kLn2;
        const float s0 = c0 * rcp_approx(1.f + fabsf(c0));
        const float s1 = c1 * rcp_approx(1.f + fabsf(c1));
        *reinterpret_cast<uint32_t *>(smem + L::kBC + t * KS_LD + i0 * 2) =
            pack_bf16(ex2_approx(-s0 * log2x_), ex2_approx(-s1 * log2x_));
      }
    }
  }
  // this block's v into registers (operand mapping) before P3 overwrites the
  // staging space with the B operand; q has landed
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int t = 8 * warp + (lane & 7), c8 = 4 * m + (lane >> 3);
    vcur[m] = *reinterpret_cast<const uint4 *>(smem + L::kWH + t * 256 + ((c8 ^ (t & 7)) << 4));
  }
  cp_async_wait_all();
  __syncthreads();
  if (kCh) {
    // per-channel factors between the sub-chunk boundaries, and the flags of
    // sub-chunks whose decay range exceeds kSubRange in some channel
    if (tid < kD) {
      const float B1 = GBUF[15 * LB_LD + tid], B2 = GBUF[31 * LB_LD + tid];
      const float B3 = GBUF[47 * LB_LD + tid], Gc = GBUF[63 * LB_LD + tid];
      TAB[0 * kD + tid] = ex2_approx(B1 * kLog2e);
      TAB[1 * kD + tid] = ex2_approx(B2 * kLog2e);
      TAB[2 * kD + tid] = ex2_approx(B3 * kLog2e);
      TAB[3 * kD + tid] = ex2_approx((B2 - B1) * kLog2e);
      TAB[4 * kD + tid] = ex2_approx((B3 - B1) * kLog2e);
      TAB[5 * kD + tid] = ex2_approx((B3 - B2) * kLog2e);
      TAB[6 * kD + tid] = ex2_approx((Gc - B1) * kLog2e);
      TAB[7 * kD + tid] = ex2_approx((Gc - B2) * kLog2e);
      TAB[8 * kD + tid] = ex2_approx((Gc - B3) * kLog2e);
      TAB[9 * kD + tid] = ex2_approx(-B1 * kLog2e);
      TAB[10 * kD + tid] = ex2_approx((B1 - B2) * kLog2e);
      TAB[11 * kD + tid] = ex2_approx((B2 - B3) * kLog2e);
      TAB[12 * kD + tid] = ex2_approx((B3 - Gc) * kLog2e);
      uint32_t m = 0;
      if (-B1 > kSubRange) m |= 1u;
      if (B1 - B2 > kSubRange) m |= 2u;
      if (B2 - B3 > kSubRange) m |= 4u;
      if (B3 - Gc > kSubRange) m |= 8u;
      m = __reduce_or_sync(0xffffffffu, m);
      if (lane == 0 && m) atomicOr(flags, m);
    }
    __syncthreads();
  }
  const uint32_t badm = kCh ? *flags : 0u;

  // ---- P3: operand tiles, (token, 8-channel) units ----
  {
    const int t = 8 * warp + (lane & 7);
    const bool ok = t < Cn;
    const size_t etok = tok0 + (size_t)t * tstride;
    const int a = t >> 4;  // sub-chunk of the token (channel decay)
    float eg_s = 1.f, ewb_s = 1.f;
    if (kSc) {
      eg_s = ex2_approx(GS[t] * kLog2e);
      ewb_s = ex2_approx((GC[0] - GS[t]) * kLog2e);
      if ((lane >> 3) == 0) EGS[t] = eg_s;
    }
    const float be = kScalarBeta ? BETA[t] : 0.f;
    float qs = P.q_scale;
    if (P.prologue & PDN_PRO_L2NORM_QK) {
      // this token's 128 query channels: 32 here, the rest in lanes ^8, ^16, ^24
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float qf[8];
        unpack8(*reinterpret_cast<const uint4 *>(smem + L::kQS + t * KS_LD + (4 * m + (lane >> 3)) * 16), qf);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(qf[e], qf[e], ss);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 8);
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      qs *= inv_norm(ss);
    }
    // channel decay: one copy of the (long) body, not four, so that the
    // kernel's straight-line code stays within the instruction cache
#pragma unroll(kCh ? 1 : 4)
    for (int m = 0; m < 4; ++m) {
      const int c8 = 4 * m + (lane >> 3);
      const int i0 = 8 * c8;
      float kf[8], qf[8], vf[8], r[8], w[8];
      unpack8(*reinterpret_cast<const uint4 *>(smem + L::kKS + t * KS_LD + c8 * 16), kf);
      unpack8(*reinterpret_cast<const uint4 *>(smem + L::kQS + t * KS_LD + c8 * 16), qf);
      unpack8(m == 0 ? vcur[0] : m == 1 ? vcur[1] : m == 2 ? vcur[2] : vcur[3], vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[e] *= qs;
      if (kPre) {
        float Bv[8];
        unpack8(*reinterpret_cast<const uint4 *>(smem + L::kBC + t * KS_LD + c8 * 16), Bv);
        if (kVariant == PDN_VAR_PLA) {
          // linear attention: no erase; the preconditioner acts on the query
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            r[e] = 0.f;
            w[e] = be * kf[e];
            qf[e] *= Bv[e];
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            r[e] = kf[e];
            w[e] = be * Bv[e] * kf[e];
          }
        }
      } else if (kFG2) {
        // key-side gain gb (and, for FG2+, a value-side gain gv of its own)
        float gb[8], gv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { gb[e] = 0.f; gv[e] = 0.f; }
        if (L::kGates) {
          const uint8_t *gsrc = smem + L::kGateStage + t * 256 + ((c8 ^ (t & 7)) << 4);
          unpack8(*reinterpret_cast<const uint4 *>(gsrc), gb);
          if (kVariant == PDN_VAR_FG2_GDN_PLUS) unpack8(*reinterpret_cast<const uint4 *>(gsrc + 16384), gv);
        } else if (ok) {
          unpack8(__ldg(reinterpret_cast<const uint4 *>(
                      reinterpret_cast<const __nv_bfloat16 *>(P.beta) + etok + i0)), gb);
          if (kVariant == PDN_VAR_FG2_GDN_PLUS)
            unpack8(__ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(P.write) + etok + i0)), gv);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float sq = sqrt_gain(gate_act(P.prologue, gb[e]));
          r[e] = sq * kf[e];
          w[e] = r[e];
          vf[e] *= kVariant == PDN_VAR_FG2_GDN_PLUS ? sqrt_gain(gate_act(P.prologue, gv[e])) : sq;
        }
      } else if (kVariant == PDN_VAR_GDN2) {
        float ge[8], gw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { ge[e] = 0.f; gw[e] = 0.f; }
        if (L::kGates) {
          const uint8_t *gsrc = smem + L::kGateStage + t * 256 + ((c8 ^ (t & 7)) << 4);
          unpack8(*reinterpret_cast<const uint4 *>(gsrc), ge);
          unpack8(*reinterpret_cast<const uint4 *>(gsrc + 16384), gw);
        } else if (ok) {
          unpack8(__ldg(reinterpret_cast<const uint4 *>(
                      reinterpret_cast<const __nv_bfloat16 *>(P.erase) + etok + i0)), ge);
          unpack8(__ldg(reinterpret_cast<const uint4 *>(
                      reinterpret_cast<const __nv_bfloat16 *>(P.write) + etok + i0)), gw);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          r[e] = gate_act(P.prologue, ge[e]) * kf[e];
          w[e] = kf[e];
          vf[e] *= gate_act(P.prologue, gw[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          r[e] = kf[e];
          w[e] = be * kf[e];
        }
      }
      float rr[8], qq[8], wh[8], qh[8], wb[8];
      if (kCh) {
        float G[8], Bl[8], Bh[8], eBl[8], wbf[8], rsub[8];
        ld8f(GBUF + t * LB_LD + i0, G);
        ld8f(GBUF + (16 * a + 15) * LB_LD + i0, Bh);  // B_{a+1} (G_C for a = 3)
        if (a > 0) {
          ld8f(GBUF + (16 * a - 1) * LB_LD + i0, Bl);
          ld8f(TAB + (a - 1) * kD + i0, eBl);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) { Bl[e] = 0.f; eBl[e] = 1.f; }
        }
        if (a < 3) {
          ld8f(TAB + (6 + a) * kD + i0, wbf);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) wbf[e] = 1.f;
        }
        const bool bad_a = (badm >> a) & 1u;
        ld8f(TAB + (9 + a) * kD + i0, rsub);  // e^{B_a - B_{a+1}}
        float wy[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float rho = ex2_approx((G[e] - Bl[e]) * kLog2e);  // e^{G_t - B_a} <= 1
          const float y = ex2_approx((Bh[e] - G[e]) * kLog2e);    // e^{B_{a+1} - G_t} <= 1
          rr[e] = r[e] * rho;
          qq[e] = qf[e] * rho;
          qh[e] = qf[e] * (rho * eBl[e]);
          wb[e] = w[e] * (y * wbf[e]);
          wh[e] = bad_a ? 0.f : w[e] * (y * rsub[e]);  // diagonal group: e^{B_a - G_t}
          wy[e] = w[e] * y;
        }
        *reinterpret_cast<uint4 *>(smem + L::kWH + tl128(grp_off(a) + t, c8)) = pack8(wh);
        // later column groups: e^{B_a2 - G_t} = y e^{B_a2 - B_{a+1}}
#pragma unroll
        for (int a2 = 1; a2 < 4; ++a2) {
          if (a2 > a) {
            float lam[8];
            if (a2 == a + 1) {
#pragma unroll
              for (int e = 0; e < 8; ++e) lam[e] = 1.f;
            } else {
              ld8f(TAB + (a == 0 ? (a2 == 2 ? 3 : 4) : 5) * kD + i0, lam);
            }
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = wy[e] * lam[e];
            *reinterpret_cast<uint4 *>(smem + L::kWH + tl128(grp_off(a2) + t, c8)) = pack8(x);
          }
        }
        if (badm) {  // undecayed rows for the exact diagonal blocks
          *reinterpret_cast<uint4 *>(smem + L::kKS + t * KS_LD + c8 * 16) = pack8(r);
          *reinterpret_cast<uint4 *>(smem + L::kQS + t * KS_LD + c8 * 16) = pack8(qf);
          *reinterpret_cast<uint4 *>(smem + L::kBC + t * KS_LD + c8 * 16) = pack8(w);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          rr[e] = r[e];
          qq[e] = qf[e];
          wh[e] = w[e];
          qh[e] = qf[e] * eg_s;
          wb[e] = w[e] * ewb_s;
        }
        *reinterpret_cast<uint4 *>(smem + L::kWH + tl128(t, c8)) = pack8(wh);
      }
      *reinterpret_cast<uint4 *>(smem + L::kRQ + tl128(t, c8)) = pack8(rr);
      *reinterpret_cast<uint4 *>(smem + L::kRQ + tl128(64 + t, c8)) = pack8(qq);
      *reinterpret_cast<uint4 *>(blk + WS_Q + tl128(t, c8)) = pack8(qh);
      *reinterpret_cast<uint4 *>(blk + WS_WB + tl128(t, c8)) = pack8(wb);
      *reinterpret_cast<uint4 *>(blk + WS_U + tl128(t, c8)) = pack8(vf);
    }
  }

  // ---- MMA1: D1 = [R;Q] B^T ----
  sync_for_mma();
  if (tid == 0) {
    const uint32_t id = make_idesc_bf16(128, L::kN1, false, false);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ss(tm + 0, make_sdesc(sb + L::kRQ + 256 * kk, 128, 2048),
                  make_sdesc(sb + L::kWH + 256 * kk, 128, 2048), id, kk > 0);
    mma_commit(bar + 0);
  }
  bool ok_all = true;
  {
    bool ok = true;
    if (warp == 0) ok = mbar_wait_timed(bar + 0, par, kWaitNs);
    ok_all = !__syncthreads_or(!ok);
    tc_fence_after();
  }

  if (ok_all) {
    if (it + (int)gridDim.x < total) {
      stage_v(it + gridDim.x);
      if (kCh) stage_k(it + gridDim.x);
    }
    // ---- epilogue of MMA1: M = strict lower (rows 0-63), P = lower (rows
    // 64-127) with their in-chunk decay, first into registers ----
    const int row = 32 * (warp & 3) + lane;
    const int tr = row & 63;
    const bool isP = row >= 64;
    float mv[2][16];
    if (kCh) {
      const int alo = 2 * (warp & 1);  // sub-chunks alo (lanes 0-15), alo + 1 (lanes 16-31)
      const int a = alo + (lane >> 4);
      const bool lo = lane < 16;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int s0 = 32 * half + 16 * cc;
        float vl[16], vh[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) { vl[e] = 0.f; vh[e] = 0.f; }
        const bool okl = s0 <= 16 * alo, okh = s0 <= 16 * (alo + 1);
        if (okl) tmem_ld16(tm + lane_q + grp_off(alo) + s0, vl);
        if (okh) tmem_ld16(tm + lane_q + grp_off(alo + 1) + s0, vh);
        tmem_wait_ld();
        const int sd = 16 * a;  // first column of this row's diagonal block
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int s = s0 + e;
          float x = lo ? vl[e] : vh[e];
          if (s0 > sd || (s0 == sd && (isP ? s > tr : s >= tr))) x = 0.f;
          mv[cc][e] = x;
        }
        if (s0 == sd && ((badm >> a) & 1u)) {
          float ex[16];  // (its own array: mv stays in registers)
          diag_exact(smem + (isP ? L::kQS : L::kKS) + tr * KS_LD, smem + L::kBC, GBUF, tr, s0,
                     !isP, ex);
#pragma unroll
          for (int e = 0; e < 16; ++e) mv[cc][e] = ex[e];
        }
      }
      // R with the chunk-start reference for MMA2: e^{G_t} r = e^{B_a} (rho_t r)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int t = 8 * warp + (lane & 7), c8 = 4 * m + (lane >> 3), a2 = t >> 4;
        if (a2 > 0) {
          float x[8], eb[8];
          unpack8(*reinterpret_cast<const uint4 *>(smem + L::kRQ + tl128(t, c8)), x);
          ld8f(TAB + (a2 - 1) * kD + 8 * c8, eb);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] *= eb[e];
          *reinterpret_cast<uint4 *>(smem + L::kRQ + tl128(t, c8)) = pack8(x);
        }
      }
      if (badm) __syncthreads();  // the exact sums read region A, which the scratch below reuses
    } else {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int s0 = 32 * half + 16 * cc;
        float v[16];
        tmem_ld16(tm + lane_q + s0, v);
        tmem_wait_ld();
        const float gt = kSc ? GS[tr] : 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int s = s0 + e;
          float x = 0.f;
          if (isP ? s <= tr : s < tr) {
            x = v[e];
            if (kSc) x *= ex2_approx((gt - GS[s]) * kLog2e);  // e^{G_t - G_s} <= 1
          }
          mv[cc][e] = x;
        }
      }
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int s0 = 32 * half + 16 * cc;
      if (!isP) {
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
          *reinterpret_cast<float4 *>(MS + tr * MS_LD + s0 + 4 * e4) =
              make_float4(mv[cc][4 * e4], mv[cc][4 * e4 + 1], mv[cc][4 * e4 + 2], mv[cc][4 * e4 + 3]);
      } else {
        float lo8[8], hi8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo8[e] = mv[cc][e]; hi8[e] = mv[cc][8 + e]; }
        // P goes straight to the workspace (only the state kernel reads it)
        *reinterpret_cast<uint4 *>(blk + WS_P + tl64(tr, s0 / 8)) = pack8(lo8);
        *reinterpret_cast<uint4 *>(blk + WS_P + tl64(tr, s0 / 8 + 1)) = pack8(hi8);
      }
    }
    tc_fence_before();
    __syncthreads();
    // ---- solve: T = (I + M)^{-1} ----
    // L0: 16x16 diagonal blocks; the other threads zero the upper blocks the merges read
    if (tid < 64) {
      const int base = 16 * (tid >> 4), cc = tid & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc0 = (r == cc) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
        for (int s = 0; s < r; s += 2) {
          acc0 = fmaf(-MS[(base + r) * MS_LD + base + s], x[s], acc0);
          if (s + 1 < r) acc1 = fmaf(-MS[(base + r) * MS_LD + base + s + 1], x[s + 1], acc1);
        }
        x[r] = acc0 + acc1;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) TS[(base + r) * TS_LD + base + cc] = x[r];
    } else {
      for (int e = tid - 64; e < 512; e += kK1Threads - 64) {
        const int blk2 = e >> 8, r = (e >> 4) & 15, cc = e & 15;
        TS[(32 * blk2 + r) * TS_LD + 32 * blk2 + 16 + cc] = 0.f;
      }
    }
    __syncthreads();
    // L1: merge 16 -> 32 within [32p, 32p + 32): X = -T_D (M_CA T_A)
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
      *reinterpret_cast<float2 *>(TS + (o + 16 + r0 + 1) * TS_LD + o + c0b) = make_float2(-a10, -a11);
    }
    __syncthreads();
    // L2: merge 32 -> 64: X = -T_D (M[32:64, 0:32] T_A)
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
    // T to the workspace and to MMA2's operand tile; for scalar decay MMA2
    // multiplies the undecayed R, so its tile holds T Diag(e^{G_s}).
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int t = 8 * warp + (lane & 7), s8 = 4 * m + (lane >> 3);
      float v[8];
      ld8f(TS + t * TS_LD + 8 * s8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = (8 * s8 + e <= t) ? v[e] : 0.f;
      *reinterpret_cast<uint4 *>(blk + WS_T + tl64(t, s8)) = pack8(v);
      if (kSc) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= EGS[8 * s8 + e];
      }
      *reinterpret_cast<uint4 *>(smem + L::kTM + tl64(t, s8)) = pack8(v);
    }

    // ---- MMA2: Y^T = R^T T^T ----
    sync_for_mma();
    if (tid == 0) {
      const uint32_t id = make_idesc_bf16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + L::kTmY, make_sdesc(sb + L::kRQ + 4096 * kk, 2048, 128),
                    make_sdesc(sb + L::kTM + 256 * kk, 128, 1024), id, kk > 0);
      mma_commit(bar + 1);
    }
    {
      bool ok = true;
      if (warp == 0) ok = mbar_wait_timed(bar + 1, par, kWaitNs);
      ok_all = !__syncthreads_or(!ok);
      tc_fence_after();
    }
    if (ok_all) {
      // R is dead: the next block's k goes into its space
      if (!kCh && it + (int)gridDim.x < total) stage_k(it + gridDim.x);
      // Y^T -> bf16, straight to the workspace (rows d_k, columns tokens)
      const int i = 32 * (warp & 3) + lane;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[16];
        tmem_ld16(tm + lane_q + L::kTmY + 32 * half + 16 * cc, v);
        tmem_wait_ld();
        float lo[8], hi[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { lo[e] = v[e]; hi[e] = v[8 + e]; }
        const int t8 = 4 * half + 2 * cc;
        *reinterpret_cast<uint4 *>(blk + WS_Y + tl64(i, t8)) = pack8(lo);
        *reinterpret_cast<uint4 *>(blk + WS_Y + tl64(i, t8 + 1)) = pack8(hi);
      }
    }
  }
  if (!ok_all) {
    if (tid == 0) record_error(P.err, PDN_ERR_TIMEOUT);
    break;
  }
  // the next block reuses the shared memory and the TMEM columns read above
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  }  // chunk blocks
  cp_async_wait_all();  // a prefetch issued before an abort
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, L::kTmemCols);
}

// ===========================================================================
// K2: state pass, one CTA per (batch, head)
// ===========================================================================
// Warp roles. 16 compute warps (TMEM lane quarter x column group) run the
// epilogues of the state chain and write each chunk's output; the S warp
// issues the MMAs of the state chain (MMA3, MMA5, MMA8); the O warp issues
// the output MMAs (MMA6, MMA7); the load warp prefetches operands. They meet
// only at mbarriers:
//   fmain[x] main operand buffer x landed (bulk copy)
//   fut[x]   U/T operand buffer x landed
//   sepi     state epilogue of the chunk done (one arrival per compute warp)
//   depi     D^T epilogue of the chunk done (one arrival per compute warp)
//   bar5     MMA3 (U~^T) and MMA5 (D^T) done      (S warp)
//   bar7     MMA8 (state update) done             (S warp)
//   baro     MMA7 (O^T += D^T P^T) done: the chunk's output and, since the O
//            warp waits on bar7 first, every MMA of the chunk
//   ufree[x] MMA3 of the chunk in U/T buffer x done (the buffer may be refilled)
//   mfree[x] every MMA of the chunk in main buffer x done (likewise)
// The load warp waits only on ufree/mfree: a buffer's barrier cannot move on
// before the load warp has refilled it, so however far the load warp falls
// behind, the phase it waits for is never overtaken.
// The O warp issues MMA6 only after MMA5 and MMA7 only after MMA8 have
// completed, so the tensor pipe never holds output work ahead of the state
// chain's. The compute warps write chunk n - 1's output while MMA5 of chunk
// n runs. The A operands that the epilogues produce (S and D^T in bf16) stay
// in TMEM; only the B operands are read from shared memory.
//
// A chunk's operands come in two parts: the main part (Qh, Y^T, Wb, P,
// e^{G_C}) in a ring of three buffers, refilled for chunk n + 3 once every MMA
// of chunk n is done; U^T and T, which MMA3 reads a chunk early, in a ring of
// two, refilled for chunk n + 2 once MMA3 of chunk n is done. Every load thus
// has about two chunk periods to land.
constexpr int kK2Compute = 512;
constexpr int kK2SWarp = kK2Compute / 32, kK2OWarp = kK2SWarp + 1, kK2LoadWarp = kK2SWarp + 2;
constexpr int kK2Threads = kK2Compute + 96;
// main buffer: Qh, Y^T, Wb, then P and e^{G_C} (adjacent in the workspace too;
// the state epilogue takes e^{G_C} from its own copy, below)
constexpr uint32_t KM_Q = 0, KM_Y = 16384, KM_WB = 32768, KM_P = 49152;
constexpr uint32_t KM_SIZE = KM_P + (WS_SET - WS_P);
// U/T buffer
constexpr uint32_t KU_U = 0, KU_T = 16384, KU_SIZE = 16384 + (WS_P - WS_T);
constexpr uint32_t K2_MAIN = 0;                    // three main buffers
constexpr uint32_t K2_UT = 3 * KM_SIZE;            // two U/T buffers
constexpr uint32_t K2_BAR = K2_UT + 2 * KU_SIZE;   // the fifteen mbarriers above
constexpr uint32_t K2_ABORT = K2_BAR + 16 * 8;
constexpr uint32_t K2_TBASE = K2_ABORT + 8;
// e^{G_C} of the current and the next chunk, one copy per compute warp (the
// 32 key channels of its column group), fetched by the warp itself
// e^{G_C} of the current and the next chunk, one copy per compute warp (the
// 32 key channels of its column group), fetched by the warp itself
constexpr uint32_t K2_EBUF = (K2_TBASE + 16 + 127) / 128 * 128;
constexpr uint32_t K2_BYTES = K2_EBUF + 16 * 2 * 128;
static_assert(K2_BYTES <= 232448, "state kernel shared memory budget");

// TMEM columns: U~^T then D^T (fp32), the two O^T buffers, S in bf16 pairs
// (the A operand of MMA5/MMA6), S (fp32), D^T in bf16 pairs (A of MMA7/MMA8);
// the bf16 operands have two buffers each, by chunk parity, so that a chunk's
// epilogues never wait for the previous chunk's output MMAs.
constexpr uint32_t TM_UD = 0, TM_OT0 = 64, TM_OT1 = 128, TM_SB0 = 192, TM_S = 256, TM_DB0 = 384,
                   TM_DB1 = 416, TM_SB1 = 448;
__device__ __forceinline__ uint32_t tm_sb(int n) { return (n & 1) ? TM_SB1 : TM_SB0; }
__device__ __forceinline__ uint32_t tm_db(int n) { return (n & 1) ? TM_DB1 : TM_DB0; }

static_assert(WS_Q == 0 && WS_Y == 16384 && WS_U == 32768 && WS_WB == 49152 && WS_T == 65536 &&
                  WS_P == WS_T + 8192 && WS_E > WS_P && WS_SET > WS_E,
              "workspace block layout the operand loads assume");
static_assert(K2_MAIN % 128 == 0 && KM_SIZE % 128 == 0 && K2_UT % 128 == 0 && KU_SIZE % 128 == 0,
              "operand buffers 128-byte aligned");

// Main part of chunk block `src` into main buffer `dst`.
__device__ __forceinline__ void load_main(uint8_t *dst, const uint8_t *src, uint64_t *bar) {
  mbar_arrive_expect_tx(bar, KM_SIZE);
  bulk_g2s(dst + KM_Q, src + WS_Q, 16384, bar);
  bulk_g2s(dst + KM_Y, src + WS_Y, 16384, bar);
  bulk_g2s(dst + KM_WB, src + WS_WB, 16384, bar);
  bulk_g2s(dst + KM_P, src + WS_P, WS_SET - WS_P, bar);
}
// U^T and T of chunk block `src` into U/T buffer `dst`.
__device__ __forceinline__ void load_ut(uint8_t *dst, const uint8_t *src, uint64_t *bar) {
  mbar_arrive_expect_tx(bar, KU_SIZE);
  bulk_g2s(dst + KU_U, src + WS_U, 16384, bar);
  bulk_g2s(dst + KU_T, src + WS_T, WS_P - WS_T, bar);
}
__device__ __forceinline__ uint32_t main_buf(int n) { return K2_MAIN + (uint32_t)(n % 3) * KM_SIZE; }
__device__ __forceinline__ uint32_t ut_buf(int n) { return K2_UT + (uint32_t)(n & 1) * KU_SIZE; }

// One lane of the warp waits (bounded) on `bar`; the outcome is the warp's.
// A wait that runs out, or an abort raised elsewhere, sets the abort flag.
__device__ __forceinline__ bool k2_warp_wait(uint64_t *bar, uint32_t parity,
                                             volatile int *abort_flag, int lane) {
  bool ok = true;
  if (lane == 0) ok = mbar_wait_timed(bar, parity, kWaitNs) && !*abort_flag;
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  tc_fence_after();
  if (!ok && lane == 0) *abort_flag = 1;
  return ok;
}
// Publishes this warp's TMEM accesses to the issuing warps.
__device__ __forceinline__ void k2_warp_arrive(uint64_t *bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}
// Single-thread bounded wait for the issuing warps.
__device__ __forceinline__ bool k2_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  const bool ok = mbar_wait_timed(bar, parity, kWaitNs) && !*abort_flag;
  tc_fence_after();
  return ok;
}

// 8 output tokens (columns 16 cg + 8 part .. + 7 of O^T in TMEM, lanes =
// value channels) of one lane quarter; two adjacent channels per 32-bit store.
__device__ __forceinline__ void k2_store_o(const KParams &P, uint32_t taddr, int b, int h,
                                           int pc0, int Cn, int lane, int quarter, int cg,
                                           int part) {
  if (!P.o) return;  // transition mode writes no output
  const size_t tstride = (size_t)P.H * kD;
  const int j = 32 * quarter + lane;
  __nv_bfloat16 *orow =
      reinterpret_cast<__nv_bfloat16 *>(P.o) + tok_index(P, b, pc0, h) * kD + (j & ~1);
  const bool odd = lane & 1;
  float v[8];
  tmem_ld8(taddr + 16 * cg + 8 * part, v);
  tmem_wait_ld();
#pragma unroll
  for (int e2 = 0; e2 < 4; ++e2) {
    const float send = odd ? v[2 * e2] : v[2 * e2 + 1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const int t = 16 * cg + 8 * part + 2 * e2 + (odd ? 1 : 0);
    const float lo = odd ? recv : v[2 * e2];
    const float hi = odd ? v[2 * e2 + 1] : recv;
    if (t < Cn) *reinterpret_cast<uint32_t *>(orow + t * tstride) = pack_bf16(lo, hi);
  }
}

// MMA3: U~^T = U^T T^T of the chunk whose U/T buffer is at shared address `ut`.
__device__ __forceinline__ void k2_mma3(uint32_t tm, uint32_t ut) {
  const uint32_t id3 = make_idesc_bf16(128, 64, true, false);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_bf16_ss(tm + TM_UD, make_sdesc(ut + KU_U + 4096 * kk, 2048, 128),
                make_sdesc(ut + KU_T + 256 * kk, 128, 1024), id3, kk > 0);
}

struct K2Bars {
  uint64_t *fmain, *fut, *bar5, *bar7, *baro, *sepi, *depi, *ufree, *mfree;
};

// The S warp's program (one lane): MMA3, MMA5, MMA8. False if a wait ran out.
__device__ __forceinline__ bool k2_issue_s(uint32_t tm, uint32_t sb, const K2Bars &B,
                                           volatile int *abort_flag, int N) {
  const uint32_t id5 = make_idesc_bf16(128, 64, false, true, true);
  const uint32_t id8 = make_idesc_bf16(128, 128, false, true);
  for (int n = 0; n < N; ++n) {
    const uint32_t mb = sb + main_buf(n);
    if (n == 0) {
      if (!k2_wait(B.fut + 0, 0, abort_flag)) return false;
      k2_mma3(tm, sb + ut_buf(0));
      mma_commit(B.ufree + 0);
    }
    // MMA5: D^T = U~^T - S Y^T, once chunk n's main operands have landed and
    // the state epilogue has written S (bf16)
    if (!k2_wait(B.fmain + (n % 3), (uint32_t)((n / 3) & 1), abort_flag)) return false;
    if (!k2_wait(B.sepi, (uint32_t)(n & 1), abort_flag)) return false;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ts(tm + TM_UD, tm + tm_sb(n) + 8 * kk, make_sdesc(mb + KM_Y + 2048 * kk, 1024, 128),
                  id5, 1);
    mma_commit(B.bar5);
    // MMA8: S += D^T Wb, once D^T is in shared memory
    if (!k2_wait(B.depi, (uint32_t)(n & 1), abort_flag)) return false;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ts(tm + TM_S, tm + tm_db(n) + 8 * kk, make_sdesc(mb + KM_WB + 4096 * kk, 2048, 128),
                  id8, 1);
    mma_commit(B.bar7);
    // MMA3 of chunk n + 1 (the D^T epilogue has read this chunk's U~^T)
    if (n + 1 < N) {
      if (!k2_wait(B.fut + ((n + 1) & 1), (uint32_t)(((n + 1) >> 1) & 1), abort_flag)) return false;
      k2_mma3(tm, sb + ut_buf(n + 1));
      mma_commit(B.ufree + ((n + 1) & 1));
    }
  }
  return true;
}

// The O warp's program (one lane): MMA6, MMA7. False if a wait ran out.
__device__ __forceinline__ bool k2_issue_o(uint32_t tm, uint32_t sb, const K2Bars &B,
                                           volatile int *abort_flag, int N) {
  const uint32_t id6 = make_idesc_bf16(128, 64, false, false);
  const uint32_t id7 = make_idesc_bf16(128, 64, false, false);
  for (int n = 0; n < N; ++n) {
    const uint32_t mb = sb + main_buf(n);
    const uint32_t ot = (n & 1) ? TM_OT1 : TM_OT0;
    // MMA6: O^T = S Qh^T after MMA5 (which also means the compute warps have
    // written out chunk n - 2's output from this buffer), on operands this
    // warp has seen land
    if (!k2_wait(B.bar5, (uint32_t)(n & 1), abort_flag)) return false;
    if (!k2_wait(B.fmain + (n % 3), (uint32_t)((n / 3) & 1), abort_flag)) return false;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ts(tm + ot, tm + tm_sb(n) + 8 * kk, make_sdesc(mb + KM_Q + 256 * kk, 128, 2048), id6,
                  kk > 0);
    // MMA7: O^T += D^T P^T after MMA8
    if (!k2_wait(B.bar7, (uint32_t)(n & 1), abort_flag)) return false;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ts(tm + ot, tm + tm_db(n) + 8 * kk, make_sdesc(mb + KM_P + 256 * kk, 128, 1024), id7,
                  1);
    mma_commit(B.baro);
    mma_commit(B.mfree + (n % 3));
  }
  return true;
}

// Walks chunks cb .. cb + N - 1, from P.S0 (or zeros; the identity in
// transition mode when P.S0 is NULL) to P.ST.
__global__ void __launch_bounds__(kK2Threads, 1) k2_state(const KParams P, void *ws, int N,
                                                          int cb) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K2_BAR);
  const K2Bars B{bars,     bars + 3, bars + 5,  bars + 6, bars + 7,
                 bars + 8, bars + 9, bars + 10, bars + 12};
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + K2_ABORT);
  uint32_t *tbase_p = reinterpret_cast<uint32_t *>(smem + K2_TBASE);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3;
  const uint32_t lane_q = (uint32_t)(32 * quarter) << 16;
  const int bh = blockIdx.x, b = bh / P.H, h = bh % P.H;

  if (warp == 0) {
    tmem_alloc(tbase_p, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(bars + i, 1);
    for (int i = 10; i < 15; ++i) mbar_init(bars + i, 1);
    mbar_init(B.sepi, kK2Compute / 32);
    mbar_init(B.depi, kK2Compute / 32);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tbase_p;

  if (warp == kK2SWarp) {
    // ======================= S warp =======================
    if (lane == 0 && !k2_issue_s(tm, sb, B, abort_flag, N)) *abort_flag = 1;
    __syncwarp();
  } else if (warp == kK2OWarp) {
    // ======================= O warp =======================
    if (lane == 0 && !k2_issue_o(tm, sb, B, abort_flag, N)) *abort_flag = 1;
    __syncwarp();
  } else if (warp == kK2LoadWarp) {
    // ======================= load warp =======================
    if (lane == 0) {
      const int BH = P.B * P.H;
      for (int m = 0; m < 3 && m < N; ++m)
        load_main(smem + main_buf(m), ws_block(ws, bh, BH, chunk_ok(P, cb + m)), B.fmain + m);
      for (int m = 0; m < 2 && m < N; ++m)
        load_ut(smem + ut_buf(m), ws_block(ws, bh, BH, chunk_ok(P, cb + m)), B.fut + m);
      // after MMA3 of chunk n, its U/T buffer takes chunk n + 2; after every
      // MMA of chunk n, its main buffer takes chunk n + 3
      for (int n = 0; n + 2 < N; ++n) {
        if (!k2_wait(B.ufree + (n & 1), (uint32_t)((n >> 1) & 1), abort_flag)) {
          *abort_flag = 1;
          break;
        }
        load_ut(smem + ut_buf(n), ws_block(ws, bh, BH, chunk_ok(P, cb + n + 2)), B.fut + (n & 1));
        if (n + 3 < N) {
          if (!k2_wait(B.mfree + (n % 3), (uint32_t)((n / 3) & 1), abort_flag)) {
            *abort_flag = 1;
            break;
          }
          load_main(smem + main_buf(n), ws_block(ws, bh, BH, chunk_ok(P, cb + n + 3)),
                    B.fmain + (n % 3));
        }
      }
    }
    __syncwarp();
  } else {
    // ======================= compute warps =======================
    const int cg = warp >> 2;          // column group 0..3
    const int j = 32 * quarter + lane; // value channel owned in the epilogues
    bool ok = true;
    // this warp's 32 values of e^{G_C} for chunk c into its buffer c & 1
    auto fetch_e = [&](int c) {
      if (lane < 8)
        cp_async16(sb + K2_EBUF + (warp * 2 + (c & 1)) * 128 + lane * 16,
                   reinterpret_cast<const float *>(ws_block(ws, bh, P.B * P.H, chunk_ok(P, cb + c)) + WS_E) + 32 * cg +
                       4 * lane,
                   true);
      cp_async_commit();
    };
    if (N > 0) fetch_e(0);
    for (int n = 0; n < N; ++n) {
      const int s = n & 1;
      // this chunk's e^{G_C} has landed (fetched by the warp a chunk ahead).
      // (MMA8 of chunk n - 1, which the state needs, was awaited at the end of
      // the previous iteration; the bf16 S buffer this chunk writes was last
      // read by MMA5 and MMA6 of chunk n - 2, both done before that chunk's
      // output.)
      cp_async_wait_all();
      __syncwarp();

      // ---- state epilogue: S -> bf16 operand; TMEM S <- S Diag(e^{G_C}) ----
      {
        const float *egc = reinterpret_cast<const float *>(smem + K2_EBUF + (warp * 2 + (n & 1)) * 128);
        float sv[2][16];
        const int col0 = 32 * cg;
        if (n == 0) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (P.transition && !P.S0) {  // the identity: S[j][i] = (i == j)
#pragma unroll
              for (int e = 0; e < 16; ++e) sv[u][e] = (col0 + 16 * u + e == j) ? 1.f : 0.f;
            } else if (P.S0) {
              const float4 *src = reinterpret_cast<const float4 *>(
                  P.S0 + ((size_t)bh * kD + j) * kD + col0 + 16 * u);
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
          tmem_ld16(tm + lane_q + TM_S + col0, sv[0]);
          tmem_ld16(tm + lane_q + TM_S + col0 + 16, sv[1]);
          tmem_wait_ld();
        }
        {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[8 * u + e] = pack_bf16(sv[u][2 * e], sv[u][2 * e + 1]);
          tmem_st16u(tm + lane_q + tm_sb(n) + 16 * cg, pk);
        }
        tmem_wait_st();
        // MMA5 and MMA6 read only the bf16 copy: hand it over now. The decayed
        // fp32 state below is MMA8's accumulator, and MMA8 waits for this
        // warp's D-epilogue arrive, which follows a tcgen05.wait::st covering
        // these stores too; nothing issued before it touches TM_S.
        k2_warp_arrive(B.sepi, lane);
        if (P.sv_ckpt) {
          // training mode: the state at the start of chunk cb + n, stored
          // transposed ([d_k][d_v] per chunk) so that a warp's 32 rows j of
          // one column are one 128-byte line (row-major, each lane's float4s
          // scattered over 32 lines and held up the epilogue on the
          // load/store unit)
          const size_t nch = (size_t)(P.T + kC - 1) / kC;
          float *dst = P.sv_ckpt + (((size_t)bh * nch + chunk_ok(P, cb + n)) * kD + col0) * kD + j;
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[(size_t)(16 * u + e) * kD] = sv[u][e];
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = col0 + 16 * u;
          float E[8];
          ld8f(egc + (col - col0), E);
#pragma unroll
          for (int e = 0; e < 8; ++e) sv[u][e] *= E[e];
          ld8f(egc + (col - col0) + 8, E);
#pragma unroll
          for (int e = 0; e < 8; ++e) sv[u][8 + e] *= E[e];
          tmem_st16(tm + lane_q + TM_S + col, sv[u]);
        }
        tmem_wait_st();
      }
      // chunk n - 1's output in two halves, under MMA5 and under MMA8 (the
      // O^T buffer they free takes chunk n + 1, whose MMA6 comes after this
      // chunk's epilogues)
      const uint32_t ot_prev = tm + lane_q + (s ? TM_OT0 : TM_OT1);
      const int pc_prev = (cb + n - 1) * kC;
      if (n > 0) {
        if (!(ok = k2_warp_wait(B.baro, (uint32_t)((n - 1) & 1), abort_flag, lane))) break;
        k2_store_o(P, ot_prev, b, h, pc_prev, min(kC, P.T - pc_prev), lane, quarter, cg, 0);
      }
      if (!(ok = k2_warp_wait(B.bar5, (uint32_t)(n & 1), abort_flag, lane))) break;

      // ---- D^T -> bf16 operand in TMEM (lanes d_v, token pairs per column) ----
      {
        float v[16];
        tmem_ld16(tm + lane_q + TM_UD + 16 * cg, v);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        tmem_st8u(tm + lane_q + tm_db(n) + 8 * cg, pk);
        tmem_wait_st();
        k2_warp_arrive(B.depi, lane);
        if (P.sv_delta) {  // training mode: delta of tokens 16 cg .. 16 cg + 15, row j (after the hand-back)
          const int t0 = chunk_ok(P, cb + n) * kC + 16 * cg;
          float *dst = P.sv_delta + ((size_t)bh * P.T + t0) * kD + j;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (t0 + e < P.T) dst[(size_t)e * kD] = v[e];
        }
      }
      if (n + 1 < N) fetch_e(n + 1);
      if (n > 0) k2_store_o(P, ot_prev, b, h, pc_prev, min(kC, P.T - pc_prev), lane, quarter, cg, 1);
      if (!(ok = k2_warp_wait(B.bar7, (uint32_t)(n & 1), abort_flag, lane))) break;
    }
    // the last chunk's output
    if (ok && N > 0 && k2_warp_wait(B.baro, (uint32_t)((N - 1) & 1), abort_flag, lane)) {
      const int pc0 = (cb + N - 1) * kC;
      for (int part = 0; part < 2; ++part)
        k2_store_o(P, tm + lane_q + (((N - 1) & 1) ? TM_OT1 : TM_OT0), b, h, pc0,
                   min(kC, P.T - pc0), lane, quarter, cg, part);
    }
    if (!*abort_flag && N > 0 && P.ST) {
      float v[2][16];
      const int col0 = 32 * cg;
      tmem_ld16(tm + lane_q + TM_S + col0, v[0]);
      tmem_ld16(tm + lane_q + TM_S + col0 + 16, v[1]);
      tmem_wait_ld();
      float4 *dst = reinterpret_cast<float4 *>(P.ST + ((size_t)bh * kD + j) * kD + col0);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[4 * u + e] = make_float4(v[u][4 * e], v[u][4 * e + 1], v[u][4 * e + 2], v[u][4 * e + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    if (tid == 0) {
      record_error(P.err, PDN_ERR_TIMEOUT);
      // drain operand loads still in flight before shared memory goes away
      for (int x = 0; x < 5; ++x) {
        mbar_wait_timed(bars + x, 0, kDrainNs);
        mbar_wait_timed(bars + x, 1, kDrainNs);
      }
    }
    __syncthreads();
  }
  if (warp == 0) tmem_dealloc(tm, 512);
}

template <int V, int Dc>
cudaError_t launch_k1(const KParams &P, void *ws, int N, int it0, int it1, int sm_budget,
                      cudaStream_t stream) {
  using L = K1Layout<V, Dc>;
  auto kern = k1_intra<V, Dc>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
  if (e != cudaSuccess) return e;
  // the largest shared-memory carveout, so that two CTAs fit on an SM
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kK1Threads, L::kBytes) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  if (sm_budget > 0 && sm_budget < sms) sms = sm_budget;
  const long long total = (long long)it1 - it0;
  if (total <= 0) return cudaSuccess;
  // At least two CTAs per SM (unless the SMs are budgeted): the blocks are
  // independent, so a CTA that does not fit yet simply starts when one
  // finishes, at no loss.
  if (per_sm < 2 && sm_budget <= 0) per_sm = 2;
  const long long grid = total < (long long)sms * per_sm ? total : (long long)sms * per_sm;
  kern<<<(unsigned)grid, kK1Threads, L::kBytes, stream>>>(P, ws, N, it0, it1);
  return cudaGetLastError();
}

template <int V>
cudaError_t launch_k1_decay(const KParams &P, void *ws, int N, int it0, int it1, int sm_budget,
                            cudaStream_t stream) {
  switch (P.decay) {
    case PDN_DECAY_NONE: return launch_k1<V, PDN_DECAY_NONE>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_DECAY_SCALAR:
      return launch_k1<V, PDN_DECAY_SCALAR>(P, ws, N, it0, it1, sm_budget, stream);
    default: return launch_k1<V, PDN_DECAY_CHANNEL>(P, ws, N, it0, it1, sm_budget, stream);
  }
}

cudaError_t launch_k1_range(const KParams &P, void *ws, int N, int it0, int it1, int sm_budget,
                            cudaStream_t stream) {
  switch (P.variant) {
    case PDN_VAR_DN: return launch_k1_decay<PDN_VAR_DN>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_GDN: return launch_k1_decay<PDN_VAR_GDN>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_KDA: return launch_k1_decay<PDN_VAR_KDA>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_PDN: return launch_k1_decay<PDN_VAR_PDN>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_PGDN: return launch_k1_decay<PDN_VAR_PGDN>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_PKDA: return launch_k1_decay<PDN_VAR_PKDA>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_FG2_GDN:
      return launch_k1_decay<PDN_VAR_FG2_GDN>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_GDN2: return launch_k1_decay<PDN_VAR_GDN2>(P, ws, N, it0, it1, sm_budget, stream);
    case PDN_VAR_PLA: return launch_k1_decay<PDN_VAR_PLA>(P, ws, N, it0, it1, sm_budget, stream);
    default:
      return launch_k1_decay<PDN_VAR_FG2_GDN_PLUS>(P, ws, N, it0, it1, sm_budget, stream);
  }
}

// Long sequences over few chains: the state pass runs one CTA per chain, so
// with B*H well below the SM count most SMs idle through it. The chunks are
// then cut into kSegs time segments; K1 of segment i + 1 runs on the SMs the
// state pass leaves free while K2 walks segment i on a second stream, joined
// by events (no kernel waits on another). K2 carries the state from segment
// to segment through P.ST (each CTA reads its rows before it rewrites them).
constexpr int kSegs = 8;
constexpr int kMaxDev = 64;
struct SegRes {
  cudaStream_t s2 = nullptr;
  cudaEvent_t ev[kSegs + 1] = {};
};
SegRes g_seg[kMaxDev];
std::mutex g_seg_mu;

bool use_segments(const KParams &P, int N, int sms) {
  return P.ST != nullptr && N >= 8 * kSegs && (long long)P.B * P.H * 3 <= sms;
}

}  // namespace

int split_supported(const KParams &P) {
  const long long N = (P.T + kC - 1) / kC;
  return P.dtype == PDN_BF16 && P.dk == kD && P.dv == kD && P.chunk == kC && P.T > 0 &&
         (long long)P.B * P.H <= 65535 && N <= 65535;
}

size_t split_workspace_bytes(const KParams &P) {
  const size_t N = (size_t)((P.T + kC - 1) / kC);
  return (size_t)P.B * P.H * N * WS_CH;
}

cudaError_t launch_chunk_split(const KParams &P, void *ws, cudaStream_t stream,
                               cudaEvent_t *ev) {
  const int N = (P.T + kC - 1) / kC;
  const int BH = P.B * P.H;
  cudaError_t e;
  if (ev && (e = cudaEventRecord(ev[0], stream)) != cudaSuccess) return e;
  if (is_precond(P.variant)) {
    const long long blocks = (long long)N * BH;
    k0_chunk_energy<<<(unsigned)(blocks < (1LL << 30) ? blocks : (1LL << 30)), 256, 0, stream>>>(P, ws, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k0_prefix<<<BH, kD * kK0Groups, 0, stream>>>(P, ws, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (ev && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k2_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K2_BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (ev || dev < 0 || dev >= kMaxDev || !use_segments(P, N, sms)) {
    if ((e = launch_k1_range(P, ws, N, 0, N * BH, 0, stream)) != cudaSuccess) return e;
    if (ev && (e = cudaEventRecord(ev[2], stream)) != cudaSuccess) return e;
    k2_state<<<BH, kK2Threads, K2_BYTES, stream>>>(P, ws, N, 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return ev ? cudaEventRecord(ev[3], stream) : cudaSuccess;
  }
  // segmented: the calls share the device's second stream and events, so
  // their enqueueing is serialised
  std::lock_guard<std::mutex> lock(g_seg_mu);
  SegRes &R = g_seg[dev];
  if (!R.s2) {
    if ((e = cudaStreamCreateWithFlags(&R.s2, cudaStreamNonBlocking)) != cudaSuccess) {
      R.s2 = nullptr;
      return e;
    }
    for (int i = 0; i <= kSegs; ++i)
      if ((e = cudaEventCreateWithFlags(&R.ev[i], cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  for (int g = 0; g < kSegs; ++g) {
    const int c0 = (int)((long long)N * g / kSegs), c1 = (int)((long long)N * (g + 1) / kSegs);
    // the first segment has the whole GPU; later ones leave the state pass its SMs
    e = launch_k1_range(P, ws, N, c0 * BH, c1 * BH, g == 0 ? 0 : sms - BH, stream);
    if (e == cudaSuccess) e = cudaEventRecord(R.ev[g], stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(R.s2, R.ev[g], 0);
    if (e != cudaSuccess) break;
    KParams Pg = P;
    if (g > 0) Pg.S0 = P.ST;  // the state where the previous segment left it
    k2_state<<<BH, kK2Threads, K2_BYTES, R.s2>>>(Pg, ws, c1 - c0, c0);
    if ((e = cudaGetLastError()) != cudaSuccess) break;
  }
  // join the second stream back into the caller's on every path
  cudaError_t j = cudaEventRecord(R.ev[kSegs], R.s2);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, R.ev[kSegs], 0);
  return e != cudaSuccess ? e : j;
}

}  // namespace pdn
