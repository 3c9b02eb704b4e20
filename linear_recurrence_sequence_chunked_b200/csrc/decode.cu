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
// (token, head) against about 7 d_k d_v flops. For d_k = d_v = 128 a
// persistent variant streams the state through shared memory with bulk
// copies (see decode_tma_kernel).
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
  }
  if (P.prologue & PDN_PRO_L2NORM_QK) {  // fused prologue: unit-norm k and q
    const float ssk = block_sum(chan ? kv * kv : 0.f, s_red);
    const float ssq = block_sum(chan ? qv * qv : 0.f, s_red);
    kv *= inv_norm(ssk);
    qv *= inv_norm(ssq);
  }
  if (chan) {
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
        w = gate_act(P.prologue, ldf<float>(P.beta, tokh)) * precond_coef(logA, mu, P.lnx) * kv;
        break;
      case PDN_VAR_PLA:  // no erase; the preconditioner acts on the query
        r = 0.f;
        w = gate_act(P.prologue, ldf<float>(P.beta, tokh)) * kv;
        qv *= precond_coef(logA, mu, P.lnx);
        break;
      case PDN_VAR_FG2_GDN: case PDN_VAR_FG2_GDN_PLUS:
        r = sqrtf(gate_act(P.prologue, ldf<Tin>(P.beta, tokh * dk + tid))) * kv;
        w = r;
        break;
      case PDN_VAR_GDN2:
        r = gate_act(P.prologue, ldf<Tin>(P.erase, tokh * dk + tid)) * kv;
        w = kv;
        break;
      default:
        r = kv;
        w = gate_act(P.prologue, ldf<float>(P.beta, tokh)) * kv;
    }
    s_r[tid] = r;
    s_w[tid] = w;
    s_q[tid] = qv;
    float al = 1.f;
    if (P.decay == PDN_DECAY_SCALAR)
      al = expf(decay_act(P.prologue, P.decay_scale, ldf<float>(P.log_alpha, tokh)));
    else if (P.decay == PDN_DECAY_CHANNEL)
      al = expf(decay_act(P.prologue, P.decay_scale, ldf<Tin>(P.log_alpha, tokh * dk + tid)));
    s_al[tid] = al;
  }
  for (int j = tid; j < dv; j += kThreads) {
    float u = ldf<Tin>(P.v, tokh * dv + j);
    if (P.variant == PDN_VAR_FG2_GDN) u *= sqrtf(gate_act(P.prologue, ldf<Tin>(P.beta, tokh * dv + j)));
    else if (P.variant == PDN_VAR_GDN2) u *= gate_act(P.prologue, ldf<Tin>(P.write, tokh * dv + j));
    else if (P.variant == PDN_VAR_FG2_GDN_PLUS)
      u *= sqrtf(gate_act(P.prologue, ldf<Tin>(P.write, tokh * dv + j)));
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

// ---------------------------------------------------------------------------
// d_k = d_v = 128: persistent, warp-specialised variant. One CTA per SM walks
// the (batch, head) items. A producer warp streams each item's 64 KiB state
// into a ring of shared-memory buffers with 1-D bulk copies (TMA) and streams
// the updated buffer back with bulk stores; eight consumer warps do the
// per-token prologue and the row updates in shared memory. Full/empty
// mbarriers hand buffers between the two; every wait is bounded.
constexpr int kTmaBufs = 3;
constexpr float kLog2eD = 1.4426950408889634f, kLn2D = 0.6931471805599453f;
constexpr int kD128 = 128;
constexpr int kConsumers = kThreads;      // 8 consumer warps
constexpr int kTmaThreads = kThreads + 32;  // + 1 producer warp
constexpr uint32_t kStateBytes = kD128 * kD128 * 4;
constexpr uint32_t kPart = 16384;  // bytes per bulk copy

// The token vectors and the reduction slots are double-buffered by item
// parity: item k + 1's prologue writes the other half, and item k - 1's
// readers are all past item k's first barrier, so no barrier closes an item.
struct DecSmem {
  float buf[kTmaBufs][kD128 * kD128];
  float r[2][kD128], w[2][kD128], q[2][kD128], al[2][kD128], u[2][kD128];
  float red[2][4][kWarps];  // per parity: |k|^2, |q|^2, mean log A, w.q
  uint64_t full[kTmaBufs];
  uint64_t empty[kTmaBufs];
  int vote[2][kWarps];
  int abort_flag;
};

// Barrier among the consumer warps only (id 1); the producer never joins it.
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kConsumers) : "memory");
}

// Sum over the consumer warps through `red` (kWarps slots no other reduction
// of the same item uses): one barrier.
__device__ __forceinline__ float consumer_sum(float v, float *red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  consumer_sync();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += red[w];
  return s;
}

__device__ __forceinline__ void issue_state_load(DecSmem &sm, int s, const float *S) {
  mbar_arrive_expect_tx(&sm.full[s], kStateBytes);
#pragma unroll
  for (int p = 0; p < (int)(kStateBytes / kPart); ++p)
    bulk_g2s(reinterpret_cast<uint8_t *>(sm.buf[s]) + p * kPart,
             reinterpret_cast<const uint8_t *>(S) + p * kPart, kPart, &sm.full[s]);
}

__device__ __forceinline__ void issue_state_store(DecSmem &sm, int s, float *S) {
#pragma unroll
  for (int p = 0; p < (int)(kStateBytes / kPart); ++p)
    bulk_s2g(reinterpret_cast<uint8_t *>(S) + p * kPart,
             reinterpret_cast<const uint8_t *>(sm.buf[s]) + p * kPart, kPart);
  bulk_commit();
}

template <typename Tin>
__global__ void __launch_bounds__(kTmaThreads, 1) decode_tma_kernel(const KParams P, int items) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem &sm = *reinterpret_cast<DecSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int nloc = blockIdx.x < items ? (items - blockIdx.x + G - 1) / G : 0;
  const bool precond = is_precond(P.variant);
  // (the debug build checks the item index; a bad one records PDN_ERR_BOUNDS
  // and streams item 0 instead, so that no copy a consumer waits for is lost)
  auto state_of = [&](int k) {
    const int it = blockIdx.x + k * G;
    return P.ST + (size_t)(in_bounds(P.err, it < items) ? it : 0) * (kD128 * kD128);
  };

  if (tid == 0) {
    for (int s = 0; s < kTmaBufs; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kWarps);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------- producer warp
    if (lane == 0) {
      int loaded = 0;  // loads issued
      for (int k = 0; k < nloc; ++k) {
        const int s = k % kTmaBufs;
        if (k >= kTmaBufs) {
          // the consumers are done with item k - kTmaBufs in buffer s
          if (!mbar_wait_timed(&sm.empty[s], (uint32_t)(((k / kTmaBufs) - 1) & 1), kWaitNs) ||
              *reinterpret_cast<volatile int *>(&sm.abort_flag)) {
            atomicExch(&sm.abort_flag, 1);
            break;
          }
          issue_state_store(sm, s, state_of(k - kTmaBufs));
          bulk_wait_read0();
        }
        issue_state_load(sm, s, state_of(k));
        loaded = k + 1;
      }
      // write back the last items, then wait for all stores
      for (int k = (loaded > kTmaBufs ? loaded - kTmaBufs : 0); k < loaded; ++k) {
        const int s = k % kTmaBufs;
        if (!mbar_wait_timed(&sm.empty[s], (uint32_t)((k / kTmaBufs) & 1), kWaitNs)) {
          atomicExch(&sm.abort_flag, 1);
          // drain the load into this buffer before giving up on it
          mbar_wait_timed(&sm.full[s], (uint32_t)((k / kTmaBufs) & 1), kDrainNs);
          continue;
        }
        issue_state_store(sm, s, state_of(k));
      }
      bulk_wait0();
      if (sm.abort_flag) record_error(P.err, PDN_ERR_TIMEOUT);
    }
    return;
  }

  // ---------------- consumer warps
  // Token data of one item, loaded one item ahead (thread = key/value channel).
  struct Tok {
    float k, q, v, a, beta, la, ge, gw;
  };
  const bool chan = tid < kD128;
  auto load_tok = [&](int kk) {
    Tok t{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 1.f, 1.f};
    const int item = blockIdx.x + kk * G;
    const size_t tokh = tok_index(P, item / P.H, 0, item % P.H);
    if (chan) {
      const size_t e = tokh * kD128 + tid;
      t.k = ldf<Tin>(P.k, e);
      t.q = ldf<Tin>(P.q, e);
      t.v = ldf<Tin>(P.v, e);
      if (precond) t.a = P.AT[(size_t)item * kD128 + tid];
      const int pro = P.prologue;
      if (P.variant == PDN_VAR_FG2_GDN || P.variant == PDN_VAR_FG2_GDN_PLUS)
        t.beta = gate_act(pro, ldf<Tin>(P.beta, e));
      else if (P.variant != PDN_VAR_GDN2)
        t.beta = gate_act(pro, ldf<float>(P.beta, tokh));
      if (P.decay == PDN_DECAY_SCALAR) t.la = decay_act(pro, P.decay_scale, ldf<float>(P.log_alpha, tokh));
      else if (P.decay == PDN_DECAY_CHANNEL) t.la = decay_act(pro, P.decay_scale, ldf<Tin>(P.log_alpha, e));
      if (P.variant == PDN_VAR_GDN2) {
        t.ge = gate_act(pro, ldf<Tin>(P.erase, e));
        t.gw = gate_act(pro, ldf<Tin>(P.write, e));
      } else if (P.variant == PDN_VAR_FG2_GDN_PLUS) {
        t.gw = gate_act(pro, ldf<Tin>(P.write, e));
      }
    }
    return t;
  };
  Tok cur = nloc > 0 ? load_tok(0) : Tok{};
  for (int k = 0; k < nloc; ++k) {
    const int s = k % kTmaBufs;
    const int item = blockIdx.x + k * G;
    const int b = item / P.H, h = item % P.H;
    const size_t tokh = tok_index(P, b, 0, h);
    const Tok nxt = (k + 1 < nloc) ? load_tok(k + 1) : cur;

    // per-token vectors (overlap the bulk loads in flight)
    const int par = k & 1;
    float kv = cur.k, qv = cur.q;
    if (P.prologue & PDN_PRO_L2NORM_QK) {  // fused prologue: unit-norm k and q
      const float ssk = consumer_sum(chan ? kv * kv : 0.f, sm.red[par][0]);
      const float ssq = consumer_sum(chan ? qv * qv : 0.f, sm.red[par][1]);
      kv *= inv_norm(ssk);
      qv *= inv_norm(ssq);
    }
    float logA = 0.f;
    if (chan && precond) {
      const float a = cur.a + kv * kv;
      P.AT[(size_t)item * kD128 + tid] = a;
      logA = lg2_approx(a + P.eps);  // base 2, as the intra-chunk kernel
    }
    float mu = 0.f;
    if (precond) mu = consumer_sum(chan ? logA : 0.f, sm.red[par][2]) * (1.f / (float)kD128);
    // B = x^{-s}, s = c / (1 + |c|), c = ln(A + eps) - mean (hardware exp2 / rcp)
    auto coef = [&]() {
      const float cc = (logA - mu) * kLn2D;
      return ex2_approx(-(cc * rcp_approx(1.f + fabsf(cc))) * (P.lnx * kLog2eD));
    };
    float w = 0.f;
    if (chan) {
      float r, u = cur.v;
      switch (P.variant) {
        case PDN_VAR_PDN: case PDN_VAR_PGDN: case PDN_VAR_PKDA:
          r = kv;
          w = cur.beta * coef() * kv;
          break;
        case PDN_VAR_PLA:  // no erase; the preconditioner acts on the query
          r = 0.f;
          w = cur.beta * kv;
          qv *= coef();
          break;
        case PDN_VAR_FG2_GDN: case PDN_VAR_FG2_GDN_PLUS: {
          const float sb = sqrtf(cur.beta);
          r = sb * kv;
          w = r;
          u *= P.variant == PDN_VAR_FG2_GDN_PLUS ? sqrtf(cur.gw) : sb;
        } break;
        case PDN_VAR_GDN2:
          r = cur.ge * kv;
          w = kv;
          u *= cur.gw;
          break;
        default:
          r = kv;
          w = cur.beta * kv;
      }
      sm.r[par][tid] = r;
      sm.w[par][tid] = w;
      sm.q[par][tid] = qv;
      sm.al[par][tid] = P.decay == PDN_DECAY_NONE ? 1.f : ex2_approx(cur.la * kLog2eD);
      sm.u[par][tid] = u;
    }
    const float wq = consumer_sum(chan ? w * qv : 0.f, sm.red[par][3]);  // ends with a barrier

    // Wait for the state. The decision to stop must be the same in every
    // consumer warp (they meet at named barriers): each warp votes once,
    // after a consumer barrier all warps read all votes.
    const bool ok = mbar_wait_timed(&sm.full[s], (uint32_t)((k / kTmaBufs) & 1), kWaitNs);
    int vote = __all_sync(0xffffffffu, ok) ? 1 : 0;
    if (lane == 0) {
      if (*reinterpret_cast<volatile int *>(&sm.abort_flag)) vote = 0;
      sm.vote[par][warp] = vote;
    }
    consumer_sync();
    bool all_ok = true;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) all_ok = all_ok && sm.vote[par][i];
    if (!all_ok) {
      if (tid == 0) atomicExch(&sm.abort_flag, 1);
      break;
    }

    const int c = lane * 4;
    const float4 rr = *reinterpret_cast<const float4 *>(&sm.r[par][c]);
    const float4 ww = *reinterpret_cast<const float4 *>(&sm.w[par][c]);
    const float4 qq = *reinterpret_cast<const float4 *>(&sm.q[par][c]);
    const float4 aa = *reinterpret_cast<const float4 *>(&sm.al[par][c]);
    float *S = sm.buf[s];
    // The warp's 16 rows j = warp + 8 m at once: decayed rows in registers,
    // their 32 partial sums (y_m = S'_j r, then z_m = S'_j q) reduced together
    // by a transposed butterfly (31 shuffles; lane l ends with sum l), the
    // deltas broadcast back, the rows updated and stored.
    constexpr int kR = kD128 / kWarps;  // 16 rows per warp
    static_assert(2 * kR == 32, "two partial sums per row, one lane per sum");
    float4 X[kR];
    float v[2 * kR];
#pragma unroll
    for (int m = 0; m < kR; ++m) {
      const int j = warp + m * kWarps;
      float4 x = *reinterpret_cast<const float4 *>(S + j * kD128 + c);
      x.x *= aa.x; x.y *= aa.y; x.z *= aa.z; x.w *= aa.w;
      X[m] = x;
      v[m] = x.x * rr.x + x.y * rr.y + x.z * rr.z + x.w * rr.w;
      v[kR + m] = x.x * qq.x + x.y * qq.y + x.z * qq.z + x.w * qq.w;
    }
#pragma unroll
    for (int off = 16, len = kR; off >= 1; off >>= 1, len >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int e = 0; e < len; ++e) {
        const float send = upper ? v[e] : v[e + len];
        const float keep = upper ? v[e + len] : v[e];
        v[e] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    // lane m < 16: y of row m -> its delta; lane 16 + m: z of row m
    const float dl = lane < kR ? sm.u[par][warp + lane * kWarps] - v[0] : 0.f;
    const float dz = __shfl_up_sync(0xffffffffu, dl, kR);  // delta of row lane - 16
#pragma unroll
    for (int m = 0; m < kR; ++m) {
      const int j = warp + m * kWarps;
      const float delta = __shfl_sync(0xffffffffu, dl, m);
      float4 x = X[m];
      x.x = fmaf(delta, ww.x, x.x);
      x.y = fmaf(delta, ww.y, x.y);
      x.z = fmaf(delta, ww.z, x.z);
      x.w = fmaf(delta, ww.w, x.w);
      *reinterpret_cast<float4 *>(S + j * kD128 + c) = x;
    }
    if (lane >= kR)
      stf<Tin>(P.o, tokh * kD128 + warp + (lane - kR) * kWarps, P.q_scale * fmaf(dz, wq, v[0]));
    // hand the buffer back: generic writes -> async proxy, then one arrive per warp
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
    cur = nxt;
  }
}

__global__ void selftest_wait_kernel(long long limit_ns, int *err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the phase never completes.
  if (threadIdx.x == 0 && !mbar_wait_timed(&bar, 0, (uint64_t)limit_ns)) record_error(err, PDN_ERR_TIMEOUT);
}

}  // namespace

static int g_num_sms[64];

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!g_num_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

cudaError_t launch_decode(const KParams &P, cudaStream_t stream) {
  const long long grid = (long long)P.B * P.H;
  if (grid <= 0) return cudaSuccess;
  if (P.dk == kD128 && P.dv == kD128) {
    const int items = (int)grid;
    const int ctas = items < num_sms() ? items : num_sms();
    const size_t smem = sizeof(DecSmem);
    cudaError_t e;
    if (P.dtype == PDN_F32) {
      e = cudaFuncSetAttribute(decode_tma_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_tma_kernel<float><<<ctas, kTmaThreads, smem, stream>>>(P, items);
    } else {
      e = cudaFuncSetAttribute(decode_tma_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_tma_kernel<__nv_bfloat16><<<ctas, kTmaThreads, smem, stream>>>(P, items);
    }
    return cudaGetLastError();
  }
  if (P.dtype == PDN_F32)
    decode_kernel<float><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  else
    decode_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(long long limit_ns, int *err, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace pdn
