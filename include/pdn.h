/*
 * pdn.h -- C ABI of the B200 (sm_100a) gated delta-rule forward library.
 *
 * The operation is the forward pass of the gated delta-rule linear
 * recurrence in its generic form (state S is d_v x d_k, o_t = S_t q_t):
 *
 *   S_t = S_{t-1} Diag(alpha_t) (I - r_t w_t^T) + u_t w_t^T,   o_t = q_scale S_t q_t
 *
 * with read key r, write key w and target u chosen per variant:
 *   DN / GDN / KDA      r = k,          w = beta k,          u = v
 *       (DeltaNet; scalar decay = Gated DeltaNet; channel decay = Kimi Delta
 *        Attention -- "Gated DeltaNet-2", ja §1, reductions paragraph)
 *   PDN / PGDN / PKDA   r = k,          w = beta (B_t . k),  u = v
 *       (apply-to-key diagonal preconditioner: A_t = A_{t-1} + k_t . k_t,
 *        B_t = x^(-s), s = c/(1+|c|), c = log(A_t + eps) - mean_i log(A_ti + eps)
 *        -- "Preconditioned DeltaNet", ja §2.2, fr §2.B-C, "Eq. 9")
 *   FG2_GDN             r = sqrt(b).k,  w = sqrt(b).k,       u = sqrt(b).v
 *       (per-channel gain vector b, needs d_k == d_v -- "FG2-GDN", ja §2.1)
 *   GDN2                r = e.k,        w = k,               u = g.v
 *       (decoupled key-side erase gate e and value-side write gate g --
 *        "Gated DeltaNet-2", ja §1 "Gated Delta Rule-2"; the page prints the
 *        transposed d_k x d_v state)
 *   PLA                 r = 0,          w = beta k,          u = v,
 *                       read-out o_t = q_scale S_t (B_t . q_t)
 *       (preconditioned linear attention: the diagonal preconditioner B_t of
 *        PDN applied to the query, apply-to-query; linear attention does not
 *        erase -- "Preconditioned DeltaNet", ja §2.1, fr §2.A)
 *   FG2_GDN_PLUS        r = sqrt(bk).k, w = sqrt(bk).k,      u = sqrt(bv).v
 *       (separate key-side and value-side gain vectors bk, bv -- "FG2-GDN",
 *        ja §2.2; the page prints no formula: this reading reduces to FG2_GDN
 *        at bk = bv)
 * The chunked forward evaluates the same result through the chunkwise WY/UT
 * form the pages describe ("Gated DeltaNet-2", ja §3; "Preconditioned
 * DeltaNet", ja §2.3). The decode step advances one token with the state
 * carried between calls (constant-memory decoding, "Gated DeltaNet-2", ja,
 * problem statement).
 *
 * Conventions (all entry points):
 *   - Every tensor pointer is a DEVICE pointer (except the `host` set of
 *     pdn_chunk_fwd_host), contiguous, 16-byte aligned, owned by the caller;
 *     the library allocates no device memory per call.
 *   - Layouts are row-major: q, k [B,T,H,d_k]; v, o [B,T,H,d_v];
 *     S0, ST [B,H,d_v,d_k] fp32; A0, AT [B,H,d_k] fp32.
 *   - Work is enqueued on the caller's CUDA stream (`stream`, a cudaStream_t;
 *     NULL = legacy default stream) and runs asynchronously. Argument errors
 *     are returned synchronously before anything is enqueued; launch errors
 *     are returned as PDN_ERR_CUDA. Errors detected on the device (a bounded
 *     wait that ran out) are recorded in a per-device error word read by
 *     pdn_get_device_error(). No device code traps.
 *   - Device addresses the library looks up once per device (the error word,
 *     the no-alloc scratch array) and the copy streams of pdn_chunk_fwd_host
 *     belong to the device's primary context: the library must not be used
 *     across a cudaDeviceReset() of that device.
 */
#ifndef PDN_H
#define PDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PDN_OK = 0,
  PDN_ERR_INVALID_ARG = 1, /* bad shape, pointer, alignment or variant/gate mix */
  PDN_ERR_UNSUPPORTED = 2, /* valid problem that the library has no kernel for */
  PDN_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  PDN_ERR_TIMEOUT = 4,     /* a bounded device wait ran out (device error word) */
  PDN_ERR_WORKSPACE = 5,   /* workspace pointer NULL or smaller than required */
  PDN_ERR_BOUNDS = 6       /* debug build only (libpdn_debug.so): an index check in
                              a kernel failed; the access was skipped (device
                              error word) */
} pdn_status_t;

/* Variant: the gain / preconditioner axes of the pages' decay-gain-
 * preconditioner-solve taxonomy ("Preconditioned DeltaNet", de §2 "DGPS"). */
typedef enum {
  PDN_VAR_DN = 0,      /* decay must be NONE    */
  PDN_VAR_GDN = 1,     /* decay must be SCALAR  */
  PDN_VAR_KDA = 2,     /* decay must be CHANNEL */
  PDN_VAR_PDN = 3,     /* decay must be NONE    */
  PDN_VAR_PGDN = 4,    /* decay must be SCALAR  */
  PDN_VAR_PKDA = 5,    /* decay must be CHANNEL */
  PDN_VAR_FG2_GDN = 6, /* any decay; needs d_k == d_v */
  PDN_VAR_GDN2 = 7,    /* any decay */
  PDN_VAR_PLA = 8,     /* any decay; preconditioned (takes A0/AT) */
  PDN_VAR_FG2_GDN_PLUS = 9 /* any decay */
} pdn_variant_t;

/* Decay axis: none (alpha = 1), scalar alpha per (token, head), or a
 * per-key-channel alpha vector (KDA, "Gated DeltaNet-2" ja §1: D_t). */
typedef enum { PDN_DECAY_NONE = 0, PDN_DECAY_SCALAR = 1, PDN_DECAY_CHANNEL = 2 } pdn_decay_t;

/* Element type of q, k, v, o and of the per-channel gate tensors. The state
 * and the preconditioner accumulator are always fp32. */
typedef enum { PDN_F32 = 0, PDN_BF16 = 1 } pdn_dtype_t;

/* Kernel selection for pdn_chunk_fwd. TC is the tensor-core (tcgen05) path
 * that runs the intra-chunk work of all chunks at once and then the
 * sequential state pass (needs a workspace; bf16 inputs, d_k = d_v = 128,
 * chunk 64); SIMT is the CUDA-core kernel (any supported shape, fp32
 * arithmetic). AUTO picks TC where it applies, else SIMT. */
typedef enum { PDN_IMPL_AUTO = 0, PDN_IMPL_SIMT = 1, PDN_IMPL_TC = 2 } pdn_impl_t;

/* Fused prologue (pdn_problem_t.prologue, a bit mask): the kernels take raw
 * projections and apply, per token and head, the activations that otherwise
 * run as separate passes before the recurrence (the workloads the pages
 * train use L2-normalised q and k, sigmoid gains and gates, and a softplus
 * or log-sigmoid decay). 0 = inputs are used as given.
 *   PDN_PRO_L2NORM_QK       q and k are divided by their L2 norm over the head
 *                           dimension (norm floored at 1e-12); the
 *                           preconditioner accumulates the normalised k
 *   PDN_PRO_SIGMOID_GATES   beta (scalar or vector), GDN2's erase and write
 *                           gates and FG2_GDN_PLUS's value gain arrive as
 *                           logits x and are used as sigmoid(x)
 *   PDN_PRO_DECAY_SOFTPLUS  log_alpha arrives as x; log alpha = -decay_scale *
 *                           softplus(x) (decay_scale > 0)
 *   PDN_PRO_DECAY_LOGSIGMOID log_alpha arrives as x; log alpha = log sigmoid(x)
 * The two decay bits exclude each other and need a decay (decay != NONE). */
enum {
  PDN_PRO_L2NORM_QK = 1,
  PDN_PRO_SIGMOID_GATES = 2,
  PDN_PRO_DECAY_SOFTPLUS = 4,
  PDN_PRO_DECAY_LOGSIGMOID = 8
};

typedef struct {
  int B, T, H;          /* batch, tokens per sequence, heads; B,H >= 1, T >= 0
                           (T == 0: per-token tensors may be NULL; ST = S0) */
  int d_k, d_v;         /* head dims: multiples of 16, 16..128                 */
  int chunk;            /* chunk length: 16, 32 or 64 (0 = 64)                */
  pdn_variant_t variant;
  pdn_decay_t decay;
  pdn_dtype_t dtype;
  pdn_impl_t impl;
  float q_scale;        /* read-out scale (the pages use 1)                   */
  float precond_x;      /* preconditioner bound x, B_t in [1/x, x]; 1 <= x <= 2 */
  float precond_eps;    /* > 0, added inside the log                          */
  int prologue;         /* PDN_PRO_* bits (0 = none)                          */
  float decay_scale;    /* PDN_PRO_DECAY_SOFTPLUS only: > 0                   */
} pdn_problem_t;

typedef struct {
  const void *q, *k, *v;  /* dtype; [B,T,H,d_k], [B,T,H,d_k], [B,T,H,d_v]        */
  const void *log_alpha;  /* log decay: NULL (NONE) | fp32 [B,T,H] (SCALAR)      */
                          /*            | dtype [B,T,H,d_k] (CHANNEL); values <= 0 */
  const void *beta;       /* gain: fp32 [B,T,H]; FG2_GDN / FG2_GDN_PLUS: dtype     */
                          /*   [B,T,H,d_k] in [0,1] (the key-side gain); GDN2: NULL */
  const void *erase;      /* GDN2 only: dtype [B,T,H,d_k] erase gate, else NULL   */
  const void *write;      /* dtype [B,T,H,d_v]: GDN2's write gate, FG2_GDN_PLUS's */
                          /*   value-side gain in [0,1]; NULL for the others      */
  const float *S0;        /* initial state [B,H,d_v,d_k]; NULL = zeros            */
  float *ST;              /* final state [B,H,d_v,d_k]; NULL = not returned       */
  const float *A0;        /* preconditioner accumulator [B,H,d_k] (PDN/PGDN/PKDA/ */
  float *AT;              /* PLA only, else both NULL); NULL A0 = zeros           */
  void *o;                /* output [B,T,H,d_v], dtype                            */
} pdn_tensors_t;

/* Bytes of caller-provided workspace pdn_chunk_fwd needs for problem p
 * (0 if none; (size_t)-1 if p is invalid). */
size_t pdn_chunk_fwd_workspace(const pdn_problem_t *p);

/* Which path pdn_chunk_fwd runs for problem p: PDN_IMPL_SIMT or PDN_IMPL_TC;
 * -1 if p is invalid or no kernel of the library supports it. Host-only,
 * touches no device. */
int pdn_chunk_fwd_impl(const pdn_problem_t *p);

/* Chunked forward over T tokens (prefill / training forward).
 * Writes o, and ST / AT when non-NULL. S0 may alias ST and A0 may alias AT
 * (in-place continuation). `workspace` must be 256-byte aligned and hold at
 * least pdn_chunk_fwd_workspace(p) bytes (may be NULL when that is 0).
 * Returns PDN_OK once the work is enqueued. */
pdn_status_t pdn_chunk_fwd(const pdn_problem_t *p, const pdn_tensors_t *t,
                           void *workspace, size_t ws_bytes, void *stream);

/* Measurement form of pdn_chunk_fwd: runs the same path on the same
 * arguments, with CUDA events between its kernels, then synchronises
 * `stream` and writes the elapsed milliseconds of each stage to kernel_ms
 * (caller array of at least 3 floats) and their count to *n_kernels:
 * PDN_IMPL_TC gives 3 (key-energy prefix, intra-chunk kernel, state kernel;
 * the first is ~0 for variants without a preconditioner), PDN_IMPL_SIMT 1.
 * Blocking; for benchmarks, not for production calls. */
pdn_status_t pdn_chunk_fwd_profiled(const pdn_problem_t *p, const pdn_tensors_t *t,
                                    void *workspace, size_t ws_bytes, void *stream,
                                    float *kernel_ms, int *n_kernels);

/* Allocation-free chunked forward. The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory for a
 * workspace (code under a framework allocator that owns all device memory,
 * latency-critical loops that cannot afford cudaMalloc's synchronisation,
 * plugins handed only their input and output buffers). It runs the same
 * tensor-core path as pdn_chunk_fwd with PDN_IMPL_TC (p->impl is ignored),
 * using as its workspace a 64 MiB device array built into the library, so it
 * calls no cudaMalloc/cudaFree and no allocating library routine; the caller
 * still passes all inputs and outputs in `t`.
 *   - Limit: problems whose workspace fits 64 MiB, i.e. B * H * ceil(T/64)
 *     <= 809; larger problems return PDN_ERR_WORKSPACE before any launch.
 *     Problems the tensor-core path does not take return PDN_ERR_UNSUPPORTED.
 *   - The array is held by every GPU that loads the library until the
 *     process exits. The first call on a device looks up its device address
 *     (and may load the library's device code): make that first call before
 *     any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; calls that overlap on the GPU (different streams or host
 *     threads) race and must be serialised by the caller. Nothing needs
 *     clearing between calls: every scratch byte a call reads it writes
 *     first.
 *   - The array's device address is cached per device; like the device error
 *     word, it does not survive cudaDeviceReset() (or any other teardown of
 *     the device's primary context): do not use the library across one. */
pdn_status_t pdn_chunk_fwd_noalloc(const pdn_problem_t *p, const pdn_tensors_t *t, void *stream);

/* Chunked forward from host memory, end to end: copies the inputs in, runs
 * pdn_chunk_fwd and copies the outputs out, in `slices` parts so that on the
 * GPU the host-to-device copy of part i + 1, the forward of part i and the
 * device-to-host copy of part i - 1 overlap. Up to B parts cut the batch
 * into contiguous groups (the batch elements are independent chains, so the
 * result is that of one pdn_chunk_fwd over the whole batch); with more parts
 * each sequence is also cut into ceil(slices / B) runs of whole chunks, run
 * in order, each starting from the state (and accumulator) the previous run
 * left in the device ST (AT) -- the forward's own continuation, the same
 * result up to the rounding of the accumulator's sums.
 *   - `dev`: the device tensors of the whole problem, as pdn_chunk_fwd takes
 *     them (they are also the staging buffers). `workspace` as for
 *     pdn_chunk_fwd on the whole problem.
 *   - `host`: host pointers, same layouts; they must be page-locked
 *     (cudaHostAlloc / registered) for the copies to run asynchronously. A
 *     non-NULL host input (q, k, v, gates, S0, A0) is copied in before use, a
 *     non-NULL host output (o, ST, AT) receives the result; a NULL one leaves
 *     that tensor on the device (an input already there, an output kept).
 *     Every non-NULL host pointer needs its device buffer.
 *   - 1 <= slices <= 128, and B x (runs per sequence) <= 128. More parts
 *     than batch elements need the device ST (and AT for the preconditioned
 *     variants). Work is ordered after the work already on `stream`,
 *     and `stream` waits for all of it; the compute runs on `stream`, the
 *     copies on two streams of the library's own, created on first use on
 *     each device together with their events (nothing is created later).
 *   - Calls on one device from several host threads are serialised inside
 *     the call while they enqueue.
 * Returns PDN_OK once everything is enqueued; argument errors are returned
 * before anything is enqueued. */
pdn_status_t pdn_chunk_fwd_host(const pdn_problem_t *p, const pdn_tensors_t *host,
                                const pdn_tensors_t *dev, void *workspace, size_t ws_bytes,
                                int slices, void *stream);

/* ---- Sequence-parallel prefill ("FG2-GDN", ja §4: 32k-token contexts) ----
 * A long sequence can be cut into segments processed on different GPUs. Every
 * update acts on the state by right-multiplication, so a segment maps its
 * start state affinely, S_end = S_start A_seg + B_seg; the three calls below
 * give A_seg, the accumulator's key energy and the composition, and the
 * exchange between GPUs is the caller's (e.g. an all-gather over NCCL):
 *   1. pdn_key_energy on each segment (A0 = NULL), exchange, prefix-sum: the
 *      accumulator at every segment start (preconditioned variants);
 *   2. B_seg = ST of pdn_chunk_fwd(segment, S0 = NULL, A0 = its start);
 *      A_seg = ST of pdn_chunk_transition(segment, A0 = its start);
 *   3. exchange (A_seg, B_seg); S_start of segment g = pdn_state_compose
 *      folded over the segments before it, from the sequence's S0;
 *   4. pdn_chunk_fwd(segment, S0 = S_start, A0 = its start) gives the outputs.
 */

/* Segment transition A_seg = prod_t Diag(alpha_t) (I - r_t w_t^T) over the
 * problem's T tokens, per (batch, head), written to t->ST as [B,H,d_k,d_k]
 * fp32: the chunked forward with zero targets from the identity state. Needs
 * d_v == d_k; t->S0 must be NULL; t->v and t->o are not used (may be NULL);
 * everything else (gates, A0/AT, workspace, impl) as for pdn_chunk_fwd. */
pdn_status_t pdn_chunk_transition(const pdn_problem_t *p, const pdn_tensors_t *t,
                                  void *workspace, size_t ws_bytes, void *stream);

/* Key energy: t->AT = t->A0 + sum_t k_t . k_t over the problem's T tokens,
 * [B,H,d_k] fp32 (A0 NULL = zeros; k L2-normalised first under
 * PDN_PRO_L2NORM_QK). Uses p's shape, dtype and prologue and t->k, A0, AT. */
pdn_status_t pdn_key_energy(const pdn_problem_t *p, const pdn_tensors_t *t, void *stream);

/* State composition: S_out = S_in A + B_add for each of BH (batch, head)
 * pairs, fp32: S_in, B_add, S_out [BH, d_v, d_k], A [BH, d_k, d_k]. S_in and
 * B_add may be NULL (zero); S_out may alias B_add but not S_in or A. */
pdn_status_t pdn_state_compose(int BH, int d_v, int d_k, const float *S_in, const float *A,
                               const float *B_add, float *S_out, void *stream);

/* out[i] = base[i] + sum_{g < n} parts[g * len + i], fp32 (base may be NULL =
 * zero; out may alias base, not parts): the accumulator at the start of
 * segment n from the gathered key energies of the segments before it. */
pdn_status_t pdn_accumulate(int n, long long len, const float *parts, const float *base,
                            float *out, void *stream);

/* One decode step: p->T must be 1. The state and, for preconditioned
 * variants, the accumulator are updated IN PLACE: pass S0 == ST (non-NULL)
 * and A0 == AT (non-NULL for PDN/PGDN/PKDA, NULL otherwise). */
pdn_status_t pdn_decode_step(const pdn_problem_t *p, const pdn_tensors_t *t, void *stream);

/* ---- Backward ("Gated DeltaNet-2", ja §3, the gate-aware backward) ------
 * Gradient of pdn_chunk_fwd's outputs (o, ST) with respect to its inputs,
 * for every variant and decay. Reverse mode of the token recurrence: two
 * sweeps over the state rows (delta_t forward, d delta_t backward), two over
 * the key columns (dq', dr forward, dw backward), a suffix sum over tokens
 * for the decay and the preconditioner, and per-token chain rules (the erase
 * and write gates receive k . dr and v . du). fp32 arithmetic on CUDA cores;
 * no per-token state is stored. Gradients are fp32, laid out like the inputs
 * they belong to; every pointer may be NULL (that gradient is not written)
 * except that a gradient must be NULL when its input is (dlog_alpha for
 * decay NONE, dbeta for GDN2, derase except for GDN2, dwrite except for GDN2
 * and FG2_GDN_PLUS, dA0 except for the preconditioned variants). Each
 * tensor is 16-byte aligned (4 bytes for the fp32 [B,T,H] ones). */
typedef struct {
  const void *dO;     /* cotangent of o: dtype [B,T,H,d_v]; NULL = zeros       */
  const float *dST;   /* cotangent of ST: [B,H,d_v,d_k]; NULL = zeros          */
  float *dq, *dk;     /* [B,T,H,d_k]                                          */
  float *dv;          /* [B,T,H,d_v]                                          */
  float *dlog_alpha;  /* [B,T,H] (SCALAR) or [B,T,H,d_k] (CHANNEL)            */
  float *dbeta;       /* [B,T,H], or [B,T,H,d_k] for FG2_GDN / FG2_GDN_PLUS     */
  float *derase;      /* GDN2: [B,T,H,d_k]                                    */
  float *dwrite;      /* GDN2 / FG2_GDN_PLUS: [B,T,H,d_v]                      */
  float *dS0;         /* [B,H,d_v,d_k]                                        */
  float *dA0;         /* preconditioned variants: [B,H,d_k]                   */
} pdn_grads_t;

/* Bytes of workspace pdn_chunk_bwd needs ((size_t)-1 if p is invalid). */
size_t pdn_chunk_bwd_workspace(const pdn_problem_t *p);

/* Backward of pdn_chunk_fwd for problem p and forward inputs t (q, k, v,
 * log_alpha, beta, erase, write, S0, A0 as given to the forward; o, ST and
 * AT are not used and may be NULL). p->chunk and p->impl are validated as
 * for the forward but do not change the result. With a fused prologue
 * (p->prologue, as for the forward) the inputs are the raw projections and
 * the gradients are with respect to them: through the L2 normalisation of
 * q and k, the sigmoid of the gains and gates, and the softplus or
 * log-sigmoid of the decay. The gradients overwrite the buffers in g.
 * `workspace`: 256-byte aligned, at least pdn_chunk_bwd_workspace(p) bytes.
 * Returns PDN_OK once the work is enqueued on `stream`. */
pdn_status_t pdn_chunk_bwd(const pdn_problem_t *p, const pdn_tensors_t *t, const pdn_grads_t *g,
                           void *workspace, size_t ws_bytes, void *stream);

/* Training mode ("Gated DeltaNet-2", ja §3: the chunkwise form's Delta = U~ -
 * Y~ S^T holds every token's delta_t = u_t - S_{t-1} D_t r_t). The
 * tensor-core forward can leave, besides o, ST and AT, what the backward's
 * forward sweep would otherwise recompute: every token's delta_t and the
 * state at the start of every 64-token chunk. pdn_chunk_bwd_saved then
 * skips that sweep. The saved values carry the forward's bf16-operand
 * rounding, so these gradients meet the bf16 bar (normalised error 2e-2),
 * not the fp32 backward's; the decay gradient, a sum over the rest of the
 * sequence, gathers most of it and grows with T (measured 1.8e-2 at
 * T = 32768), so pdn_chunk_bwd stays the choice where it must be exact.
 *   - `delta`: fp32 [B,H,T,d_v]; `ckpt`: fp32 [B,H,ceil(T/64),d_k,d_v],
 *     the state S (d_v x d_k) before each chunk's first token stored
 *     transposed (ckpt[..][c][i][j] = S[j][i]); device pointers, 16-byte
 *     aligned, written by pdn_chunk_fwd_save.
 *   - Only problems the tensor-core path takes (pdn_chunk_fwd_impl ==
 *     PDN_IMPL_TC, p->impl not SIMT; T >= 1); others: PDN_ERR_UNSUPPORTED.
 * pdn_chunk_fwd_save: as pdn_chunk_fwd (same arguments and checks), also
 * writing delta and ckpt.
 * pdn_chunk_bwd_saved: as pdn_chunk_bwd for the same problem and inputs,
 * from the saved delta and ckpt and the forward's final state t->ST
 * (required). */
pdn_status_t pdn_chunk_fwd_save(const pdn_problem_t *p, const pdn_tensors_t *t, float *delta,
                                float *ckpt, void *workspace, size_t ws_bytes, void *stream);
pdn_status_t pdn_chunk_bwd_saved(const pdn_problem_t *p, const pdn_tensors_t *t,
                                 const pdn_grads_t *g, const float *delta, const float *ckpt,
                                 void *workspace, size_t ws_bytes, void *stream);

/* Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (PDN_OK if none) and clears it. */
pdn_status_t pdn_get_device_error(void *stream);

/* Self-test of the bounded-wait mechanism every device wait uses: launches
 * one block that waits on an mbarrier nothing arrives on, giving up after
 * `limit_ns` nanoseconds of device time (0 <= limit_ns <= 1e10). The kernel
 * records PDN_ERR_TIMEOUT in the device error word and returns; the host
 * reads it with pdn_get_device_error(). The library's own waits give up after
 * two seconds. */
pdn_status_t pdn_selftest_bounded_wait(long long limit_ns, void *stream);

/* Human-readable name of a status code (static storage). */
const char *pdn_status_string(pdn_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* PDN_H */
