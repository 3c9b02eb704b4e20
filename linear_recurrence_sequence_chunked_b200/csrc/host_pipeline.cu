// host_pipeline.cu -- pdn_chunk_fwd_host: the chunked forward from host
// memory with the copies overlapped with the compute.
//
// The (batch, head) chains are independent ("Gated DeltaNet-2", ja, problem
// statement: one fixed-size state per sequence), so the batch can be cut into
// contiguous parts that each run as a pdn_chunk_fwd of their own; with more
// parts than batch elements each sequence is also cut into runs of whole
// chunks, run in order, the state (and accumulator) handed from one run to
// the next through ST (AT) -- the forward's own continuation. Part i's inputs
// go in on one copy stream, its forward runs on the caller's stream once they
// have landed, and its outputs go out on a second copy stream once the
// forward is done: on the GPU the copy in of part i + 1, the forward of part
// i and the copy out of part i - 1 run at the same time (PCIe moves both
// directions at once). Smaller parts leave less of the last part's compute
// and copy out exposed.
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSlices = 128;

struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr, done_in = nullptr;
  cudaEvent_t landed[kMaxSlices] = {}, computed[kMaxSlices] = {};
  bool ready = false;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

cudaError_t make_pipe(HostPipe &hp) {
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&hp.done_in, cudaEventDisableTiming)) != cudaSuccess) return e;
  for (int i = 0; i < kMaxSlices; ++i) {
    if ((e = cudaEventCreateWithFlags(&hp.landed[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&hp.computed[i], cudaEventDisableTiming)) != cudaSuccess)
      return e;
  }
  hp.ready = true;
  return cudaSuccess;
}

// Bytes per token of each per-token tensor, and per batch element of the
// state and the accumulator (0 for a tensor the problem does not take).
struct Sizes {
  size_t q, k, v, o, la, beta, erase, write, S, A;
};
Sizes sizes_of(const pdn_problem_t *p) {
  const size_t es = p->dtype == PDN_F32 ? 4 : 2;
  const size_t h = p->H;
  Sizes z;
  z.q = z.k = h * p->d_k * es;
  z.v = z.o = h * p->d_v * es;
  z.la = p->decay == PDN_DECAY_SCALAR ? h * 4 : p->decay == PDN_DECAY_CHANNEL ? h * p->d_k * es : 0;
  z.beta = p->variant == PDN_VAR_GDN2 ? 0 : has_scalar_beta(p->variant) ? h * 4 : h * p->d_k * es;
  z.erase = p->variant == PDN_VAR_GDN2 ? h * p->d_k * es : 0;
  z.write = (p->variant == PDN_VAR_GDN2 || p->variant == PDN_VAR_FG2_GDN_PLUS) ? h * p->d_v * es : 0;
  z.S = (size_t)p->H * p->d_v * p->d_k * 4;
  z.A = (size_t)p->H * p->d_k * 4;
  return z;
}

const void *offset(const void *base, size_t bytes) {
  return base ? static_cast<const uint8_t *>(base) + bytes : nullptr;
}
void *offset(void *base, size_t bytes) {
  return base ? static_cast<uint8_t *>(base) + bytes : nullptr;
}

// One part: batch elements [b0, b0 + nb) over tokens [t0, t1) (the whole
// sequence unless nb == 1); `first` / `last`: it starts / ends its sequences.
struct Part {
  int b0, nb, t0, t1;
  bool first, last;
};

// The parts of a call, in the order they run (the runs of one sequence in
// token order). Returns their number (0: too many for the pipeline).
int plan_parts(const pdn_problem_t *p, int slices, Part *parts) {
  if (slices <= p->B) {
    for (int i = 0; i < slices; ++i) {
      const int b0 = (int)((long long)p->B * i / slices);
      const int b1 = (int)((long long)p->B * (i + 1) / slices);
      parts[i] = Part{b0, b1 - b0, 0, p->T, true, true};
    }
    return slices;
  }
  const int C = p->chunk ? p->chunk : 64;
  const int N = (p->T + C - 1) / C;  // chunks per sequence
  int runs = (slices + p->B - 1) / p->B;
  if (runs > N) runs = N;
  const int L = (N + runs - 1) / runs;  // chunks per run
  runs = (N + L - 1) / L;
  if ((long long)p->B * runs > kMaxSlices) return 0;
  int n = 0;
  for (int b = 0; b < p->B; ++b)
    for (int j = 0; j < runs; ++j) {
      const int t0 = j * L * C, t1 = (j + 1 == runs) ? p->T : (j + 1) * L * C;
      parts[n++] = Part{b, 1, t0, t1, j == 0, j + 1 == runs};
    }
  return n;
}

// Byte offset and length of a part's rows of a per-token tensor.
size_t tok_off(const pdn_problem_t *p, const Part &q, size_t per_tok) {
  return ((size_t)q.b0 * p->T + q.t0) * per_tok;
}
size_t tok_len(const Part &q, size_t per_tok) { return (size_t)q.nb * (q.t1 - q.t0) * per_tok; }

cudaError_t copy_tok(void *dst, const void *src, const pdn_problem_t *p, const Part &q,
                     size_t per_tok, cudaMemcpyKind kind, cudaStream_t s) {
  if (!src || !dst || per_tok == 0 || q.t1 <= q.t0) return cudaSuccess;
  const size_t off = tok_off(p, q, per_tok);
  return cudaMemcpyAsync(offset(dst, off), offset(src, off), tok_len(q, per_tok), kind, s);
}
cudaError_t copy_batch(void *dst, const void *src, const Part &q, size_t per, cudaMemcpyKind kind,
                       cudaStream_t s) {
  if (!src || !dst || per == 0) return cudaSuccess;
  return cudaMemcpyAsync(offset(dst, per * q.b0), offset(src, per * q.b0), per * q.nb, kind, s);
}

// The problem and device tensors of one part. A run after the first starts
// from the state (and accumulator) the previous run left in ST (AT).
void part_of(const pdn_problem_t *p, const pdn_tensors_t *dev, const Sizes &z, const Part &q,
             pdn_problem_t *pi, pdn_tensors_t *ti) {
  *pi = *p;
  pi->B = q.nb;
  pi->T = q.t1 - q.t0;
  ti->q = offset(dev->q, tok_off(p, q, z.q));
  ti->k = offset(dev->k, tok_off(p, q, z.k));
  ti->v = offset(dev->v, tok_off(p, q, z.v));
  ti->log_alpha = offset(dev->log_alpha, tok_off(p, q, z.la));
  ti->beta = offset(dev->beta, tok_off(p, q, z.beta));
  ti->erase = offset(dev->erase, tok_off(p, q, z.erase));
  ti->write = offset(dev->write, tok_off(p, q, z.write));
  ti->o = offset(dev->o, tok_off(p, q, z.o));
  ti->S0 = static_cast<const float *>(q.first ? offset(dev->S0, z.S * q.b0) : offset(dev->ST, z.S * q.b0));
  ti->ST = static_cast<float *>(offset(dev->ST, z.S * q.b0));
  ti->A0 = static_cast<const float *>(q.first ? offset(dev->A0, z.A * q.b0) : offset(dev->AT, z.A * q.b0));
  ti->AT = static_cast<float *>(offset(dev->AT, z.A * q.b0));
}

}  // namespace
}  // namespace pdn

using namespace pdn;

extern "C" pdn_status_t pdn_chunk_fwd_host(const pdn_problem_t *p, const pdn_tensors_t *host,
                                           const pdn_tensors_t *dev, void *workspace,
                                           size_t ws_bytes, int slices, void *stream) {
  if (!p || !host || !dev) return PDN_ERR_INVALID_ARG;
  const size_t need = pdn_chunk_fwd_workspace(p);
  if (need == (size_t)-1) return PDN_ERR_INVALID_ARG;
  if (slices < 1 || slices > kMaxSlices) return PDN_ERR_INVALID_ARG;
  if (ws_bytes < need || (need > 0 && !workspace)) return PDN_ERR_WORKSPACE;
  // a device buffer wherever there is a host one (a device buffer without a
  // host one stays on the device: an input already there, an output kept)
  const void *hs[] = {host->q, host->k, host->v, host->o, host->log_alpha, host->beta,
                      host->erase, host->write, host->S0, host->ST, host->A0, host->AT};
  const void *ds[] = {dev->q, dev->k, dev->v, dev->o, dev->log_alpha, dev->beta,
                      dev->erase, dev->write, dev->S0, dev->ST, dev->A0, dev->AT};
  for (int i = 0; i < 12; ++i)
    if (hs[i] && !ds[i]) return PDN_ERR_INVALID_ARG;
  // the whole problem and every part's forward must pass pdn_chunk_fwd's
  // checks before anything is enqueued
  pdn_status_t st = pdn::check_chunk_fwd(p, dev, workspace, ws_bytes, nullptr);
  if (st != PDN_OK) return st;
  Part parts[kMaxSlices];
  const int np = plan_parts(p, slices, parts);
  if (np < 1) return PDN_ERR_INVALID_ARG;
  // runs of one sequence hand the state on through the device ST (and AT)
  if (np > p->B && (!dev->ST || (is_precond(p->variant) && !dev->AT))) return PDN_ERR_INVALID_ARG;
  const Sizes z = sizes_of(p);
  for (int i = 0; i < np; ++i) {
    pdn_problem_t pi;
    pdn_tensors_t ti;
    part_of(p, dev, z, parts[i], &pi, &ti);
    if ((st = pdn::check_chunk_fwd(&pi, &ti, workspace, ws_bytes, nullptr)) != PDN_OK) return st;
  }

  int devno = 0;
  if (cudaGetDevice(&devno) != cudaSuccess || devno < 0 || devno >= kMaxDevices) return PDN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe &hp = g_pipe[devno];
  if (!hp.ready && make_pipe(hp) != cudaSuccess) return PDN_ERR_CUDA;

  const cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaEventRecord(hp.start, s0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.in, hp.start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.out, hp.start, 0);
  if (e != cudaSuccess) return PDN_ERR_CUDA;

  const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
  st = PDN_OK;
  for (int i = 0; i < np && st == PDN_OK; ++i) {
    const Part &q = parts[i];
    // inputs of part i (the initial state and accumulator with a sequence's first run)
    e = copy_tok(const_cast<void *>(dev->q), host->q, p, q, z.q, h2d, hp.in);
    if (e == cudaSuccess) e = copy_tok(const_cast<void *>(dev->k), host->k, p, q, z.k, h2d, hp.in);
    if (e == cudaSuccess) e = copy_tok(const_cast<void *>(dev->v), host->v, p, q, z.v, h2d, hp.in);
    if (e == cudaSuccess)
      e = copy_tok(const_cast<void *>(dev->log_alpha), host->log_alpha, p, q, z.la, h2d, hp.in);
    if (e == cudaSuccess)
      e = copy_tok(const_cast<void *>(dev->beta), host->beta, p, q, z.beta, h2d, hp.in);
    if (e == cudaSuccess)
      e = copy_tok(const_cast<void *>(dev->erase), host->erase, p, q, z.erase, h2d, hp.in);
    if (e == cudaSuccess)
      e = copy_tok(const_cast<void *>(dev->write), host->write, p, q, z.write, h2d, hp.in);
    if (e == cudaSuccess && q.first)
      e = copy_batch(const_cast<float *>(dev->S0), host->S0, q, z.S, h2d, hp.in);
    if (e == cudaSuccess && q.first)
      e = copy_batch(const_cast<float *>(dev->A0), host->A0, q, z.A, h2d, hp.in);
    if (e == cudaSuccess) e = cudaEventRecord(hp.landed[i], hp.in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, hp.landed[i], 0);
    if (e != cudaSuccess) { st = PDN_ERR_CUDA; break; }
    // forward of part i on the caller's stream
    pdn_problem_t pi;
    pdn_tensors_t ti;
    part_of(p, dev, z, q, &pi, &ti);
    st = pdn_chunk_fwd(&pi, &ti, workspace, ws_bytes, stream);
    if (st != PDN_OK) break;
    if (cudaEventRecord(hp.computed[i], s0) != cudaSuccess) { st = PDN_ERR_CUDA; break; }
    // outputs of part i (the final state and accumulator with a sequence's last run)
    e = cudaStreamWaitEvent(hp.out, hp.computed[i], 0);
    if (e == cudaSuccess) e = copy_tok(host->o, dev->o, p, q, z.o, d2h, hp.out);
    if (e == cudaSuccess && q.last) e = copy_batch(host->ST, dev->ST, q, z.S, d2h, hp.out);
    if (e == cudaSuccess && q.last) e = copy_batch(host->AT, dev->AT, q, z.A, d2h, hp.out);
    if (e != cudaSuccess) st = PDN_ERR_CUDA;
  }
  // the caller's stream waits for everything enqueued, also after an error
  // part-way (nothing may still be copying once the stream has drained)
  e = cudaEventRecord(hp.done, hp.out);
  const cudaError_t e2 = cudaEventRecord(hp.done_in, hp.in);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, hp.done, 0);
  if (e == cudaSuccess) e = e2;
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, hp.done_in, 0);
  if (st != PDN_OK) return st;
  return e == cudaSuccess ? PDN_OK : PDN_ERR_CUDA;
}
