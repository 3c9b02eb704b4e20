// host_pipeline.cu -- pdn_chunk_fwd_host: the chunked forward from host
// memory with the copies overlapped with the compute.
//
// The (batch, head) chains are independent ("Gated DeltaNet-2", ja, problem
// statement: one fixed-size state per sequence), so the batch can be cut into
// contiguous parts that each run as a pdn_chunk_fwd of their own. Part i's
// inputs go in on one copy stream, its forward runs on the caller's stream
// once they have landed, and its outputs go out on a second copy stream once
// the forward is done: on the GPU the copy in of part i + 1, the forward of
// part i and the copy out of part i - 1 run at the same time (PCIe moves
// both directions at once).
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSlices = 64;

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

// Bytes per batch element of each tensor (0 for one the problem does not take).
struct Sizes {
  size_t q, k, v, o, la, beta, erase, write, S, A;
};
Sizes sizes_of(const pdn_problem_t *p) {
  const size_t es = p->dtype == PDN_F32 ? 4 : 2;
  const size_t th = (size_t)p->T * p->H;
  Sizes z;
  z.q = z.k = th * p->d_k * es;
  z.v = z.o = th * p->d_v * es;
  z.la = p->decay == PDN_DECAY_SCALAR ? th * 4 : p->decay == PDN_DECAY_CHANNEL ? th * p->d_k * es : 0;
  z.beta = p->variant == PDN_VAR_GDN2 ? 0 : has_scalar_beta(p->variant) ? th * 4 : th * p->d_k * es;
  z.erase = p->variant == PDN_VAR_GDN2 ? th * p->d_k * es : 0;
  z.write = (p->variant == PDN_VAR_GDN2 || p->variant == PDN_VAR_FG2_GDN_PLUS) ? th * p->d_v * es : 0;
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

// Host -> device copy of `n` batch elements starting at element b0.
cudaError_t copy_in(void *dst, const void *src, size_t per, int b0, int n, cudaStream_t s) {
  if (!src || per == 0 || n == 0) return cudaSuccess;
  return cudaMemcpyAsync(offset(dst, per * b0), offset(src, per * b0), per * n,
                         cudaMemcpyHostToDevice, s);
}
cudaError_t copy_out(void *dst, const void *src, size_t per, int b0, int n, cudaStream_t s) {
  if (!dst || per == 0 || n == 0) return cudaSuccess;
  return cudaMemcpyAsync(offset(dst, per * b0), offset(src, per * b0), per * n,
                         cudaMemcpyDeviceToHost, s);
}


using namespace pdn;

// The problem and device tensors of slice [b0, b0 + n) of the batch.
void slice_of(const pdn_problem_t *p, const pdn_tensors_t *dev, const Sizes &z, int b0, int n,
              pdn_problem_t *pi, pdn_tensors_t *ti) {
  *pi = *p;
  pi->B = n;
  ti->q = offset(dev->q, z.q * b0);
  ti->k = offset(dev->k, z.k * b0);
  ti->v = offset(dev->v, z.v * b0);
  ti->log_alpha = offset(dev->log_alpha, z.la * b0);
  ti->beta = offset(dev->beta, z.beta * b0);
  ti->erase = offset(dev->erase, z.erase * b0);
  ti->write = offset(dev->write, z.write * b0);
  ti->S0 = static_cast<const float *>(offset(dev->S0, z.S * b0));
  ti->ST = static_cast<float *>(offset(dev->ST, z.S * b0));
  ti->A0 = static_cast<const float *>(offset(dev->A0, z.A * b0));
  ti->AT = static_cast<float *>(offset(dev->AT, z.A * b0));
  ti->o = offset(dev->o, z.o * b0);
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
  if (slices < 1 || slices > p->B || slices > kMaxSlices) return PDN_ERR_INVALID_ARG;
  if (ws_bytes < need || (need > 0 && !workspace)) return PDN_ERR_WORKSPACE;
  // a device buffer wherever there is a host one (a device buffer without a
  // host one stays on the device: an input already there, an output kept)
  const void *hs[] = {host->q, host->k, host->v, host->o, host->log_alpha, host->beta,
                      host->erase, host->write, host->S0, host->ST, host->A0, host->AT};
  const void *ds[] = {dev->q, dev->k, dev->v, dev->o, dev->log_alpha, dev->beta,
                      dev->erase, dev->write, dev->S0, dev->ST, dev->A0, dev->AT};
  for (int i = 0; i < 12; ++i)
    if (hs[i] && !ds[i]) return PDN_ERR_INVALID_ARG;
  // the whole problem and every slice's forward must pass pdn_chunk_fwd's
  // checks before anything is enqueued
  pdn_status_t st = pdn::check_chunk_fwd(p, dev, workspace, ws_bytes, nullptr);
  if (st != PDN_OK) return st;
  const Sizes z = sizes_of(p);
  for (int i = 0; i < slices; ++i) {
    const int b0 = (int)((long long)p->B * i / slices);
    const int b1 = (int)((long long)p->B * (i + 1) / slices);
    pdn_problem_t pi;
    pdn_tensors_t ti;
    slice_of(p, dev, z, b0, b1 - b0, &pi, &ti);
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

  st = PDN_OK;
  for (int i = 0; i < slices && st == PDN_OK; ++i) {
    const int b0 = (int)((long long)p->B * i / slices);
    const int b1 = (int)((long long)p->B * (i + 1) / slices);
    const int n = b1 - b0;
    // inputs of part i
    e = copy_in(const_cast<void *>(dev->q), host->q, z.q, b0, n, hp.in);
    if (e == cudaSuccess) e = copy_in(const_cast<void *>(dev->k), host->k, z.k, b0, n, hp.in);
    if (e == cudaSuccess) e = copy_in(const_cast<void *>(dev->v), host->v, z.v, b0, n, hp.in);
    if (e == cudaSuccess)
      e = copy_in(const_cast<void *>(dev->log_alpha), host->log_alpha, z.la, b0, n, hp.in);
    if (e == cudaSuccess) e = copy_in(const_cast<void *>(dev->beta), host->beta, z.beta, b0, n, hp.in);
    if (e == cudaSuccess)
      e = copy_in(const_cast<void *>(dev->erase), host->erase, z.erase, b0, n, hp.in);
    if (e == cudaSuccess)
      e = copy_in(const_cast<void *>(dev->write), host->write, z.write, b0, n, hp.in);
    if (e == cudaSuccess)
      e = copy_in(const_cast<float *>(dev->S0), host->S0, z.S, b0, n, hp.in);
    if (e == cudaSuccess)
      e = copy_in(const_cast<float *>(dev->A0), host->A0, z.A, b0, n, hp.in);
    if (e == cudaSuccess) e = cudaEventRecord(hp.landed[i], hp.in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, hp.landed[i], 0);
    if (e != cudaSuccess) { st = PDN_ERR_CUDA; break; }
    // forward of part i on the caller's stream
    pdn_problem_t pi;
    pdn_tensors_t ti;
    slice_of(p, dev, z, b0, n, &pi, &ti);
    st = pdn_chunk_fwd(&pi, &ti, workspace, ws_bytes, stream);
    if (st != PDN_OK) break;
    if (cudaEventRecord(hp.computed[i], s0) != cudaSuccess) { st = PDN_ERR_CUDA; break; }
    // outputs of part i
    e = cudaStreamWaitEvent(hp.out, hp.computed[i], 0);
    if (e == cudaSuccess) e = copy_out(host->o, dev->o, z.o, b0, n, hp.out);
    if (e == cudaSuccess) e = copy_out(host->ST, dev->ST, z.S, b0, n, hp.out);
    if (e == cudaSuccess) e = copy_out(host->AT, dev->AT, z.A, b0, n, hp.out);
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
