// api.cu -- the C ABI declared in include/pdn.h: argument validation, kernel
// selection and the per-device error word. No device memory is allocated.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pdn {
namespace {

// First device-side error recorded by any kernel of this library (0 = none).
// One instance per device that loads the library.
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int *g_err_ptr[kMaxDevices];
std::mutex g_err_mu;

int *device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int *>(p);
  }
  return g_err_ptr[dev];
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

bool head_dim_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

pdn_decay_t required_decay(pdn_variant_t v, bool *fixed) {
  *fixed = true;
  switch (v) {
    case PDN_VAR_DN: case PDN_VAR_PDN: return PDN_DECAY_NONE;
    case PDN_VAR_GDN: case PDN_VAR_PGDN: return PDN_DECAY_SCALAR;
    case PDN_VAR_KDA: case PDN_VAR_PKDA: return PDN_DECAY_CHANNEL;
    default: *fixed = false; return PDN_DECAY_NONE;
  }
}

// Shape / scalar checks shared by every entry point.
pdn_status_t check_problem(const pdn_problem_t *p) {
  if (!p) return PDN_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->T < 0) return PDN_ERR_INVALID_ARG;
  if (!head_dim_ok(p->d_k) || !head_dim_ok(p->d_v)) return PDN_ERR_INVALID_ARG;
  const int chunk = p->chunk == 0 ? 64 : p->chunk;
  if (chunk != 16 && chunk != 32 && chunk != 64) return PDN_ERR_INVALID_ARG;
  if ((int)p->variant < PDN_VAR_DN || (int)p->variant > PDN_VAR_FG2_GDN_PLUS) return PDN_ERR_INVALID_ARG;
  if ((int)p->decay < PDN_DECAY_NONE || (int)p->decay > PDN_DECAY_CHANNEL) return PDN_ERR_INVALID_ARG;
  if (p->dtype != PDN_F32 && p->dtype != PDN_BF16) return PDN_ERR_INVALID_ARG;
  if ((int)p->impl < PDN_IMPL_AUTO || (int)p->impl > PDN_IMPL_TC) return PDN_ERR_INVALID_ARG;
  bool fixed;
  const pdn_decay_t need = required_decay(p->variant, &fixed);
  if (fixed && p->decay != need) return PDN_ERR_INVALID_ARG;
  if (p->variant == PDN_VAR_FG2_GDN && p->d_k != p->d_v) return PDN_ERR_INVALID_ARG;
  if (!isfinite(p->q_scale)) return PDN_ERR_INVALID_ARG;
  const int pro_all = PDN_PRO_L2NORM_QK | PDN_PRO_SIGMOID_GATES | PDN_PRO_DECAY_SOFTPLUS |
                      PDN_PRO_DECAY_LOGSIGMOID;
  if (p->prologue & ~pro_all) return PDN_ERR_INVALID_ARG;
  const int pro_decay = p->prologue & (PDN_PRO_DECAY_SOFTPLUS | PDN_PRO_DECAY_LOGSIGMOID);
  if (pro_decay == (PDN_PRO_DECAY_SOFTPLUS | PDN_PRO_DECAY_LOGSIGMOID)) return PDN_ERR_INVALID_ARG;
  if (pro_decay && p->decay == PDN_DECAY_NONE) return PDN_ERR_INVALID_ARG;
  if ((p->prologue & PDN_PRO_DECAY_SOFTPLUS) && !(p->decay_scale > 0.f && isfinite(p->decay_scale)))
    return PDN_ERR_INVALID_ARG;
  if (is_precond(p->variant)) {
    if (!(p->precond_x >= 1.0f && p->precond_x <= 2.0f)) return PDN_ERR_INVALID_ARG;
    if (!(p->precond_eps > 0.0f) || !isfinite(p->precond_eps)) return PDN_ERR_INVALID_ARG;
  }
  // flattened grids and 64-bit element offsets
  const long long units = (long long)p->B * p->H * ((p->d_v + 31) / 32);
  if (units > 0x7fffffffLL) return PDN_ERR_INVALID_ARG;
  return PDN_OK;
}

pdn_status_t check_tensors(const pdn_problem_t *p, const pdn_tensors_t *t, bool need_o = true) {
  if (!t) return PDN_ERR_INVALID_ARG;
  // 16-byte alignment for every tensor the kernels read or write in 16-byte
  // vectors; the fp32 per-(token, head) gates (scalar log decay, scalar beta)
  // are read one element at a time and need only 4
  const bool scalar_la = p->decay == PDN_DECAY_SCALAR;
  const bool scalar_beta = has_scalar_beta(p->variant);
  const void *v16[] = {t->q, t->k, t->v, t->o, t->erase, t->write, t->S0, t->ST, t->A0, t->AT,
                       scalar_la ? nullptr : t->log_alpha, scalar_beta ? nullptr : t->beta};
  for (const void *ptr : v16)
    if (ptr && !aligned(ptr, 16)) return PDN_ERR_INVALID_ARG;
  if (scalar_la && t->log_alpha && !aligned(t->log_alpha, 4)) return PDN_ERR_INVALID_ARG;
  if (scalar_beta && t->beta && !aligned(t->beta, 4)) return PDN_ERR_INVALID_ARG;
  // With T == 0 the per-token tensors are empty and may be NULL; nothing
  // reads them.
  if (p->T == 0) {
    if (p->variant == PDN_VAR_GDN2 && t->beta) return PDN_ERR_INVALID_ARG;
  } else {
    if (!t->q || !t->k || !t->v || (need_o && !t->o)) return PDN_ERR_INVALID_ARG;
    if ((p->decay == PDN_DECAY_NONE) != (t->log_alpha == nullptr)) return PDN_ERR_INVALID_ARG;
    if (p->variant == PDN_VAR_GDN2) {
      if (t->beta || !t->erase || !t->write) return PDN_ERR_INVALID_ARG;
    } else if (p->variant == PDN_VAR_FG2_GDN_PLUS) {
      if (!t->beta || t->erase || !t->write) return PDN_ERR_INVALID_ARG;
    } else {
      if (!t->beta || t->erase || t->write) return PDN_ERR_INVALID_ARG;
    }
  }
  if (!is_precond(p->variant) && (t->A0 || t->AT)) return PDN_ERR_INVALID_ARG;
  return PDN_OK;
}

KParams make_params(const pdn_problem_t *p, const pdn_tensors_t *t, int *err) {
  KParams P;
  memset(&P, 0, sizeof(P));
  P.B = p->B; P.T = p->T; P.H = p->H; P.dk = p->d_k; P.dv = p->d_v;
  P.chunk = p->chunk == 0 ? 64 : p->chunk;
  P.variant = p->variant; P.decay = p->decay; P.dtype = p->dtype;
  P.q_scale = p->q_scale;
  P.prologue = p->prologue;
  P.decay_scale = p->decay_scale;
  P.x = is_precond(p->variant) ? p->precond_x : 1.0f;
  P.lnx = logf(P.x);
  P.eps = is_precond(p->variant) ? p->precond_eps : 1.0f;
  P.q = t->q; P.k = t->k; P.v = t->v; P.log_alpha = t->log_alpha; P.beta = t->beta;
  P.erase = t->erase; P.write = t->write;
  P.S0 = t->S0; P.ST = t->ST; P.A0 = t->A0; P.AT = t->AT; P.o = t->o;
  P.err = err;
  return P;
}

// The path pdn_chunk_fwd takes, or -1 when the requested one cannot run.
int select_impl(const pdn_problem_t *p, const KParams &P) {
  switch (p->impl) {
    case PDN_IMPL_SIMT: return simt_supported(P) ? PDN_IMPL_SIMT : -1;
    case PDN_IMPL_TC: return split_supported(P) ? PDN_IMPL_TC : -1;
    default:
      if (split_supported(P)) return PDN_IMPL_TC;
      return simt_supported(P) ? PDN_IMPL_SIMT : -1;
  }
}

size_t workspace_for(int impl, const KParams &P) {
  return impl == PDN_IMPL_TC ? split_workspace_bytes(P) : 0;
}

}  // namespace

// Everything pdn_chunk_fwd checks before it enqueues work (host-only).
pdn_status_t check_chunk_fwd(const pdn_problem_t *p, const pdn_tensors_t *t,
                             const void *workspace, size_t ws_bytes, int *impl_out) {
  pdn_status_t st = check_problem(p);
  if (st != PDN_OK) return st;
  if ((st = check_tensors(p, t)) != PDN_OK) return st;
  const KParams P = make_params(p, t, nullptr);
  const int impl = select_impl(p, P);
  if (impl < 0) return PDN_ERR_UNSUPPORTED;
  const size_t need = workspace_for(impl, P);
  if (need > 0) {
    if (!workspace || ws_bytes < need || ((uintptr_t)workspace & 255u)) return PDN_ERR_WORKSPACE;
  }
  if (impl_out) *impl_out = impl;
  return PDN_OK;
}

// Everything pdn_chunk_bwd checks before it enqueues work (host-only).
pdn_status_t check_chunk_bwd(const pdn_problem_t *p, const pdn_tensors_t *t, const pdn_grads_t *g,
                             const void *workspace, size_t ws_bytes) {
  pdn_status_t st = check_problem(p);
  if (st != PDN_OK) return st;
  if ((st = check_tensors(p, t, false)) != PDN_OK) return st;
  if (!g) return PDN_ERR_INVALID_ARG;
  const bool scalar_la = p->decay == PDN_DECAY_SCALAR;
  const bool scalar_beta = has_scalar_beta(p->variant);
  const void *v16[] = {g->dO, g->dST, g->dq, g->dk, g->dv, g->derase, g->dwrite, g->dS0, g->dA0,
                       scalar_la ? nullptr : g->dlog_alpha, scalar_beta ? nullptr : g->dbeta};
  for (const void *ptr : v16)
    if (ptr && !aligned(ptr, 16)) return PDN_ERR_INVALID_ARG;
  if (scalar_la && g->dlog_alpha && !aligned(g->dlog_alpha, 4)) return PDN_ERR_INVALID_ARG;
  if (scalar_beta && g->dbeta && !aligned(g->dbeta, 4)) return PDN_ERR_INVALID_ARG;
  // a gradient only where the forward has the input
  if (p->decay == PDN_DECAY_NONE && g->dlog_alpha) return PDN_ERR_INVALID_ARG;
  if (p->variant == PDN_VAR_GDN2 && g->dbeta) return PDN_ERR_INVALID_ARG;
  if (p->variant != PDN_VAR_GDN2 && g->derase) return PDN_ERR_INVALID_ARG;
  if (p->variant != PDN_VAR_GDN2 && p->variant != PDN_VAR_FG2_GDN_PLUS && g->dwrite)
    return PDN_ERR_INVALID_ARG;
  if (!is_precond(p->variant) && g->dA0) return PDN_ERR_INVALID_ARG;
  const KParams P = make_params(p, t, nullptr);
  if (p->T > 0 && (!workspace || ws_bytes < bwd_workspace_bytes(P) || ((uintptr_t)workspace & 255u)))
    return PDN_ERR_WORKSPACE;
  return PDN_OK;
}

}  // namespace pdn

using namespace pdn;

extern "C" size_t pdn_chunk_fwd_workspace(const pdn_problem_t *p) {
  if (check_problem(p) != PDN_OK) return (size_t)-1;
  pdn_tensors_t dummy;
  memset(&dummy, 0, sizeof(dummy));
  const KParams P = make_params(p, &dummy, nullptr);
  const int impl = select_impl(p, P);
  return impl < 0 ? 0 : workspace_for(impl, P);
}

extern "C" int pdn_chunk_fwd_impl(const pdn_problem_t *p) {
  if (check_problem(p) != PDN_OK) return -1;
  pdn_tensors_t dummy;
  memset(&dummy, 0, sizeof(dummy));
  const KParams P = make_params(p, &dummy, nullptr);
  return select_impl(p, P);
}

extern "C" pdn_status_t pdn_chunk_fwd(const pdn_problem_t *p, const pdn_tensors_t *t,
                                      void *workspace, size_t ws_bytes, void *stream) {
  int impl = -1;
  const pdn_status_t st = check_chunk_fwd(p, t, workspace, ws_bytes, &impl);
  if (st != PDN_OK) return st;
  KParams P = make_params(p, t, nullptr);
  P.err = device_error_word();
  if (!P.err) return PDN_ERR_CUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (impl == PDN_IMPL_TC) e = launch_chunk_split(P, workspace, s);
  else e = launch_chunk_simt(P, s);
  return e == cudaSuccess ? PDN_OK : PDN_ERR_CUDA;
}

extern "C" size_t pdn_chunk_bwd_workspace(const pdn_problem_t *p) {
  if (check_problem(p) != PDN_OK) return (size_t)-1;
  pdn_tensors_t dummy;
  memset(&dummy, 0, sizeof(dummy));
  return p->T == 0 ? 0 : bwd_workspace_bytes(make_params(p, &dummy, nullptr));
}

extern "C" pdn_status_t pdn_chunk_bwd(const pdn_problem_t *p, const pdn_tensors_t *t,
                                      const pdn_grads_t *g, void *workspace, size_t ws_bytes,
                                      void *stream) {
  const pdn_status_t st = check_chunk_bwd(p, t, g, workspace, ws_bytes);
  if (st != PDN_OK) return st;
  KParams P = make_params(p, t, nullptr);
  P.err = device_error_word();
  if (!P.err) return PDN_ERR_CUDA;
  return launch_chunk_bwd(P, g, workspace, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PDN_OK
             : PDN_ERR_CUDA;
}

// Training mode: the forward that also leaves every token's delta and the
// chunk-start states, and the backward that reuses them.
extern "C" pdn_status_t pdn_chunk_fwd_save(const pdn_problem_t *p, const pdn_tensors_t *t,
                                           float *delta, float *ckpt, void *workspace,
                                           size_t ws_bytes, void *stream) {
  int impl = -1;
  const pdn_status_t st = check_chunk_fwd(p, t, workspace, ws_bytes, &impl);
  if (st != PDN_OK) return st;
  if (!delta || !ckpt || !aligned(delta, 16) || !aligned(ckpt, 16)) return PDN_ERR_INVALID_ARG;
  if (impl != PDN_IMPL_TC || p->T == 0) return PDN_ERR_UNSUPPORTED;
  KParams P = make_params(p, t, nullptr);
  P.sv_delta = delta;
  P.sv_ckpt = ckpt;
  P.err = device_error_word();
  if (!P.err) return PDN_ERR_CUDA;
  return launch_chunk_split(P, workspace, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PDN_OK
             : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_chunk_bwd_saved(const pdn_problem_t *p, const pdn_tensors_t *t,
                                            const pdn_grads_t *g, const float *delta,
                                            const float *ckpt, void *workspace, size_t ws_bytes,
                                            void *stream) {
  const pdn_status_t st = check_chunk_bwd(p, t, g, workspace, ws_bytes);
  if (st != PDN_OK) return st;
  if (!delta || !ckpt || !aligned(delta, 16) || !aligned(ckpt, 16) || !t->ST)
    return PDN_ERR_INVALID_ARG;
  KParams P = make_params(p, t, nullptr);
  if (select_impl(p, P) != PDN_IMPL_TC || p->T == 0) return PDN_ERR_UNSUPPORTED;
  P.sv_delta = const_cast<float *>(delta);
  P.sv_ckpt = const_cast<float *>(ckpt);
  P.err = device_error_word();
  if (!P.err) return PDN_ERR_CUDA;
  return launch_chunk_bwd(P, g, workspace, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PDN_OK
             : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_chunk_fwd_profiled(const pdn_problem_t *p, const pdn_tensors_t *t,
                                               void *workspace, size_t ws_bytes, void *stream,
                                               float *kernel_ms, int *n_kernels) {
  if (!kernel_ms || !n_kernels) return PDN_ERR_INVALID_ARG;
  int impl = -1;
  const pdn_status_t st = check_chunk_fwd(p, t, workspace, ws_bytes, &impl);
  if (st != PDN_OK) return st;
  KParams P = make_params(p, t, nullptr);
  P.err = device_error_word();
  if (!P.err) return PDN_ERR_CUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev[4] = {};
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = cudaEventCreate(&ev[i]);
  if (e == cudaSuccess) {
    if (impl == PDN_IMPL_TC) {
      e = launch_chunk_split(P, workspace, s, ev);
    } else {
      e = cudaEventRecord(ev[0], s);
      if (e == cudaSuccess) e = launch_chunk_simt(P, s);
      if (e == cudaSuccess) e = cudaEventRecord(ev[1], s);
    }
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  const int n = impl == PDN_IMPL_TC ? 3 : 1;
  for (int i = 0; i < n && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&kernel_ms[i], ev[i], ev[i + 1]);
  for (int i = 0; i < 4; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  if (e != cudaSuccess) return PDN_ERR_CUDA;
  *n_kernels = n;
  return PDN_OK;
}

extern "C" pdn_status_t pdn_chunk_transition(const pdn_problem_t *p, const pdn_tensors_t *t,
                                             void *workspace, size_t ws_bytes, void *stream) {
  pdn_status_t st = check_problem(p);
  if (st != PDN_OK) return st;
  if (!t || p->d_v != p->d_k || t->S0 || !t->ST) return PDN_ERR_INVALID_ARG;
  // v and o are not used: check the rest with stand-ins of the right alignment
  pdn_tensors_t c = *t;
  if (!c.v) c.v = c.k;
  if (!c.o) c.o = const_cast<void *>(c.k);
  int impl = -1;
  if ((st = check_chunk_fwd(p, &c, workspace, ws_bytes, &impl)) != PDN_OK) return st;
  KParams P = make_params(p, t, device_error_word());
  if (!P.err) return PDN_ERR_CUDA;
  P.transition = 1;
  P.v = nullptr;
  P.o = nullptr;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = impl == PDN_IMPL_TC ? launch_chunk_split(P, workspace, s) : launch_chunk_simt(P, s);
  return e == cudaSuccess ? PDN_OK : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_key_energy(const pdn_problem_t *p, const pdn_tensors_t *t,
                                       void *stream) {
  pdn_status_t st = check_problem(p);
  if (st != PDN_OK) return st;
  if (!t || !t->AT || (p->T > 0 && !t->k)) return PDN_ERR_INVALID_ARG;
  if ((t->k && !aligned(t->k, 16)) || !aligned(t->AT, 16) || (t->A0 && !aligned(t->A0, 16)))
    return PDN_ERR_INVALID_ARG;
  KParams P = make_params(p, t, nullptr);
  return launch_key_energy(P, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PDN_OK
                                                                                 : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_accumulate(int n, long long len, const float *parts,
                                       const float *base, float *out, void *stream) {
  if (n < 0 || len < 0 || !out || (n > 0 && !parts)) return PDN_ERR_INVALID_ARG;
  if (out == parts) return PDN_ERR_INVALID_ARG;
  return launch_accumulate(n, len, parts, base, out, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? PDN_OK
             : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_state_compose(int BH, int d_v, int d_k, const float *S_in,
                                          const float *A, const float *B_add, float *S_out,
                                          void *stream) {
  if (BH < 1 || !head_dim_ok(d_v) || !head_dim_ok(d_k) || !A || !S_out) return PDN_ERR_INVALID_ARG;
  if (S_out == S_in || S_out == A) return PDN_ERR_INVALID_ARG;
  const void *all[] = {S_in, A, B_add, S_out};
  for (const void *ptr : all)
    if (ptr && !aligned(ptr, 16)) return PDN_ERR_INVALID_ARG;
  return launch_compose(BH, d_v, d_k, S_in, A, B_add, S_out, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? PDN_OK
             : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_decode_step(const pdn_problem_t *p, const pdn_tensors_t *t,
                                        void *stream) {
  pdn_status_t st = check_problem(p);
  if (st != PDN_OK) return st;
  if ((st = check_tensors(p, t)) != PDN_OK) return st;
  if (p->T != 1) return PDN_ERR_INVALID_ARG;
  if (!t->ST || t->S0 != t->ST) return PDN_ERR_INVALID_ARG;
  if (is_precond(p->variant) && (!t->AT || t->A0 != t->AT)) return PDN_ERR_INVALID_ARG;
  KParams P = make_params(p, t, device_error_word());
  if (!P.err) return PDN_ERR_CUDA;
  return launch_decode(P, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PDN_OK
                                                                             : PDN_ERR_CUDA;
}

extern "C" pdn_status_t pdn_get_device_error(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PDN_ERR_CUDA;
  int *w = device_error_word();
  if (!w) return PDN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PDN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return PDN_ERR_CUDA;
  return static_cast<pdn_status_t>(v);
}

extern "C" pdn_status_t pdn_selftest_bounded_wait(long long limit_ns, void *stream) {
  if (limit_ns < 0 || limit_ns > 10000000000LL) return PDN_ERR_INVALID_ARG;
  int *w = device_error_word();
  if (!w) return PDN_ERR_CUDA;
  return launch_selftest_wait(limit_ns, w, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PDN_OK : PDN_ERR_CUDA;
}

extern "C" const char *pdn_status_string(pdn_status_t s) {
  switch (s) {
    case PDN_OK: return "PDN_OK";
    case PDN_ERR_INVALID_ARG: return "PDN_ERR_INVALID_ARG";
    case PDN_ERR_UNSUPPORTED: return "PDN_ERR_UNSUPPORTED";
    case PDN_ERR_CUDA: return "PDN_ERR_CUDA";
    case PDN_ERR_TIMEOUT: return "PDN_ERR_TIMEOUT";
    case PDN_ERR_WORKSPACE: return "PDN_ERR_WORKSPACE";
    case PDN_ERR_BOUNDS: return "PDN_ERR_BOUNDS";
  }
  return "PDN_ERR_UNKNOWN";
}
