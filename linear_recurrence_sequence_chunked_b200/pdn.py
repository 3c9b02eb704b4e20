"""ctypes binding of ``libpdn.so`` (the C ABI in ``include/pdn.h``).

The functions named like the C entry points (``pdn_chunk_fwd``,
``pdn_decode_step``, ...) only marshal arguments: every step of the
computation runs in the library's CUDA kernels. ``chunk_fwd`` and
``decode_step`` are conveniences that take torch tensors, allocate the outputs
with torch and call those entry points on torch's current stream.

There is no CPU fallback: importing the binding without a built library
raises, and so does calling it on a machine without a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

# The release library; PDN_LIBRARY may name another build of the same ABI
# (libpdn_debug.so: the kernels' index checks compiled in).
_LIB_PATH = os.environ.get("PDN_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libpdn.so")
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpdn_debug.so")

PDN_OK, PDN_ERR_INVALID_ARG, PDN_ERR_UNSUPPORTED, PDN_ERR_CUDA, PDN_ERR_TIMEOUT, \
    PDN_ERR_WORKSPACE, PDN_ERR_BOUNDS = range(7)
VARIANTS = {"DN": 0, "GDN": 1, "KDA": 2, "PDN": 3, "PGDN": 4, "PKDA": 5, "FG2_GDN": 6, "GDN2": 7,
            "PLA": 8, "FG2_GDN_PLUS": 9}
DECAYS = {"none": 0, "scalar": 1, "channel": 2}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
IMPLS = {"auto": 0, "simt": 1, "tc": 2}
PRECOND_VARIANTS = ("PDN", "PGDN", "PKDA", "PLA")
# fused prologue bits (pdn_problem_t.prologue)
PRO_L2NORM_QK, PRO_SIGMOID_GATES, PRO_DECAY_SOFTPLUS, PRO_DECAY_LOGSIGMOID = 1, 2, 4, 8


class PdnProblem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("chunk", ctypes.c_int),
                ("variant", ctypes.c_int), ("decay", ctypes.c_int), ("dtype", ctypes.c_int),
                ("impl", ctypes.c_int), ("q_scale", ctypes.c_float),
                ("precond_x", ctypes.c_float), ("precond_eps", ctypes.c_float),
                ("prologue", ctypes.c_int), ("decay_scale", ctypes.c_float)]


class PdnTensors(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k", "v", "log_alpha", "beta", "erase", "write", "S0", "ST", "A0", "AT", "o")]


class PdnGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dO", "dST", "dq", "dk", "dv", "dlog_alpha", "dbeta", "derase", "dwrite", "dS0",
                 "dA0")]


class PdnError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s returned %s" % (where, status_string(code)))


_lib = None


def load() -> ctypes.CDLL:
    """Load libpdn.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError("libpdn.so is not built (run python -m "
                              "linear_recurrence_sequence_chunked_b200.build)")
        lib = ctypes.CDLL(_LIB_PATH)
        P, T, vp = ctypes.POINTER(PdnProblem), ctypes.POINTER(PdnTensors), ctypes.c_void_p
        lib.pdn_chunk_fwd_workspace.restype = ctypes.c_size_t
        lib.pdn_chunk_fwd_workspace.argtypes = [P]
        lib.pdn_chunk_fwd_impl.restype = ctypes.c_int
        lib.pdn_chunk_fwd_impl.argtypes = [P]
        lib.pdn_chunk_fwd.restype = ctypes.c_int
        lib.pdn_chunk_fwd.argtypes = [P, T, vp, ctypes.c_size_t, vp]
        lib.pdn_chunk_fwd_profiled.restype = ctypes.c_int
        lib.pdn_chunk_fwd_profiled.argtypes = [P, T, vp, ctypes.c_size_t, vp,
                                               ctypes.POINTER(ctypes.c_float),
                                               ctypes.POINTER(ctypes.c_int)]
        lib.pdn_chunk_fwd_noalloc.restype = ctypes.c_int
        lib.pdn_chunk_fwd_noalloc.argtypes = [P, T, vp]
        lib.pdn_chunk_fwd_host.restype = ctypes.c_int
        lib.pdn_chunk_fwd_host.argtypes = [P, T, T, vp, ctypes.c_size_t, ctypes.c_int, vp]
        G = ctypes.POINTER(PdnGrads)
        lib.pdn_chunk_bwd_workspace.restype = ctypes.c_size_t
        lib.pdn_chunk_bwd_workspace.argtypes = [P]
        lib.pdn_chunk_bwd.restype = ctypes.c_int
        lib.pdn_chunk_bwd.argtypes = [P, T, G, vp, ctypes.c_size_t, vp]
        lib.pdn_chunk_fwd_save.restype = ctypes.c_int
        lib.pdn_chunk_fwd_save.argtypes = [P, T, vp, vp, vp, ctypes.c_size_t, vp]
        lib.pdn_chunk_bwd_saved.restype = ctypes.c_int
        lib.pdn_chunk_bwd_saved.argtypes = [P, T, G, vp, vp, vp, ctypes.c_size_t, vp]
        lib.pdn_chunk_transition.restype = ctypes.c_int
        lib.pdn_chunk_transition.argtypes = [P, T, vp, ctypes.c_size_t, vp]
        lib.pdn_key_energy.restype = ctypes.c_int
        lib.pdn_key_energy.argtypes = [P, T, vp]
        lib.pdn_accumulate.restype = ctypes.c_int
        lib.pdn_accumulate.argtypes = [ctypes.c_int, ctypes.c_longlong, vp, vp, vp, vp]
        lib.pdn_state_compose.restype = ctypes.c_int
        lib.pdn_state_compose.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp]
        lib.pdn_decode_step.restype = ctypes.c_int
        lib.pdn_decode_step.argtypes = [P, T, vp]
        lib.pdn_get_device_error.restype = ctypes.c_int
        lib.pdn_get_device_error.argtypes = [vp]
        lib.pdn_selftest_bounded_wait.restype = ctypes.c_int
        lib.pdn_selftest_bounded_wait.argtypes = [ctypes.c_longlong, vp]
        lib.pdn_status_string.restype = ctypes.c_char_p
        lib.pdn_status_string.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


# ------------------------------------------------------------------ C-ABI names
def pdn_chunk_fwd_workspace(problem: PdnProblem) -> int:
    return load().pdn_chunk_fwd_workspace(ctypes.byref(problem))


def pdn_chunk_fwd_impl(problem: PdnProblem) -> int:
    return load().pdn_chunk_fwd_impl(ctypes.byref(problem))


def pdn_chunk_fwd(problem: PdnProblem, tensors: PdnTensors, workspace: int, ws_bytes: int,
                  stream: int) -> int:
    return load().pdn_chunk_fwd(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                ws_bytes, stream)


def pdn_chunk_fwd_profiled(problem: PdnProblem, tensors: PdnTensors, workspace: int,
                           ws_bytes: int, stream: int):
    """pdn_chunk_fwd with CUDA events between its kernels (blocking). Returns
    (status, [milliseconds per kernel stage])."""
    ms = (ctypes.c_float * 4)()
    n = ctypes.c_int(0)
    rc = load().pdn_chunk_fwd_profiled(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                       ws_bytes, stream, ms, ctypes.byref(n))
    return rc, [float(ms[i]) for i in range(n.value)]


def pdn_chunk_bwd_workspace(problem: PdnProblem) -> int:
    return load().pdn_chunk_bwd_workspace(ctypes.byref(problem))


def pdn_chunk_bwd(problem: PdnProblem, tensors: PdnTensors, grads: PdnGrads, workspace: int,
                  ws_bytes: int, stream: int) -> int:
    return load().pdn_chunk_bwd(ctypes.byref(problem), ctypes.byref(tensors), ctypes.byref(grads),
                                workspace, ws_bytes, stream)


def pdn_chunk_fwd_save(problem: PdnProblem, tensors: PdnTensors, delta: int, ckpt: int,
                       workspace: int, ws_bytes: int, stream: int) -> int:
    return load().pdn_chunk_fwd_save(ctypes.byref(problem), ctypes.byref(tensors), delta, ckpt,
                                     workspace, ws_bytes, stream)


def pdn_chunk_bwd_saved(problem: PdnProblem, tensors: PdnTensors, grads: PdnGrads, delta: int,
                        ckpt: int, workspace: int, ws_bytes: int, stream: int) -> int:
    return load().pdn_chunk_bwd_saved(ctypes.byref(problem), ctypes.byref(tensors),
                                      ctypes.byref(grads), delta, ckpt, workspace, ws_bytes,
                                      stream)


def pdn_chunk_transition(problem: PdnProblem, tensors: PdnTensors, workspace: int,
                         ws_bytes: int, stream: int) -> int:
    return load().pdn_chunk_transition(ctypes.byref(problem), ctypes.byref(tensors), workspace,
                                       ws_bytes, stream)


def pdn_key_energy(problem: PdnProblem, tensors: PdnTensors, stream: int) -> int:
    return load().pdn_key_energy(ctypes.byref(problem), ctypes.byref(tensors), stream)


def pdn_accumulate(n: int, length: int, parts: int, base: Optional[int], out: int,
                   stream: int) -> int:
    return load().pdn_accumulate(n, length, parts, base, out, stream)


def pdn_state_compose(BH: int, d_v: int, d_k: int, S_in: Optional[int], A: int,
                      B_add: Optional[int], S_out: int, stream: int) -> int:
    return load().pdn_state_compose(BH, d_v, d_k, S_in, A, B_add, S_out, stream)


def pdn_chunk_fwd_noalloc(problem: PdnProblem, tensors: PdnTensors, stream: int) -> int:
    """Allocation-free chunked forward (see include/pdn.h): scratch comes
    from a fixed array inside the library instead of a caller workspace."""
    return load().pdn_chunk_fwd_noalloc(ctypes.byref(problem), ctypes.byref(tensors), stream)


def pdn_chunk_fwd_host(problem: PdnProblem, host: PdnTensors, dev: PdnTensors, workspace: int,
                       ws_bytes: int, slices: int, stream: int) -> int:
    """Chunked forward from (page-locked) host memory with the copies
    overlapped with the compute over `slices` parts of the batch (see
    include/pdn.h)."""
    return load().pdn_chunk_fwd_host(ctypes.byref(problem), ctypes.byref(host), ctypes.byref(dev),
                                     workspace, ws_bytes, slices, stream)


def pdn_decode_step(problem: PdnProblem, tensors: PdnTensors, stream: int) -> int:
    return load().pdn_decode_step(ctypes.byref(problem), ctypes.byref(tensors), stream)


def pdn_get_device_error(stream: int) -> int:
    return load().pdn_get_device_error(stream)


def pdn_selftest_bounded_wait(spin_limit: int, stream: int) -> int:
    return load().pdn_selftest_bounded_wait(spin_limit, stream)


def pdn_status_string(code: int) -> str:
    return load().pdn_status_string(code).decode()


status_string = pdn_status_string


# ------------------------------------------------------------------ torch helpers
def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("all tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("all tensors must be contiguous")
    return t.data_ptr() or None


def make_problem(variant: str, B: int, T: int, H: int, d_k: int, d_v: int, dtype,
                 decay: Optional[str] = None, chunk: int = 64, impl: str = "auto",
                 q_scale: float = 1.0, precond_x: float = 1.5,
                 precond_eps: float = 1e-6, prologue: int = 0,
                 decay_scale: float = 1.0) -> PdnProblem:
    if decay is None:
        decay = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar"}.get(variant, "channel")
    return PdnProblem(B, T, H, d_k, d_v, chunk, VARIANTS[variant], DECAYS[decay], DTYPES[dtype],
                      IMPLS[impl], q_scale, precond_x, precond_eps, prologue, decay_scale)


def _host_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda or not t.is_pinned():
        raise ValueError("host tensors must be page-locked CPU tensors (pin_memory())")
    if not t.is_contiguous():
        raise ValueError("all tensors must be contiguous")
    return t.data_ptr() or None


def make_host_tensors(q=None, k=None, v=None, o=None, log_alpha=None, beta=None, erase=None,
                      write=None, S0=None, ST=None, A0=None, AT=None) -> PdnTensors:
    """The `host` argument of pdn_chunk_fwd_host: page-locked CPU tensors;
    None leaves that tensor on the device."""
    return PdnTensors(_host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(log_alpha),
                      _host_ptr(beta), _host_ptr(erase), _host_ptr(write), _host_ptr(S0),
                      _host_ptr(ST), _host_ptr(A0), _host_ptr(AT), _host_ptr(o))


def make_tensors(q, k, v, o, log_alpha=None, beta=None, erase=None, write=None, S0=None,
                 ST=None, A0=None, AT=None) -> PdnTensors:
    return PdnTensors(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(erase),
                      _ptr(write), _ptr(S0), _ptr(ST), _ptr(A0), _ptr(AT), _ptr(o))


def _decay_of(log_alpha):
    if log_alpha is None:
        return "none"
    return "scalar" if log_alpha.dim() == 3 else "channel"


def _check(code, where):
    if code != PDN_OK:
        raise PdnError(code, where)


def chunk_fwd(variant: str, q, k, v, log_alpha=None, beta=None, erase=None, write=None,
              S0=None, A0=None, chunk: int = 64, impl: str = "auto", q_scale: float = 1.0,
              precond_x: float = 1.5, precond_eps: float = 1e-6, want_state: bool = True,
              out=None, workspace=None, prologue: int = 0, decay_scale: float = 1.0,
              saved: Optional[dict] = None):
    """Chunked forward on torch tensors (all on one CUDA device, contiguous).

    Returns (o, S_T, A_T); S_T/A_T are None when not requested / not used.
    With ``saved`` (a dict) the tensor-core forward also leaves every token's
    delta and the chunk-start states in saved["delta"] / saved["ckpt"] for
    ``chunk_bwd(..., saved=saved, ST=S_T)`` (training mode, pdn_chunk_fwd_save).
    """
    B, T, H, d_k = k.shape
    d_v = v.shape[3]
    dev = k.device
    p = make_problem(variant, B, T, H, d_k, d_v, k.dtype, _decay_of(log_alpha), chunk, impl,
                     q_scale, precond_x, precond_eps, prologue, decay_scale)
    o = out if out is not None else torch.empty(B, T, H, d_v, dtype=k.dtype, device=dev)
    ST = torch.empty(B, H, d_v, d_k, dtype=torch.float32, device=dev) if want_state else None
    AT = (torch.empty(B, H, d_k, dtype=torch.float32, device=dev)
          if (want_state and variant in PRECOND_VARIANTS) else None)
    t = make_tensors(q, k, v, o, log_alpha, beta, erase, write, S0, ST, A0, AT)
    need = pdn_chunk_fwd_workspace(p)
    if need == ctypes.c_size_t(-1).value:
        raise PdnError(PDN_ERR_INVALID_ARG, "pdn_chunk_fwd_workspace")
    ws_ptr, ws_bytes = None, 0
    if need > 0:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    stream = torch.cuda.current_stream(dev).cuda_stream
    if saved is not None:
        f32 = dict(dtype=torch.float32, device=dev)
        saved["delta"] = torch.empty(B, H, T, d_v, **f32)
        saved["ckpt"] = torch.empty(B, H, (T + 63) // 64, d_k, d_v, **f32)  # S^T per chunk
        _check(pdn_chunk_fwd_save(p, t, saved["delta"].data_ptr(), saved["ckpt"].data_ptr(),
                                  ws_ptr, ws_bytes, stream), "pdn_chunk_fwd_save")
    else:
        _check(pdn_chunk_fwd(p, t, ws_ptr, ws_bytes, stream), "pdn_chunk_fwd")
    return o, ST, AT


def make_grads(dO=None, dST=None, dq=None, dk=None, dv=None, dlog_alpha=None, dbeta=None,
               derase=None, dwrite=None, dS0=None, dA0=None) -> PdnGrads:
    return PdnGrads(_ptr(dO), _ptr(dST), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlog_alpha),
                    _ptr(dbeta), _ptr(derase), _ptr(dwrite), _ptr(dS0), _ptr(dA0))


def chunk_bwd(variant: str, q, k, v, dO=None, dST=None, log_alpha=None, beta=None, erase=None,
              write=None, S0=None, A0=None, q_scale: float = 1.0, precond_x: float = 1.5,
              precond_eps: float = 1e-6, workspace=None, prologue: int = 0,
              decay_scale: float = 1.0, saved: Optional[dict] = None, ST=None):
    """Gradients of chunk_fwd's (o, S_T) with respect to its inputs, given the
    cotangents dO [B,T,H,d_v] (input dtype) and dST [B,H,d_v,d_k] (fp32);
    either may be None (zero). Returns a dict of fp32 tensors with keys q, k,
    v, log_alpha, beta, erase, write, S0, A0 (None where the variant has no
    such input). With ``prologue`` bits the inputs are raw projections and the
    gradients are with respect to them. With ``saved`` (from chunk_fwd(...,
    saved=...)) and the forward's final state ``ST`` the backward reuses the
    forward's deltas and chunk-start states (pdn_chunk_bwd_saved)."""
    B, T, H, d_k = k.shape
    d_v = v.shape[3]
    dev = k.device
    p = make_problem(variant, B, T, H, d_k, d_v, k.dtype, _decay_of(log_alpha), 64, "auto",
                     q_scale, precond_x, precond_eps, prologue, decay_scale)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"q": torch.empty(B, T, H, d_k, **f32), "k": torch.empty(B, T, H, d_k, **f32),
         "v": torch.empty(B, T, H, d_v, **f32),
         "log_alpha": None if log_alpha is None else torch.empty(log_alpha.shape, **f32),
         "beta": None if beta is None else torch.empty(beta.shape, **f32),
         "erase": None if variant != "GDN2" else torch.empty(B, T, H, d_k, **f32),
         "write": (torch.empty(B, T, H, d_v, **f32) if variant in ("GDN2", "FG2_GDN_PLUS")
                   else None),
         "S0": torch.empty(B, H, d_v, d_k, **f32),
         "A0": torch.empty(B, H, d_k, **f32) if variant in PRECOND_VARIANTS else None}
    t = make_tensors(q, k, v, None, log_alpha, beta, erase, write, S0, ST, A0, None)
    gr = make_grads(dO, dST, g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["erase"],
                    g["write"], g["S0"], g["A0"])
    need = pdn_chunk_bwd_workspace(p)
    if need == ctypes.c_size_t(-1).value:
        raise PdnError(PDN_ERR_INVALID_ARG, "pdn_chunk_bwd_workspace")
    ws_ptr, ws_bytes = None, 0
    if need > 0:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    stream = torch.cuda.current_stream(dev).cuda_stream
    if saved is not None:
        _check(pdn_chunk_bwd_saved(p, t, gr, saved["delta"].data_ptr(), saved["ckpt"].data_ptr(),
                                   ws_ptr, ws_bytes, stream), "pdn_chunk_bwd_saved")
    else:
        _check(pdn_chunk_bwd(p, t, gr, ws_ptr, ws_bytes, stream), "pdn_chunk_bwd")
    return g


def decode_step(variant: str, q, k, v, S, A=None, log_alpha=None, beta=None, erase=None,
                write=None, q_scale: float = 1.0, precond_x: float = 1.5,
                precond_eps: float = 1e-6, out=None, prologue: int = 0,
                decay_scale: float = 1.0):
    """One decode token per sequence: q, k [B,1,H,d_k], v [B,1,H,d_v]; updates
    the fp32 state S [B,H,d_v,d_k] (and accumulator A [B,H,d_k]) in place and
    returns o [B,1,H,d_v]."""
    B, T, H, d_k = k.shape
    d_v = v.shape[3]
    p = make_problem(variant, B, T, H, d_k, d_v, k.dtype, _decay_of(log_alpha), 64, "auto",
                     q_scale, precond_x, precond_eps, prologue, decay_scale)
    o = out if out is not None else torch.empty(B, T, H, d_v, dtype=k.dtype, device=k.device)
    t = make_tensors(q, k, v, o, log_alpha, beta, erase, write, S, S, A, A)
    stream = torch.cuda.current_stream(k.device).cuda_stream
    _check(pdn_decode_step(p, t, stream), "pdn_decode_step")
    return o


def device_error(stream: Optional[int] = None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return pdn_get_device_error(stream)
