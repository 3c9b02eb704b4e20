"""Host-side checks of the C ABI (no GPU needed, no compute calls):
the library loads, exports every function include/pdn.h declares, its structs
have the layout the binding assumes, and invalid arguments are rejected
before anything touches a device."""
import ctypes
import os
import re
import subprocess

import pytest

from linear_recurrence_sequence_chunked_b200 import build as pdn_build
from linear_recurrence_sequence_chunked_b200 import pdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pdn.h")


@pytest.fixture(scope="module")
def lib():
    pdn_build.build()
    return pdn.load()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(pdn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("pdn_chunk_fwd", "pdn_chunk_fwd_workspace", "pdn_decode_step",
              "pdn_get_device_error", "pdn_status_string", "pdn_selftest_bounded_wait"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), "libpdn.so does not export %s" % n
    out = subprocess.run(["nm", "-D", "--defined-only", pdn._LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in declared_functions():
        assert re.search(r"\bT %s$" % n, out, flags=re.M), n


def test_struct_layout_matches_header(tmp_path):
    """Compile a probe against include/pdn.h with the host compiler and
    compare sizeof/offsetof with the ctypes mirrors."""
    src = tmp_path / "layout.c"
    fields_p = [f[0] for f in pdn.PdnProblem._fields_]
    fields_t = [f[0] for f in pdn.PdnTensors._fields_]
    fields_g = [f[0] for f in pdn.PdnGrads._fields_]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "pdn.h"', 'int main(void){',
             'printf("%zu %zu %zu\\n", sizeof(pdn_problem_t), sizeof(pdn_tensors_t), '
             'sizeof(pdn_grads_t));']
    for f in fields_p:
        lines.append('printf("p %s %%zu\\n", offsetof(pdn_problem_t, %s));' % (f, f))
    for f in fields_t:
        lines.append('printf("t %s %%zu\\n", offsetof(pdn_tensors_t, %s));' % (f, f))
    for f in fields_g:
        lines.append('printf("g %s %%zu\\n", offsetof(pdn_grads_t, %s));' % (f, f))
    lines.append("return 0;}")
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    sp, stt, sg = map(int, out[0].split())
    assert sp == ctypes.sizeof(pdn.PdnProblem)
    assert stt == ctypes.sizeof(pdn.PdnTensors)
    assert sg == ctypes.sizeof(pdn.PdnGrads)
    for line in out[1:]:
        if not line:
            continue
        kind, name, off = line.split()
        cls = {"p": pdn.PdnProblem, "t": pdn.PdnTensors, "g": pdn.PdnGrads}[kind]
        assert getattr(cls, name).offset == int(off), name


def test_status_strings(lib):
    assert pdn.pdn_status_string(0) == "PDN_OK"
    assert pdn.pdn_status_string(4) == "PDN_ERR_TIMEOUT"
    assert pdn.pdn_status_string(99) == "PDN_ERR_UNKNOWN"


FAKE = 0x7f0000000000  # a 16-byte aligned address that is never dereferenced


def _tensors(**over):
    d = dict(q=FAKE, k=FAKE + 0x1000, v=FAKE + 0x2000, log_alpha=FAKE + 0x3000,
             beta=FAKE + 0x4000, erase=None, write=None, S0=None, ST=None, A0=None, AT=None,
             o=FAKE + 0x5000)
    d.update(over)
    return pdn.PdnTensors(**d)


def _problem(**over):
    p = dict(B=2, T=100, H=4, d_k=64, d_v=64, chunk=64, variant=pdn.VARIANTS["PGDN"],
             decay=pdn.DECAYS["scalar"], dtype=1, impl=0, q_scale=1.0, precond_x=1.5,
             precond_eps=1e-6, prologue=0, decay_scale=1.0)
    p.update(over)
    return pdn.PdnProblem(**p)


INVALID_PROBLEMS = [
    dict(B=0), dict(H=0), dict(T=-1), dict(d_k=0), dict(d_k=24), dict(d_v=256), dict(chunk=48),
    dict(variant=10), dict(variant=-1), dict(decay=3), dict(dtype=5), dict(impl=7),
    dict(decay=pdn.DECAYS["channel"]),              # PGDN needs scalar decay
    dict(precond_x=2.5), dict(precond_x=0.5), dict(precond_eps=0.0),
    dict(q_scale=float("nan")),
    dict(prologue=16), dict(prologue=-1), dict(prologue=4 | 8),  # unknown bits / both decays
    dict(prologue=4, decay_scale=0.0), dict(prologue=4, decay_scale=float("inf")),
    dict(prologue=8, variant=pdn.VARIANTS["PDN"], decay=pdn.DECAYS["none"]),  # decay bit, no decay
]


@pytest.mark.parametrize("over", INVALID_PROBLEMS)
def test_invalid_problem_rejected(lib, over):
    p = _problem(**over)
    assert pdn.pdn_chunk_fwd(p, _tensors(), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd_workspace(p) == ctypes.c_size_t(-1).value


INVALID_TENSORS = [
    dict(q=None), dict(o=None), dict(k=FAKE + 8),           # missing / misaligned
    dict(log_alpha=None),                                    # PGDN needs a decay
    dict(beta=None),                                         # needs beta
    dict(erase=FAKE + 0x6000),                               # GDN2-only gate
    dict(S0=FAKE + 0x7004),                                  # misaligned state
]


@pytest.mark.parametrize("over", INVALID_TENSORS)
def test_invalid_tensors_rejected(lib, over):
    assert pdn.pdn_chunk_fwd(_problem(), _tensors(**over), None, 0, None) == pdn.PDN_ERR_INVALID_ARG


def test_variant_specific_rules(lib):
    # FG2 needs d_k == d_v
    p = _problem(variant=pdn.VARIANTS["FG2_GDN"], d_v=32)
    assert pdn.pdn_chunk_fwd(p, _tensors(), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    # GDN2 takes erase/write and no beta
    p = _problem(variant=pdn.VARIANTS["GDN2"], decay=pdn.DECAYS["channel"])
    assert pdn.pdn_chunk_fwd(p, _tensors(), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    # a non-preconditioned variant must not get an accumulator
    p = _problem(variant=pdn.VARIANTS["GDN"])
    assert pdn.pdn_chunk_fwd(p, _tensors(A0=FAKE + 0x8000), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    # FG2-GDN+ takes the key-side gain (beta) and the value-side gain (write), no erase gate
    p = _problem(variant=pdn.VARIANTS["FG2_GDN_PLUS"], decay=pdn.DECAYS["channel"])
    assert pdn.pdn_chunk_fwd(p, _tensors(), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd(p, _tensors(write=FAKE + 0x6000, erase=FAKE + 0x7000), None, 0,
                             None) == pdn.PDN_ERR_INVALID_ARG
    # PLA takes the scalar gain and no gates; it is preconditioned (accumulator allowed)
    p = _problem(variant=pdn.VARIANTS["PLA"], decay=pdn.DECAYS["channel"])
    assert pdn.pdn_chunk_fwd(p, _tensors(write=FAKE + 0x6000), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd(p, _tensors(beta=None), None, 0, None) == pdn.PDN_ERR_INVALID_ARG


def test_decode_rules(lib):
    p = _problem(T=1)
    # state must be updated in place
    assert pdn.pdn_decode_step(p, _tensors(S0=FAKE + 0x9000, ST=FAKE + 0xa000,
                                           A0=FAKE + 0xb000, AT=FAKE + 0xb000),
                               None) == pdn.PDN_ERR_INVALID_ARG
    # preconditioned decode needs the accumulator, in place
    assert pdn.pdn_decode_step(p, _tensors(S0=FAKE + 0x9000, ST=FAKE + 0x9000),
                               None) == pdn.PDN_ERR_INVALID_ARG
    # T must be 1
    p = _problem(T=2)
    assert pdn.pdn_decode_step(p, _tensors(S0=FAKE + 0x9000, ST=FAKE + 0x9000, A0=FAKE + 0xb000,
                                           AT=FAKE + 0xb000), None) == pdn.PDN_ERR_INVALID_ARG


def test_selftest_rejects_negative_limit(lib):
    assert pdn.pdn_selftest_bounded_wait(-1, None) == pdn.PDN_ERR_INVALID_ARG


def test_host_pipeline_argument_errors(lib):
    """pdn_chunk_fwd_host rejects bad arguments before it touches a device."""
    p = _problem()
    t = _tensors()
    need = pdn.pdn_chunk_fwd_workspace(p)
    ws = FAKE + 0x100000
    # slices outside [1, 128]
    assert pdn.pdn_chunk_fwd_host(p, t, t, ws, need, 0, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd_host(p, t, t, ws, need, 129, None) == pdn.PDN_ERR_INVALID_ARG
    # more parts than batch elements cut the sequences into runs that hand
    # the state on through the device ST (and AT, preconditioned variants)
    assert pdn.pdn_chunk_fwd_host(p, t, t, ws, need, p.B + 1, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd_host(p, t, _tensors(ST=FAKE + 0x6000), ws, need, p.B + 1,
                                  None) == pdn.PDN_ERR_INVALID_ARG
    # a host tensor without its device buffer
    assert pdn.pdn_chunk_fwd_host(p, _tensors(S0=FAKE + 0x9000), t, ws, need, 1,
                                  None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd_host(p, t, _tensors(q=None), ws, need, 1,
                                  None) == pdn.PDN_ERR_INVALID_ARG
    # an invalid problem
    assert pdn.pdn_chunk_fwd_host(_problem(B=0), t, t, ws, need, 1, None) == pdn.PDN_ERR_INVALID_ARG
    # a workspace smaller than the whole problem needs
    if need > 0:
        assert pdn.pdn_chunk_fwd_host(p, t, t, ws, need - 1, 1, None) == pdn.PDN_ERR_WORKSPACE


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (4, 4096, 16), (2, 130, 3), (3, 64, 2)])
def test_workspace_size_of_the_tensor_core_paths(lib, B, T, H):
    """The three-kernel path needs one 82,944-byte block per (batch, head,
    chunk); the CUDA-core path needs none (host-only queries)."""
    p = _problem(B=B, T=T, H=H, d_k=128, d_v=128)
    assert pdn.pdn_chunk_fwd_impl(p) == pdn.IMPLS["tc"]
    assert pdn.pdn_chunk_fwd_workspace(p) == B * H * ((T + 63) // 64) * 82944
    p = _problem(B=B, T=T, H=H, d_k=128, d_v=128, impl=3)  # no third kernel
    assert pdn.pdn_chunk_fwd_impl(p) == -1
    assert pdn.pdn_chunk_fwd_workspace(p) == (1 << 64) - 1
    p = _problem(B=B, T=T, H=H, d_k=64, d_v=64)
    assert pdn.pdn_chunk_fwd_impl(p) == pdn.IMPLS["simt"]
    assert pdn.pdn_chunk_fwd_workspace(p) == 0


def test_noalloc_size_gate(lib):
    """Host-only: B*H*ceil(T/64) = 810 chunk blocks exceeds the built-in array
    (PDN_ERR_WORKSPACE before anything touches a device); 809 passes the size
    gate and only then needs a device (PDN_ERR_CUDA here, without one)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("the 809-block case would launch on a real device")
    fake = 0x7f0000000000
    t = pdn.PdnTensors(q=fake, k=fake, v=fake, log_alpha=fake, beta=fake, o=fake)
    mk = lambda T: pdn.make_problem("GDN", 1, T, 1, 128, 128, torch.bfloat16, "scalar", 64, "tc")
    assert pdn.pdn_chunk_fwd_noalloc(mk(810 * 64), t, None) == pdn.PDN_ERR_WORKSPACE
    assert pdn.pdn_chunk_fwd_noalloc(mk(809 * 64), t, None) == pdn.PDN_ERR_CUDA
    assert pdn.pdn_chunk_fwd_noalloc(mk(808 * 64 + 1), t, None) == pdn.PDN_ERR_CUDA


def test_scalar_gate_alignment(lib):
    """fp32 per-(token, head) gates are read one element at a time: 4-byte
    alignment passes the argument checks (the call then needs a device:
    PDN_ERR_CUDA without one), 2-byte alignment does not. Vector tensors
    still need 16 bytes."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a passing check would launch on a real device")
    p = _problem()
    assert pdn.pdn_chunk_fwd(p, _tensors(log_alpha=FAKE + 0x3004, beta=FAKE + 0x4008), None, 0,
                             None) == pdn.PDN_ERR_CUDA
    assert pdn.pdn_chunk_fwd(p, _tensors(log_alpha=FAKE + 0x3002), None, 0,
                             None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd(p, _tensors(beta=FAKE + 0x4001), None, 0,
                             None) == pdn.PDN_ERR_INVALID_ARG
    # a per-channel gate (FG2 beta vector) keeps the 16-byte rule
    p = _problem(variant=pdn.VARIANTS["FG2_GDN"], decay=pdn.DECAYS["channel"])
    assert pdn.pdn_chunk_fwd(p, _tensors(beta=FAKE + 0x4004), None, 0,
                             None) == pdn.PDN_ERR_INVALID_ARG


def test_host_pipeline_validates_before_enqueueing(lib):
    """Every argument error of pdn_chunk_fwd_host comes back before anything
    is enqueued (without a device, reaching the enqueue stage would give
    PDN_ERR_CUDA instead)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a passing check would enqueue on a real device")
    p = _problem(B=3, T=131, H=1)
    need = pdn.pdn_chunk_fwd_workspace(p)
    ws = FAKE + 0x100000
    t = _tensors()
    assert pdn.pdn_chunk_fwd_host(p, t, _tensors(k=FAKE + 0x1008), ws, need, 2,
                                  None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_fwd_host(p, t, _tensors(log_alpha=FAKE + 0x3002), ws, need, 2,
                                  None) == pdn.PDN_ERR_INVALID_ARG
    # T * H odd: slice 1's scalar gates are 4-byte aligned, which is accepted
    assert pdn.pdn_chunk_fwd_host(p, t, t, ws, need, 2, None) == pdn.PDN_ERR_CUDA


# ------------------------------------------------------------------ backward
def _grads(**over):
    d = dict(dO=FAKE + 0x10000, dST=None, dq=FAKE + 0x11000, dk=FAKE + 0x12000,
             dv=FAKE + 0x13000, dlog_alpha=FAKE + 0x14000, dbeta=FAKE + 0x15000, derase=None,
             dwrite=None, dS0=None, dA0=None)
    d.update(over)
    return pdn.PdnGrads(**d)


@pytest.mark.parametrize("over", INVALID_PROBLEMS)
def test_backward_invalid_problem_rejected(lib, over):
    p = _problem(**over)
    assert pdn.pdn_chunk_bwd(p, _tensors(), _grads(), None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_bwd_workspace(p) == ctypes.c_size_t(-1).value


BWD_INVALID = [
    (dict(), dict(dq=FAKE + 0x11008)),                       # misaligned gradient
    (dict(), dict(dO=FAKE + 0x10004)),                       # misaligned cotangent
    (dict(), dict(dlog_alpha=FAKE + 0x14002)),               # scalar decay: 4-byte rule
    (dict(variant=pdn.VARIANTS["PDN"], decay=pdn.DECAYS["none"]), dict()),  # dlog_alpha, no decay
    (dict(), dict(derase=FAKE + 0x16000)),                   # GDN2-only gradient
    (dict(), dict(dwrite=FAKE + 0x16000)),                   # GDN2 / FG2+ only
    (dict(variant=pdn.VARIANTS["GDN"]), dict(dA0=FAKE + 0x17000)),  # no accumulator
]


@pytest.mark.parametrize("pover,gover", BWD_INVALID)
def test_backward_invalid_gradients_rejected(lib, pover, gover):
    p = _problem(**pover)
    t = _tensors(log_alpha=None) if p.decay == 0 else _tensors()
    assert pdn.pdn_chunk_bwd(p, t, _grads(**gover), FAKE, 1 << 40, None) == pdn.PDN_ERR_INVALID_ARG


def test_backward_rules(lib):
    # the forward output is not needed
    p = _problem()
    ws_need = pdn.pdn_chunk_bwd_workspace(p)
    assert 0 < ws_need < (1 << 40)
    # workspace missing, too small or misaligned
    assert pdn.pdn_chunk_bwd(p, _tensors(o=None), _grads(), None, 0, None) == pdn.PDN_ERR_WORKSPACE
    assert pdn.pdn_chunk_bwd(p, _tensors(o=None), _grads(), FAKE, ws_need - 1,
                             None) == pdn.PDN_ERR_WORKSPACE
    assert pdn.pdn_chunk_bwd(p, _tensors(o=None), _grads(), FAKE + 128, ws_need,
                             None) == pdn.PDN_ERR_WORKSPACE
    # prologue bits are checked as for the forward: unknown bits, both decay
    # maps, a softplus decay without a positive scale
    for bad in (dict(prologue=16), dict(prologue=4 | 8), dict(prologue=4, decay_scale=0.0)):
        assert pdn.pdn_chunk_bwd(_problem(**bad), _tensors(), _grads(), FAKE, ws_need,
                                 None) == pdn.PDN_ERR_INVALID_ARG, bad
    # T == 0 needs no workspace
    assert pdn.pdn_chunk_bwd_workspace(_problem(T=0)) == 0
    # the gradient struct itself is required
    assert load_bwd_null(lib) == pdn.PDN_ERR_INVALID_ARG


def load_bwd_null(lib):
    return lib.pdn_chunk_bwd(ctypes.byref(_problem()), ctypes.byref(_tensors()), None, None, 0,
                             None)


def test_debug_library_exports_every_declared_symbol():
    """libpdn_debug.so (index checks compiled in) offers the same C ABI."""
    lib = pdn_build.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True,
                         text=True).stdout
    for n in declared_functions():
        assert re.search(r"\bT %s$" % n, out, flags=re.M), n


def test_bounds_status_string(lib):
    assert pdn.pdn_status_string(pdn.PDN_ERR_BOUNDS) == "PDN_ERR_BOUNDS"


def test_training_mode_argument_errors(lib):
    """pdn_chunk_fwd_save / pdn_chunk_bwd_saved: the forward's and the
    backward's own checks first, then the saved buffers (present, 16-byte
    aligned; the backward also needs the forward's S_T), then the path: only
    problems the tensor-core forward takes. All decided before any launch."""
    D, C = FAKE + 0x20000, FAKE + 0x40000
    # the forward's checks come first
    p = _problem(B=0)
    assert pdn.pdn_chunk_fwd_save(p, _tensors(), D, C, None, 0, None) == pdn.PDN_ERR_INVALID_ARG
    # the saved buffers
    p = _problem()
    for d, c in ((None, C), (D, None), (D + 4, C), (D, C + 8)):
        assert pdn.pdn_chunk_fwd_save(p, _tensors(), d, c, None, 0,
                                      None) == pdn.PDN_ERR_INVALID_ARG, (d, c)
    # d = 64 runs on the CUDA-core path, which saves nothing
    assert pdn.pdn_chunk_fwd_save(p, _tensors(), D, C, None, 0, None) == pdn.PDN_ERR_UNSUPPORTED
    # the backward: its own checks, then the saved buffers and S_T, then the path
    ws = pdn.pdn_chunk_bwd_workspace(p)
    assert pdn.pdn_chunk_bwd_saved(_problem(B=0), _tensors(ST=FAKE + 0x9000), _grads(), D, C,
                                   FAKE, ws, None) == pdn.PDN_ERR_INVALID_ARG
    assert pdn.pdn_chunk_bwd_saved(p, _tensors(ST=FAKE + 0x9000), _grads(), D, C, None, 0,
                                   None) == pdn.PDN_ERR_WORKSPACE
    for d, c, st in ((None, C, FAKE + 0x9000), (D, None, FAKE + 0x9000), (D + 4, C, FAKE + 0x9000),
                     (D, C, None)):
        assert pdn.pdn_chunk_bwd_saved(p, _tensors(ST=st), _grads(), d, c, FAKE, ws,
                                       None) == pdn.PDN_ERR_INVALID_ARG, (d, c, st)
    assert pdn.pdn_chunk_bwd_saved(p, _tensors(ST=FAKE + 0x9000), _grads(), D, C, FAKE, ws,
                                   None) == pdn.PDN_ERR_UNSUPPORTED
