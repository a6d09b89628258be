"""ctypes binding of libssd (include/ssd.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
turns torch tensors into device pointers, the current torch stream into a
``cudaStream_t`` and status codes into exceptions.  There is no fallback: if
``libssd.so`` is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd.so")
# the index-checked build, loaded instead when SSD_DEBUG_CHECKS=1
DEBUG_LIB_PATH = os.path.join(_HERE, "libssd_debug.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_WORKSPACE, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(6)
SSD_DTYPE_F32, SSD_DTYPE_BF16 = 0, 1
PATH_AUTO, PATH_MODULAR, PATH_SIMT, PATH_FUSED, PATH_SPLIT = 0, 1, 2, 3, 4
IMPL_AUTO, IMPL_SIMT, IMPL_TC = 0, 1, 2
FLAG_TEST_STALL = 0x100

EXPORTS = [
    "ssd_status_string", "ssd_workspace_size", "ssd_path_supported", "ssd_forward",
    "ssd_forward_path", "ssd_device_status", "ssd_chunk_cumsum", "ssd_chunk_state",
    "ssd_state_pass", "ssd_chunk_scan", "ssd_diag_scan", "ssd_forward_host_bytes",
    "ssd_forward_host", "ssd_forward_noalloc", "ssd_auto_path", "ssd_forward_init",
    "ssd_decode_step", "ssd_discretize", "ssd_decay_total", "ssd_state_combine",
    "ssd_segment_state", "ssd_backward", "ssd_backward_workspace_size",
    "ssd_test_fail_calls", "ssd_test_pending_failures", "ssd_split_pieces",
    "ssd_device_status_where", "ssd_forward_discretized", "ssd_debug_build", "ssd_debug_record",
    "ssd_debug_fail_all",
]


class SSDError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)}")


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "T", "H", "P", "G", "N", "chunk", "a_per_state", "dtype")]

    def __repr__(self):
        return "Shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lib = None


def load(path: str = None):
    """Open libssd.so (built by ``ssd_chunked_forward_b200.build``), or the
    index-checked libssd_debug.so when the environment sets SSD_DEBUG_CHECKS=1."""
    global _lib
    if _lib is not None:
        return _lib
    if path is None:
        path = DEBUG_LIB_PATH if os.environ.get("SSD_DEBUG_CHECKS") == "1" else LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libssd.so not built ({path}); run python -m ssd_chunked_forward_b200.build")
    lib = ctypes.CDLL(path)
    vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    sp = ctypes.POINTER(Shape)
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_workspace_size.argtypes = [sp]
    lib.ssd_workspace_size.restype = sz
    lib.ssd_path_supported.argtypes = [sp, ctypes.c_uint]
    lib.ssd_path_supported.restype = ctypes.c_int
    lib.ssd_auto_path.argtypes = [sp]
    lib.ssd_auto_path.restype = ctypes.c_int
    lib.ssd_split_pieces.argtypes = [sp]
    lib.ssd_split_pieces.restype = ctypes.c_int
    lib.ssd_forward.argtypes = [sp, vp, fp, vp, vp, fp, vp, fp, vp, sz, vp]
    lib.ssd_forward_path.argtypes = [sp, vp, fp, vp, vp, fp, vp, fp, vp, sz, vp, ctypes.c_uint, ctypes.c_uint]
    lib.ssd_forward_init.argtypes = [sp, vp, fp, vp, vp, fp, fp, vp, fp, vp, sz, vp, ctypes.c_uint,
                                     ctypes.c_uint]
    lib.ssd_device_status.argtypes = [vp, vp]
    ip = ctypes.POINTER(ctypes.c_int)
    lib.ssd_device_status_where.argtypes = [vp, vp, ip, ip, ip]
    lib.ssd_debug_build.argtypes = []
    lib.ssd_debug_build.restype = ctypes.c_int
    lib.ssd_debug_record.argtypes = [ip, ip, ip, ip]
    lib.ssd_debug_fail_all.argtypes = [ctypes.c_int]
    lib.ssd_chunk_cumsum.argtypes = [sp, fp, fp, vp]
    lib.ssd_chunk_state.argtypes = [sp, vp, vp, fp, fp, vp, ctypes.c_uint]
    lib.ssd_state_pass.argtypes = [sp, fp, fp, fp, vp]
    lib.ssd_chunk_scan.argtypes = [sp, vp, vp, vp, fp, fp, fp, vp, vp, ctypes.c_uint]
    lib.ssd_diag_scan.argtypes = [sp, vp, vp, vp, fp, fp, fp, vp, vp, ctypes.c_uint]
    lib.ssd_forward_host_bytes.argtypes = [sp]
    lib.ssd_forward_host_bytes.restype = sz
    lib.ssd_forward_host.argtypes = [sp, vp, fp, vp, vp, fp, vp, fp, vp, sz, vp]
    lib.ssd_forward_noalloc.argtypes = [sp, vp, fp, vp, vp, fp, vp, fp, vp]
    lib.ssd_decode_step.argtypes = [sp, vp, fp, vp, vp, fp, fp, vp, vp]
    lib.ssd_discretize.argtypes = [sp, fp, fp, fp, vp, fp, vp, vp]
    lib.ssd_forward_discretized.argtypes = [sp, vp, fp, fp, fp, vp, vp, fp, vp, fp, vp, sz, vp]
    lib.ssd_decay_total.argtypes = [sp, fp, fp, vp]
    lib.ssd_state_combine.argtypes = [sp, ctypes.c_int, fp, fp, fp, fp, vp]
    lib.ssd_segment_state.argtypes = [sp, vp, fp, vp, fp, fp, vp, sz, vp]
    lib.ssd_test_fail_calls.argtypes = [ctypes.c_int]
    lib.ssd_test_fail_calls.restype = None
    lib.ssd_test_pending_failures.argtypes = []
    lib.ssd_test_pending_failures.restype = ctypes.c_int
    lib.ssd_backward.argtypes = [sp, vp, fp, vp, vp, fp, fp, vp, fp, vp, fp, vp, vp, fp, fp, vp, sz, vp]
    lib.ssd_backward_workspace_size.argtypes = [sp]
    lib.ssd_backward_workspace_size.restype = sz
    for name in ("ssd_forward_noalloc", "ssd_forward", "ssd_forward_path", "ssd_forward_init",
                 "ssd_device_status", "ssd_chunk_cumsum", "ssd_decode_step", "ssd_discretize",
                 "ssd_decay_total", "ssd_state_combine", "ssd_segment_state", "ssd_backward",
                 "ssd_chunk_state", "ssd_state_pass", "ssd_chunk_scan", "ssd_diag_scan",
                 "ssd_forward_host", "ssd_device_status_where", "ssd_forward_discretized"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().ssd_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != SSD_OK:
        raise SSDError(code, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(B, T, H, P, G, N, chunk, a_per_state=False, dtype="bf16") -> Shape:
    dt = SSD_DTYPE_BF16 if dtype in ("bf16", torch.bfloat16) else SSD_DTYPE_F32
    return Shape(int(B), int(T), int(H), int(P), int(G), int(N), int(chunk), int(bool(a_per_state)), dt)


def shape_of(x: torch.Tensor, a: torch.Tensor, Bm: torch.Tensor, chunk: int) -> Shape:
    B, T, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    return make_shape(B, T, H, P, G, N, chunk, a.dim() == 4, x.dtype)


def workspace_size(shape: Shape) -> int:
    return int(load().ssd_workspace_size(ctypes.byref(shape)))


def path_supported(shape: Shape, path: int) -> bool:
    return bool(load().ssd_path_supported(ctypes.byref(shape), int(path)))


def auto_path(shape: Shape) -> int:
    """The path SSD_PATH_AUTO takes for this shape (PATH_FUSED, PATH_SPLIT or
    PATH_MODULAR)."""
    return int(load().ssd_auto_path(ctypes.byref(shape)))


def split_pieces(shape: Shape) -> int:
    """Pieces per sequence of the split path (1: not split, 0: invalid)."""
    return int(load().ssd_split_pieces(ctypes.byref(shape)))


def alloc_workspace(shape: Shape, device=None) -> torch.Tensor:
    n = workspace_size(shape)
    if n == 0:
        raise SSDError(SSD_ERR_INVALID_ARG, "ssd_workspace_size")
    # torch's caching allocator returns >= 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _check_inputs(x, a, Bm, Cm, D):
    for name, t in (("x", x), ("a", a), ("Bm", Bm), ("Cm", Cm)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if a.dtype != torch.float32:
        raise ValueError("a must be float32")
    if x.dtype not in (torch.float32, torch.bfloat16) or Bm.dtype != x.dtype or Cm.dtype != x.dtype:
        raise ValueError("x, Bm, Cm must share dtype float32 or bfloat16")
    if D is not None and (D.dtype != torch.float32 or not D.is_cuda or not D.is_contiguous()):
        raise ValueError("D must be a contiguous float32 CUDA tensor")


def forward(x, a, Bm, Cm, D=None, chunk=256, *, y=None, final_state=None, want_final=True,
            workspace=None, path=PATH_AUTO, flags=0, stream=None, initial_state=None):
    """y[B,T,H,P] (and final state [B,H,N,P] fp32) of the chunked SSD forward.

    x [B,T,H,P], Bm/Cm [B,T,G,N] (float32 or bfloat16, same dtype), a [B,T,H]
    or [B,T,H,N] float32 log-decays, D [H] float32 or None, initial_state
    [B,H,N,P] float32 or None (zero).  Asynchronous on the current torch
    stream (or ``stream``)."""
    _check_inputs(x, a, Bm, Cm, D)
    if initial_state is not None and (initial_state.dtype != torch.float32 or not initial_state.is_cuda
                                      or not initial_state.is_contiguous()):
        raise ValueError("initial_state must be a contiguous float32 CUDA tensor")
    shape = shape_of(x, a, Bm, chunk)
    B, T, H, P = x.shape
    N = Bm.shape[3]
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((B, H, N, P), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    if initial_state is not None:
        if tuple(initial_state.shape) != (B, H, N, P):
            raise ValueError("initial_state must be [B,H,N,P]")
        code = load().ssd_forward_init(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(Cm),
                                       _ptr(D), _ptr(initial_state), _ptr(y), _ptr(final_state),
                                       _ptr(workspace), workspace.numel(), _stream(stream), int(path),
                                       int(flags))
        _check(code, "ssd_forward_init")
        return y, final_state
    code = load().ssd_forward_path(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(Cm),
                                   _ptr(D), _ptr(y), _ptr(final_state), _ptr(workspace),
                                   workspace.numel(), _stream(stream), int(path), int(flags))
    _check(code, "ssd_forward_path")
    return y, final_state


def device_status(workspace, stream=None) -> int:
    """Synchronise and return the workspace status word (SSD_OK or an error)."""
    return int(load().ssd_device_status(_ptr(workspace), _stream(stream)))


def debug_build() -> bool:
    """True when the loaded library is the index-checked debug build."""
    return bool(load().ssd_debug_build())


def debug_record():
    """(failed checks, line, block, thread) since the last call, then cleared;
    debug build only (raises SSDError otherwise)."""
    vals = [ctypes.c_int(0) for _ in range(4)]
    _check(load().ssd_debug_record(*(ctypes.byref(v) for v in vals)), "ssd_debug_record")
    return tuple(v.value for v in vals)


def debug_fail_all(on: bool) -> None:
    """Debug build only: make every index check fail (and skip its access)."""
    _check(load().ssd_debug_fail_all(1 if on else 0), "ssd_debug_fail_all")


def device_status_where(workspace, stream=None):
    """(status, source line, block, thread) of the first bounded wait that ran
    out in a fused-path kernel; zeros when none did."""
    line, block, thread = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = int(load().ssd_device_status_where(_ptr(workspace), _stream(stream), ctypes.byref(line),
                                            ctypes.byref(block), ctypes.byref(thread)))
    return st, line.value, block.value, thread.value


def chunk_cumsum(shape: Shape, a, cum=None, stream=None):
    nc = -(-shape.T // shape.chunk)  # the last chunk may end past T
    if cum is None:
        dims = (shape.B, shape.H, nc, shape.chunk) + ((shape.N,) if shape.a_per_state else ())
        cum = torch.empty(dims, dtype=torch.float32, device=a.device)
    _check(load().ssd_chunk_cumsum(ctypes.byref(shape), _ptr(a), _ptr(cum), _stream(stream)),
           "ssd_chunk_cumsum")
    return cum


def chunk_state(shape: Shape, x, Bm, cum, states=None, impl=IMPL_AUTO, stream=None):
    nc = -(-shape.T // shape.chunk)  # the last chunk may end past T
    if states is None:
        states = torch.empty((shape.B, shape.H, nc, shape.N, shape.P), dtype=torch.float32,
                             device=x.device)
    _check(load().ssd_chunk_state(ctypes.byref(shape), _ptr(x), _ptr(Bm), _ptr(cum), _ptr(states),
                                  _stream(stream), int(impl)), "ssd_chunk_state")
    return states


def state_pass(shape: Shape, cum, states, final_state=None, stream=None):
    _check(load().ssd_state_pass(ctypes.byref(shape), _ptr(cum), _ptr(states), _ptr(final_state),
                                 _stream(stream)), "ssd_state_pass")
    return states, final_state


def chunk_scan(shape: Shape, x, Bm, Cm, cum, Hin, D=None, y=None, impl=IMPL_AUTO, stream=None):
    if y is None:
        y = torch.empty_like(x)
    fn = load().ssd_diag_scan if shape.a_per_state else load().ssd_chunk_scan
    _check(fn(ctypes.byref(shape), _ptr(x), _ptr(Bm), _ptr(Cm), _ptr(cum), _ptr(Hin), _ptr(D),
              _ptr(y), _stream(stream), int(impl)),
           "ssd_diag_scan" if shape.a_per_state else "ssd_chunk_scan")
    return y


def forward_host_bytes(shape: Shape) -> int:
    return int(load().ssd_forward_host_bytes(ctypes.byref(shape)))


def forward_host(shape: Shape, x_h, a_h, Bm_h, Cm_h, D_h, y_h, final_h, dev_buf, stream=None):
    """The forward from HOST buffers (pinned for asynchrony): the library copies
    the inputs to ``dev_buf``, runs, and copies y (and the final state) back,
    all queued on the stream.  The caller synchronises."""
    _check(load().ssd_forward_host(ctypes.byref(shape), _ptr(x_h), _ptr(a_h), _ptr(Bm_h), _ptr(Cm_h),
                                   _ptr(D_h), _ptr(y_h), _ptr(final_h), _ptr(dev_buf),
                                   dev_buf.numel(), _stream(stream)), "ssd_forward_host")


def forward_noalloc(x, a, Bm, Cm, D=None, chunk=256, *, y=None, final_state=None, stream=None):
    """The fused forward with the library's own fixed scratch (no workspace,
    nothing allocated by the library); see ssd_forward_noalloc in ssd.h."""
    _check_inputs(x, a, Bm, Cm, D)
    shape = shape_of(x, a, Bm, chunk)
    B, T, H, P = x.shape
    N = Bm.shape[3]
    if y is None:
        y = torch.empty_like(x)
    if final_state is None:
        final_state = torch.empty((B, H, N, P), dtype=torch.float32, device=x.device)
    _check(load().ssd_forward_noalloc(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(Cm),
                                      _ptr(D), _ptr(y), _ptr(final_state), _stream(stream)),
           "ssd_forward_noalloc")
    return y, final_state


def decode_step(x, a, Bm, Cm, D, state, *, y=None, stream=None):
    """One recurrent step for a batch of single tokens, in place on ``state``.

    x [B,H,P], Bm/Cm [B,G,N] (float32 or bfloat16), a [B,H] or [B,H,N] float32
    log-decays, D [H] float32 or None, state [B,H,N,P] float32 (updated).
    Returns y [B,H,P]."""
    for name, t in (("x", x), ("a", a), ("Bm", Bm), ("Cm", Cm), ("state", state)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if a.dtype != torch.float32 or state.dtype != torch.float32:
        raise ValueError("a and state must be float32")
    if Bm.dtype != x.dtype or Cm.dtype != x.dtype:
        raise ValueError("x, Bm, Cm must share dtype")
    B, H, P = x.shape
    G, N = Bm.shape[1], Bm.shape[2]
    if tuple(state.shape) != (B, H, N, P):
        raise ValueError("state must be [B,H,N,P]")
    shape = make_shape(B, 1, H, P, G, N, 1, a.dim() == 3, x.dtype)
    if y is None:
        y = torch.empty_like(x)
    _check(load().ssd_decode_step(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(Cm), _ptr(D),
                                  _ptr(state), _ptr(y), _stream(stream)), "ssd_decode_step")
    return y


def discretize(dt_raw, dt_bias, A_log, x, *, a_out=None, x_out=None, stream=None):
    """dt = softplus(dt_raw + dt_bias); returns (a, x_out): a = -dt exp(A_log)
    ([B,T,H], or [B,T,H,N] when A_log is [H,N]) and x_out = dt x ([B,T,H,P],
    x's dtype), the inputs of forward()."""
    for name, t in (("dt_raw", dt_raw), ("A_log", A_log), ("x", x)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dt_raw.dtype != torch.float32 or A_log.dtype != torch.float32:
        raise ValueError("dt_raw and A_log must be float32")
    B, T, H, P = x.shape
    per_state = A_log.dim() == 2
    N = A_log.shape[1] if per_state else 1
    shape = make_shape(B, T, H, P, 1, N, 1, per_state, x.dtype)
    if a_out is None:
        a_out = torch.empty((B, T, H) + ((N,) if per_state else ()), dtype=torch.float32, device=x.device)
    if x_out is None:
        x_out = torch.empty_like(x)
    _check(load().ssd_discretize(ctypes.byref(shape), _ptr(dt_raw), _ptr(dt_bias), _ptr(A_log), _ptr(x),
                                 _ptr(a_out), _ptr(x_out), _stream(stream)), "ssd_discretize")
    return a_out, x_out


def forward_discretized(x, dt_raw, dt_bias, A_log, Bm, Cm, D=None, chunk=256, *, y=None, final_state=None,
                        want_final=True, workspace=None, stream=None):
    """discretize() followed by forward() in one fused pass (x_out and a are never
    written): y = SSD(dt x, -dt exp(A_log), Bm, Cm) + D (dt x), dt = softplus(dt_raw
    + dt_bias).  x [B,T,H,P] bf16, dt_raw [B,T,H] float32, dt_bias [H] or None,
    A_log [H] float32 (scalar decay only)."""
    for name, t in (("dt_raw", dt_raw), ("A_log", A_log)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float32:
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    B, T, H, P = x.shape
    if tuple(dt_raw.shape) != (B, T, H) or tuple(A_log.shape) != (H,):
        raise ValueError("dt_raw must be [B,T,H] and A_log [H]")
    _check_inputs(x, dt_raw, Bm, Cm, D)
    shape = shape_of(x, dt_raw, Bm, chunk)
    N = Bm.shape[3]
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((B, H, N, P), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    _check(load().ssd_forward_discretized(ctypes.byref(shape), _ptr(x), _ptr(dt_raw), _ptr(dt_bias),
                                          _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(y),
                                          _ptr(final_state), _ptr(workspace), workspace.numel(),
                                          _stream(stream)), "ssd_forward_discretized")
    return y, final_state


def decay_total(a, *, out=None, stream=None):
    """Total log-decay of each chain over the sequence: a [B,T,H] -> [B,H]
    (a [B,T,H,N] -> [B,H,N])."""
    if not a.is_cuda or not a.is_contiguous() or a.dtype != torch.float32:
        raise ValueError("a must be a contiguous float32 CUDA tensor")
    B, T, H = a.shape[:3]
    per_state = a.dim() == 4
    N = a.shape[3] if per_state else 1
    shape = make_shape(B, T, H, 1, 1, N, 1, per_state, torch.float32)
    if out is None:
        out = torch.empty((B, H) + ((N,) if per_state else ()), dtype=torch.float32, device=a.device)
    _check(load().ssd_decay_total(ctypes.byref(shape), _ptr(a), _ptr(out), _stream(stream)),
           "ssd_decay_total")
    return out


def state_combine(finals, totals, h0=None, *, out=None, stream=None):
    """finals [S,B,H,N,P] (each segment's final state from zero), totals
    [S,B,H] or [S,B,H,N] -> h_in [S+1,B,H,N,P]: h_in[s] enters segment s,
    h_in[S] is the state after all of them (h0, or zero, enters segment 0)."""
    for name, t in (("finals", finals), ("totals", totals)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float32:
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    S, B, H, N, P = finals.shape
    per_state = totals.dim() == 4
    shape = make_shape(B, 1, H, P, 1, N, 1, per_state, torch.float32)
    if out is None:
        out = torch.empty((S + 1, B, H, N, P), dtype=torch.float32, device=finals.device)
    _check(load().ssd_state_combine(ctypes.byref(shape), int(S), _ptr(finals), _ptr(totals), _ptr(h0),
                                    _ptr(out), _stream(stream)), "ssd_state_combine")
    return out


def segment_state(x, a, Bm, chunk=256, *, final_state=None, total=None, workspace=None, stream=None):
    """The state a segment builds from a zero start, [B,H,N,P] fp32, and its
    total log-decay [B,H] (or [B,H,N]), without computing its outputs."""
    for name, t in (("x", x), ("a", a), ("Bm", Bm)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    shape = shape_of(x, a, Bm, chunk)
    B, T, H, P = x.shape
    N = Bm.shape[3]
    if final_state is None:
        final_state = torch.empty((B, H, N, P), dtype=torch.float32, device=x.device)
    if total is None:
        total = torch.empty((B, H) + ((N,) if a.dim() == 4 else ()), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    _check(load().ssd_segment_state(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(final_state),
                                    _ptr(total), _ptr(workspace), workspace.numel(), _stream(stream)),
           "ssd_segment_state")
    return final_state, total


def backward_workspace_size(shape: Shape) -> int:
    return int(load().ssd_backward_workspace_size(ctypes.byref(shape)))


def backward(x, a, Bm, Cm, D, dy, chunk=256, *, dfinal=None, initial_state=None, want_dD=True,
             want_dinit=True, workspace=None, stream=None):
    """Gradients of sum(dy * y) + <dfinal, final_state> for the forward of the
    same inputs (scalar decay, or per-state up to N = 128): returns dict dx,
    da, dBm, dCm, dD (or None), dinit (or None).  Shapes and dtypes as for
    forward(); dy like x; dfinal and initial_state [B,H,N,P] float32 or None.  Asynchronous on the current
    torch stream (or ``stream``)."""
    _check_inputs(x, a, Bm, Cm, D)
    if dy.shape != x.shape or dy.dtype != x.dtype or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous tensor of x's shape and dtype")
    B, T, H, P = x.shape
    N = Bm.shape[3]
    for name, t in (("dfinal", dfinal), ("initial_state", initial_state)):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()
                              or tuple(t.shape) != (B, H, N, P)):
            raise ValueError(f"{name} must be a contiguous float32 [B,H,N,P] tensor")
    shape = shape_of(x, a, Bm, chunk)
    need = backward_workspace_size(shape)
    if need == 0:
        raise SSDError(SSD_ERR_UNSUPPORTED, "ssd_backward_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    out = {
        "dx": torch.empty_like(x), "da": torch.empty_like(a),
        "dBm": torch.empty_like(Bm), "dCm": torch.empty_like(Cm),
        "dD": torch.empty(H, dtype=torch.float32, device=x.device) if want_dD else None,
        "dinit": torch.empty((B, H, N, P), dtype=torch.float32, device=x.device) if want_dinit else None,
    }
    _check(load().ssd_backward(ctypes.byref(shape), _ptr(x), _ptr(a), _ptr(Bm), _ptr(Cm), _ptr(D),
                               _ptr(initial_state), _ptr(dy), _ptr(dfinal), _ptr(out["dx"]),
                               _ptr(out["da"]), _ptr(out["dBm"]), _ptr(out["dCm"]), _ptr(out["dD"]),
                               _ptr(out["dinit"]), _ptr(workspace), workspace.numel(), _stream(stream)),
           "ssd_backward")
    return out

