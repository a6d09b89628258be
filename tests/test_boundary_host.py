"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/ssd.h declares, sizes workspaces as documented and
rejects bad arguments with the documented status before touching the GPU."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from ssd_chunked_forward_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from ssd_chunked_forward_b200.build import build
    build()
    return ssd.load()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "ssd_forward" in names and len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(ssd.EXPORTS) == names


def test_debug_build_exports_and_reports(lib):
    """The index-checked variant exports the same symbols and says it is the
    debug build; the normal build says it is not and refuses the debug calls
    (neither call touches the device)."""
    import ctypes as C
    from ssd_chunked_forward_b200.build import build
    dbg = C.CDLL(build(debug=True))
    for n in declared_functions():
        assert hasattr(dbg, n), n
    assert dbg.ssd_debug_build() == 1
    assert lib.ssd_debug_build() == 0
    assert lib.ssd_debug_record(None, None, None, None) == ssd.SSD_ERR_UNSUPPORTED
    assert lib.ssd_debug_fail_all(1) == ssd.SSD_ERR_UNSUPPORTED


def test_status_strings(lib):
    for code in range(6):
        s = ssd.status_string(code)
        assert s.startswith("SSD_")
    assert ssd.status_string(99) == "SSD_ERR_UNKNOWN"


def _shape(**kw):
    base = dict(B=2, T=512, H=4, P=64, G=1, N=128, chunk=256, a_per_state=False, dtype="bf16")
    base.update(kw)
    return ssd.make_shape(**base)


def test_workspace_size_arithmetic(lib):
    s = _shape()
    nc = 512 // 256
    cum = 2 * 4 * nc * 256 * 4
    states = 2 * 4 * nc * 128 * 64 * 4
    rup = lambda v: (v + 255) // 256 * 256
    assert ssd.workspace_size(s) >= 256 + rup(cum) + rup(states)
    s4 = _shape(a_per_state=True, N=64, chunk=128)
    assert ssd.workspace_size(s4) >= 256 + rup(2 * 4 * 4 * 128 * 64 * 4)


@pytest.mark.parametrize("bad", [
    dict(H=3, G=2),         # H % G
    dict(B=0), dict(N=0), dict(P=0), dict(chunk=0),
    dict(chunk=2048, T=2048),
    dict(N=512), dict(P=300),
    dict(dtype=7),
])
def test_invalid_shapes_rejected(lib, bad):
    if bad.get("dtype") == 7:
        s = _shape()
        s.dtype = 7
    else:
        s = _shape(**bad)
    assert ssd.workspace_size(s) == 0
    assert not ssd.path_supported(s, ssd.PATH_AUTO)
    code = lib.ssd_forward(ctypes.byref(s), 256, 256, 256, 256, None, 256, None, 256, 1 << 40, None)
    assert code == ssd.SSD_ERR_INVALID_ARG


@pytest.mark.parametrize("T,chunk", [(500, 256), (1000, 256), (997, 256), (384, 256),
                                     (640, 512), (1024, 1000), (96, 256)])
def test_ragged_T_is_a_partial_last_chunk(lib, T, chunk):
    """T % chunk != 0: the last chunk holds the remaining tokens; the buffers
    are laid out for ceil(T / chunk) chunks (ceil(T / 128) blocks on the
    tensor-core modular path), never more than the padded length needs, and
    the paths served and AUTO's choice equal those of the padded length."""
    s = _shape(T=T, chunk=chunk)
    Tp = -(-T // chunk) * chunk
    padded = _shape(T=Tp, chunk=chunk)
    assert 0 < ssd.workspace_size(s) <= ssd.workspace_size(padded)
    for path in (ssd.PATH_AUTO, ssd.PATH_SIMT, ssd.PATH_MODULAR, ssd.PATH_FUSED):
        assert ssd.path_supported(s, path) == ssd.path_supported(padded, path)
    assert ssd.auto_path(s) == ssd.auto_path(padded)


def test_backward_workspace_and_validation(lib):
    """The backward's workspace holds the recomputed and adjoint chunk states
    and, on CUDA cores, the fp32 per-head partials (the tensor-core path keeps
    three row sums per token and head instead); the per-state variant is
    served up to N = 128; bad pointers and a short workspace are refused
    before any launch."""
    s = _shape()  # B=2, T=512, H=4, P=64, N=128, chunk 256, bf16: tensor cores
    need = ssd.backward_workspace_size(s)
    nc, f = 2, 4
    states = [2 * 4 * nc * 256 * f, 2 * 2 * 4 * nc * 128 * 64 * f, 2 * 4 * 128 * 64 * f]
    partials = [2 * 2 * 512 * 4 * 64 * f, 2 * 2 * 512 * 4 * 128 * f]
    assert sum(states) + 3 * 2 * 512 * 4 * f <= need < sum(states) + sum(partials)
    s32 = _shape(dtype="f32")  # CUDA cores: the per-head partials too
    assert ssd.backward_workspace_size(s32) >= sum(states) + sum(partials)
    # the per-state variant is served up to N = 128
    assert ssd.backward_workspace_size(_shape(a_per_state=True)) > need
    assert ssd.backward_workspace_size(_shape(a_per_state=True, N=256)) == 0
    ok = 1 << 20
    f_ = lambda *a: lib.ssd_backward(ctypes.byref(s), *a)
    args = [ok, ok, ok, ok, None, None, ok, None, ok, ok, ok, ok, None, None, ok, need, None]
    bad = list(args); bad[6] = None            # dy missing
    assert f_(*bad) == ssd.SSD_ERR_INVALID_ARG
    bad = list(args); bad[8] = ok + 4          # dx misaligned
    assert f_(*bad) == ssd.SSD_ERR_INVALID_ARG
    bad = list(args); bad[15] = need - 1       # workspace too small
    assert f_(*bad) == ssd.SSD_ERR_WORKSPACE
    bad = list(args); bad[14] = ok + 16        # workspace misaligned
    assert f_(*bad) == ssd.SSD_ERR_WORKSPACE
    sp = _shape(a_per_state=True, N=256)
    assert lib.ssd_backward(ctypes.byref(sp), *args) == ssd.SSD_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected(lib):
    s = _shape()
    ok = 1 << 20  # a 16-byte aligned fake address; never dereferenced
    ws = ssd.workspace_size(s)
    f = lambda *a: lib.ssd_forward(ctypes.byref(s), *a)
    assert f(None, ok, ok, ok, None, ok, None, ok, ws, None) == ssd.SSD_ERR_INVALID_ARG
    assert f(ok, None, ok, ok, None, ok, None, ok, ws, None) == ssd.SSD_ERR_INVALID_ARG
    assert f(ok, ok, ok, ok, None, None, None, ok, ws, None) == ssd.SSD_ERR_INVALID_ARG
    assert f(ok + 2, ok, ok, ok, None, ok, None, ok, ws, None) == ssd.SSD_ERR_INVALID_ARG
    assert f(ok, ok, ok, ok, ok + 4, ok, None, ok, ws, None) == ssd.SSD_ERR_INVALID_ARG
    # workspace: missing, misaligned, too small
    assert f(ok, ok, ok, ok, None, ok, None, None, ws, None) == ssd.SSD_ERR_WORKSPACE
    assert f(ok, ok, ok, ok, None, ok, None, ok + 16, ws, None) == ssd.SSD_ERR_WORKSPACE
    assert f(ok, ok, ok, ok, None, ok, None, ok, ws - 1, None) == ssd.SSD_ERR_WORKSPACE
    # unknown path or flag
    g = lambda path, flags: lib.ssd_forward_path(ctypes.byref(s), ok, ok, ok, ok, None, ok, None,
                                                 ok, ws, None, path, flags)
    assert g(9, 0) == ssd.SSD_ERR_INVALID_ARG
    assert g(0, 0x1) == ssd.SSD_ERR_INVALID_ARG


def test_step_entry_points_validate(lib):
    s = _shape()
    ok = 1 << 20
    assert lib.ssd_chunk_cumsum(ctypes.byref(s), None, ok, None) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_chunk_state(ctypes.byref(s), ok, ok, ok, None, None, 0) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_chunk_state(ctypes.byref(s), ok, ok, ok, ok, None, 7) == ssd.SSD_ERR_INVALID_ARG
    assert lib.ssd_state_pass(ctypes.byref(s), ok, None, None, None) == ssd.SSD_ERR_INVALID_ARG
    # scan entry points check the decay variant they serve
    assert lib.ssd_diag_scan(ctypes.byref(s), ok, ok, ok, ok, ok, None, ok, None, 0) == \
        ssd.SSD_ERR_INVALID_ARG
    s4 = _shape(a_per_state=True)
    assert lib.ssd_chunk_scan(ctypes.byref(s4), ok, ok, ok, ok, ok, None, ok, None, 0) == \
        ssd.SSD_ERR_INVALID_ARG


def test_host_entry_point_validates(lib):
    s = _shape()
    ok = 1 << 20
    need = ssd.forward_host_bytes(s)
    assert need > ssd.workspace_size(s)
    f = lambda *a: lib.ssd_forward_host(ctypes.byref(s), *a)
    assert f(None, ok, ok, ok, None, ok, None, ok, need, None) == ssd.SSD_ERR_INVALID_ARG
    assert f(ok, ok, ok, ok, None, ok, None, ok, need - 1, None) == ssd.SSD_ERR_WORKSPACE
    assert f(ok, ok, ok, ok, None, ok, None, ok + 16, need, None) == ssd.SSD_ERR_WORKSPACE


def test_auto_path_choice(lib):
    """AUTO takes the fused kernel for the Mamba-2 shapes with enough (batch,
    head) chains, the split path for few long chains whose length divides into
    pieces of >= 4096 tokens, and the modular path for the rest, fp32 and the
    per-state variant; an invalid shape gives -1."""
    fused = ssd.make_shape(4, 8192, 80, 64, 1, 128, 256)            # 320 chains
    assert ssd.auto_path(fused) == ssd.PATH_FUSED
    assert ssd.auto_path(ssd.make_shape(8, 2048, 24, 64, 1, 128, 256)) == ssd.PATH_FUSED   # 192
    assert ssd.auto_path(ssd.make_shape(1, 8192, 80, 64, 1, 128, 256)) == ssd.PATH_FUSED   # 80
    assert ssd.auto_path(ssd.make_shape(1, 262144, 32, 64, 8, 128, 256)) == ssd.PATH_SPLIT  # 32
    assert ssd.auto_path(ssd.make_shape(1, 4096, 32, 64, 8, 128, 256)) == ssd.PATH_MODULAR  # too short
    assert ssd.auto_path(ssd.make_shape(1, 8193, 32, 64, 8, 128, 256)) == ssd.PATH_MODULAR  # T odd
    long1 = ssd.make_shape(1, 262144, 32, 64, 8, 128, 256)
    assert ssd.path_supported(long1, ssd.PATH_SPLIT)
    assert not ssd.path_supported(ssd.make_shape(1, 262144, 32, 64, 8, 128, 256, dtype="f32"),
                                  ssd.PATH_SPLIT)
    assert ssd.auto_path(ssd.make_shape(4, 8192, 80, 64, 1, 128, 256, dtype="f32")) == ssd.PATH_MODULAR
    assert ssd.auto_path(ssd.make_shape(4, 4096, 16, 64, 1, 64, 128, a_per_state=True)) == ssd.PATH_MODULAR
    # T % chunk != 0: a partial last chunk; 2 chains is few, so modular
    assert ssd.auto_path(ssd.make_shape(1, 100, 2, 64, 1, 128, 64)) == ssd.PATH_MODULAR
    assert ssd.auto_path(ssd.make_shape(1, 100, 3, 64, 2, 128, 64)) == -1  # H % G != 0


def test_decode_step_validates(lib):
    """The decode step takes T == 1 and chunk == 1 and rejects null or
    misaligned pointers before any launch."""
    good = ssd.make_shape(2, 1, 4, 64, 1, 128, 1)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails validation
    f = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    def call(shape, x=p, a=f, bm=p, cm=p, st=f, y=p):
        return lib.ssd_decode_step(ctypes.byref(shape), x, a, bm, cm, None, st, y, None)
    assert call(ssd.make_shape(2, 4, 4, 64, 1, 128, 1)) == ssd.SSD_ERR_INVALID_ARG   # T != 1
    assert call(ssd.make_shape(2, 1, 4, 64, 1, 128, 4)) == ssd.SSD_ERR_INVALID_ARG   # chunk != 1
    assert call(good, x=None) == ssd.SSD_ERR_INVALID_ARG
    assert call(good, st=None) == ssd.SSD_ERR_INVALID_ARG
    assert call(good, y=ctypes.c_void_p((1 << 20) + 4)) == ssd.SSD_ERR_INVALID_ARG  # misaligned


def test_chain_count_beyond_grid_y_refused_before_launch(lib):
    """The CUDA-core steps and the backward index (batch, head) chains along
    gridDim.y (at most 65535).  A batch with more chains is refused with
    SSD_ERR_UNSUPPORTED before anything is queued; the fused kernel (a flat
    grid) still serves it, so AUTO picks it."""
    big = ssd.make_shape(1024, 256, 80, 64, 1, 128, 256)        # 81920 chains
    assert ssd.path_supported(big, ssd.PATH_FUSED)
    assert not ssd.path_supported(big, ssd.PATH_MODULAR)
    assert not ssd.path_supported(big, ssd.PATH_SIMT)
    assert ssd.auto_path(big) == ssd.PATH_FUSED
    assert ssd.backward_workspace_size(big) == 0
    ok = 1 << 20
    ws = ssd.workspace_size(big)
    g = lambda path: lib.ssd_forward_path(ctypes.byref(big), ok, ok, ok, ok, None, ok, None,
                                          ok, ws, None, path, 0)
    assert g(ssd.PATH_MODULAR) == ssd.SSD_ERR_UNSUPPORTED
    assert g(ssd.PATH_SIMT) == ssd.SSD_ERR_UNSUPPORTED
    args = [ok, ok, ok, ok, None, None, ok, None, ok, ok, ok, ok, None, None, ok, 1 << 40, None]
    assert lib.ssd_backward(ctypes.byref(big), *args) == ssd.SSD_ERR_UNSUPPORTED
    assert lib.ssd_chunk_cumsum(ctypes.byref(big), ok, ok, None) == ssd.SSD_ERR_UNSUPPORTED
    assert lib.ssd_state_pass(ctypes.byref(big), ok, ok, None, None) == ssd.SSD_ERR_UNSUPPORTED
    assert lib.ssd_chunk_scan(ctypes.byref(big), ok, ok, ok, ok, ok, None, ok, None, 0) == \
        ssd.SSD_ERR_UNSUPPORTED
    f32 = ssd.make_shape(1024, 256, 80, 64, 1, 128, 256, dtype="f32")  # no fused kernel for fp32
    assert not ssd.path_supported(f32, ssd.PATH_AUTO)


def test_injected_cuda_failure_hook(lib):
    """ssd_test_fail_calls(n): the next n calls that would queue GPU work
    return SSD_ERR_CUDA after their argument checks (which still come first),
    and the binding raises SSDError with that code."""
    s = _shape()
    ok = 1 << 20
    ws = ssd.workspace_size(s)
    lib.ssd_test_fail_calls(3)
    try:
        assert lib.ssd_test_pending_failures() == 3
        # a bad argument is still reported as such, and does not consume the count
        assert lib.ssd_forward(ctypes.byref(s), None, ok, ok, ok, None, ok, None, ok, ws, None) == \
            ssd.SSD_ERR_INVALID_ARG
        assert lib.ssd_test_pending_failures() == 3
        assert lib.ssd_forward(ctypes.byref(s), ok, ok, ok, ok, None, ok, None, ok, ws, None) == \
            ssd.SSD_ERR_CUDA
        assert lib.ssd_chunk_cumsum(ctypes.byref(s), ok, ok, None) == ssd.SSD_ERR_CUDA
        assert lib.ssd_test_pending_failures() == 1
        with pytest.raises(ssd.SSDError) as e:
            ssd._check(lib.ssd_decay_total(ctypes.byref(s), ok, ok, None), "ssd_decay_total")
        assert e.value.code == ssd.SSD_ERR_CUDA
        assert lib.ssd_test_pending_failures() == 0
    finally:
        lib.ssd_test_fail_calls(0)
