"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

from test_layer_reconstruction_b200 import build, ttt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ttt.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "ttt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_bound_symbols():
    assert _declared_functions() == sorted(ttt.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(0, -7, -1):
        assert ttt.status_str(code) != "unknown status"
    assert ttt.status_str(-99) == "unknown status"


def _dims(**kw):
    base = dict(n_views=2, grid_h=8, grid_w=8, n_special=0, heads=1, d=16, h=32)
    base.update(kw)
    return ttt.Dims(**base)


FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
FAKE_MIS = ctypes.c_void_p(0x10008)   # 8-byte aligned, not 16


def _write(lib, dims, K=FAKE, ws=FAKE, steps=1):
    return lib.ttt_write(ctypes.byref(dims), K, FAKE, FAKE, FAKE, 0.1, steps, FAKE, ws, 1 << 20, None)


def test_host_validation_codes(lib):
    assert _write(lib, _dims(), K=None) == -1                       # null pointer
    assert _write(lib, _dims(), steps=-1) == -1                     # negative steps
    assert _write(lib, _dims(), K=FAKE_MIS) == -2                   # misaligned
    assert _write(lib, _dims(d=48)) == -3                           # unsupported head width
    assert _write(lib, _dims(h=300)) == -3                          # hidden too wide
    assert _write(lib, _dims(grid_h=0)) == -1                       # empty grid
    assert _write(lib, _dims(), ws=None) == -1                      # no workspace
    assert _write(lib, _dims(), ws=ctypes.c_void_p(0x10010)) == -2  # workspace not 256-aligned
    assert lib.ttt_read(ctypes.byref(_dims()), None, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert lib.ttt_shortconv2d(ctypes.byref(_dims(d=20)), FAKE, FAKE, FAKE, None) == -3
    assert lib.ttt_check_status(None, None) == -1


def test_workspace_bytes_rejects_bad_dims(lib):
    assert lib.ttt_workspace_bytes(ctypes.byref(_dims(d=48)), 0) == 0
    assert lib.ttt_workspace_bytes(ctypes.byref(_dims()), 7) == 0


def test_host_validation_codes_of_the_sharded_muon_and_host_entry_points(lib):
    dm = ctypes.byref(_dims())
    wide = ctypes.byref(_dims(d=128, h=192))
    # gradient passes of the sharded write
    for fn in (lib.ttt_grad, lib.ttt_grad_dot):
        assert fn(dm, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -1
        assert fn(dm, FAKE, FAKE, FAKE_MIS, FAKE, FAKE, 1 << 20, None) == -2
        assert fn(ctypes.byref(_dims(d=48)), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -3
    assert lib.ttt_grad_dot(wide, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == -1   # wide heads take the GEMM path
    # updates
    assert lib.ttt_sgd_update(dm, FAKE, FAKE, 0, 1.0, FAKE, None) == -1               # no gradients
    assert lib.ttt_sgd_update(dm, None, FAKE, 1, 1.0, FAKE, None) == -1
    assert lib.ttt_sgd_update(dm, FAKE, FAKE_MIS, 1, 1.0, FAKE, None) == -2
    assert lib.ttt_muon_update(dm, FAKE, FAKE, 0, 0.1, FAKE, None) == -1
    assert lib.ttt_muon_update(wide, FAKE, FAKE, 1, 0.1, FAKE, None) == -3            # needs a workspace when wide
    # the Muon write and layer
    assert lib.ttt_write_muon(dm, FAKE, FAKE, FAKE, FAKE, 0.1, -1, FAKE, FAKE, 1 << 20, None) == -1
    assert lib.ttt_write_muon(dm, FAKE_MIS, FAKE, FAKE, FAKE, 0.1, 1, FAKE, FAKE, 1 << 20, None) == -2
    assert lib.ttt_write_muon(wide, FAKE, FAKE, FAKE, FAKE, 0.1, -1, FAKE, FAKE, 1 << 20, None) == -1
    assert lib.ttt_layer_muon(dm, None, FAKE, FAKE, FAKE, FAKE, 0.1, 1, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    # a wide layer passes the shape checks; it then stops at the first CUDA query (no device) or at the
    # workspace size (a device), before anything is enqueued
    assert lib.ttt_layer_muon(wide, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 1, FAKE, FAKE, FAKE, 16, None) in (-5, -4)
    # host buffers
    assert lib.ttt_layer_host(dm, None, FAKE, FAKE, FAKE, FAKE, 0.1, 1, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert lib.ttt_layer_host(dm, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, -1, FAKE, FAKE, FAKE, 1 << 20, None) == -1



def test_host_validation_codes_of_the_surround_and_the_gemm(lib):
    d64 = ctypes.byref(_dims(d=64, h=256, heads=2))

    def att(dm, X=FAKE, inner=0, steps=1):
        return lib.ttt_attention(dm, X, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, steps, inner, FAKE, FAKE, FAKE,
                                 1 << 20, None)

    assert att(d64, X=None) == -1
    assert att(d64, steps=-1) == -1
    assert att(d64, inner=2) == -1                                   # unknown inner loop
    assert att(d64, X=FAKE_MIS) == -2
    assert att(ctypes.byref(_dims(d=32, h=64))) == -3                # heads of 64 only
    assert att(ctypes.byref(_dims(d=128, h=192))) == -3              # no wide path
    assert lib.ttt_workspace_bytes(d64, 5) == 0                      # no such op

    def gemm(M=16, N=16, K=16, A=FAKE, lda=16, at=0, ldb=16, bt=0, ldc=16):
        return lib.ttt_gemm_bf16(M, N, K, A, lda, at, FAKE, ldb, bt, FAKE, ldc, None)

    assert gemm(A=None) == -1
    assert gemm(M=0) == -1
    assert gemm(at=2) == -1
    assert gemm(lda=8) == -1                                         # lda < K
    assert gemm(N=12, ldb=16, ldc=16) == -2                          # N not a multiple of 8
    assert gemm(K=20, lda=20, ldb=16) == -2                          # lda not a multiple of 8
    assert gemm(A=FAKE_MIS) == -2
