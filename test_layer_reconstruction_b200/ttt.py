"""Python binding of the C ABI in include/ttt.h (argument marshalling only).

Every step of the layer runs in the CUDA kernels of libttt.so; PyTorch only
provides device memory and the current stream.  There is no fallback: if the
library is not built, or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple, Union

import torch

from .inputs import LayerConfig

__all__ = [
    "TTTError", "Dims", "library_path", "load_library", "workspace_bytes", "make_workspace",
    "shortconv2d", "write", "grad", "sgd_update", "read", "layer", "layer_host", "check_status",
    "write_muon", "layer_muon", "grad_dot", "muon_update",
    "OP_WRITE", "OP_READ", "OP_LAYER", "OP_LAYER_HOST", "OP_ATTENTION", "INNER_SGD", "INNER_MUON",
    "attention", "gemm_bf16", "set_wait_limit", "EXPORTED_SYMBOLS", "profile_start", "profile_stop",
]

OP_WRITE, OP_READ, OP_LAYER, OP_LAYER_HOST, OP_ATTENTION = 0, 1, 2, 3, 4
INNER_SGD, INNER_MUON = 0, 1
EXPORTED_SYMBOLS = ("ttt_workspace_bytes", "ttt_shortconv2d", "ttt_write", "ttt_read", "ttt_layer",
                    "ttt_layer_host", "ttt_check_status", "ttt_status_str", "ttt_profile_start",
                    "ttt_profile_stop", "ttt_kernel_name", "ttt_read_noalloc", "ttt_read_noalloc_status",
                    "ttt_grad", "ttt_sgd_update", "ttt_write_muon", "ttt_layer_muon", "ttt_grad_dot",
                    "ttt_muon_update", "ttt_attention", "ttt_gemm_bf16", "ttt_set_wait_limit")
KERNEL_KINDS = 12


class KernelTimes(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int32 * KERNEL_KINDS), ("total_ms", ctypes.c_float * KERNEL_KINDS),
                ("dropped", ctypes.c_int32)]


class Dims(ctypes.Structure):
    """ttt_dims: token layout and fast-weight shape."""
    _fields_ = [("n_views", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("n_special", ctypes.c_int32), ("heads", ctypes.c_int32), ("d", ctypes.c_int32),
                ("h", ctypes.c_int32)]

    @classmethod
    def of(cls, x: Union["Dims", LayerConfig, dict]) -> "Dims":
        if isinstance(x, Dims):
            return x
        if isinstance(x, LayerConfig):
            x = x.dims()
        return cls(**{k: int(x[k]) for k in ("n_views", "grid_h", "grid_w", "n_special", "heads", "d", "h")})

    @property
    def n(self) -> int:
        return self.n_views * (self.n_special + self.grid_h * self.grid_w)


class TTTError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


_LIB: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libttt.so")


def load_library() -> ctypes.CDLL:
    """Load libttt.so (built by ``python -m test_layer_reconstruction_b200.build``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m test_layer_reconstruction_b200.build`")
    lib = ctypes.CDLL(path)
    P, S, F, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float, ctypes.c_int
    DP = ctypes.POINTER(Dims)
    lib.ttt_workspace_bytes.argtypes = [DP, I]
    lib.ttt_workspace_bytes.restype = S
    lib.ttt_shortconv2d.argtypes = [DP, P, P, P, P]
    lib.ttt_write.argtypes = [DP, P, P, P, P, F, I, P, P, S, P]
    lib.ttt_read.argtypes = [DP, P, P, P, P, S, P]
    lib.ttt_grad.argtypes = [DP, P, P, P, P, P, S, P]
    lib.ttt_sgd_update.argtypes = [DP, P, P, I, F, P, P]
    lib.ttt_write_muon.argtypes = [DP, P, P, P, P, F, I, P, P, S, P]
    lib.ttt_layer_muon.argtypes = [DP, P, P, P, P, P, F, I, P, P, P, S, P]
    lib.ttt_grad_dot.argtypes = [DP, P, P, P, P, P, S, P]
    lib.ttt_muon_update.argtypes = [DP, P, P, I, F, P, P]
    lib.ttt_layer.argtypes = [DP, P, P, P, P, P, F, I, P, P, P, S, P]
    lib.ttt_layer_host.argtypes = [DP, P, P, P, P, P, F, I, P, P, P, S, P]
    lib.ttt_attention.argtypes = [DP, P, P, P, P, P, P, P, F, I, I, P, P, P, S, P]
    L64 = ctypes.c_int64
    lib.ttt_gemm_bf16.argtypes = [I, I, I, P, L64, I, P, L64, I, P, L64, P]
    lib.ttt_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.ttt_check_status.argtypes = [P, P]
    lib.ttt_status_str.argtypes = [I]
    lib.ttt_status_str.restype = ctypes.c_char_p
    lib.ttt_read_noalloc.argtypes = [DP, P, P, P, P]
    lib.ttt_read_noalloc.restype = I
    lib.ttt_read_noalloc_status.argtypes = [P]
    lib.ttt_read_noalloc_status.restype = I
    lib.ttt_profile_start.argtypes = []
    lib.ttt_profile_stop.argtypes = [ctypes.POINTER(KernelTimes)]
    lib.ttt_kernel_name.argtypes = [I]
    lib.ttt_kernel_name.restype = ctypes.c_char_p
    for f in ("ttt_shortconv2d", "ttt_write", "ttt_read", "ttt_layer", "ttt_layer_host", "ttt_check_status",
              "ttt_profile_start", "ttt_profile_stop", "ttt_grad", "ttt_sgd_update", "ttt_write_muon",
              "ttt_layer_muon", "ttt_grad_dot", "ttt_muon_update", "ttt_attention", "ttt_gemm_bf16",
              "ttt_set_wait_limit"):
        getattr(lib, f).restype = I
    _LIB = lib
    return lib


def status_str(status: int) -> str:
    try:
        return load_library().ttt_status_str(status).decode()
    except Exception:  # pragma: no cover
        return "unknown"


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise TTTError(rc, what)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def workspace_bytes(dims, op: int) -> int:
    return int(load_library().ttt_workspace_bytes(ctypes.byref(Dims.of(dims)), op))


def make_workspace(dims, op: int, device="cuda") -> torch.Tensor:
    nb = workspace_bytes(dims, op)
    if nb == 0:
        raise TTTError(-3, "ttt_workspace_bytes")
    return torch.empty(nb, dtype=torch.uint8, device=device)


def shortconv2d(V: torch.Tensor, conv_w: torch.Tensor, dims, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """V' = ShortConv2D(V); V, out: bf16 [n, heads, d]; conv_w: f32 [heads*d, 3, 3]."""
    dm = Dims.of(dims)
    out = torch.empty_like(V) if out is None else out
    _check(load_library().ttt_shortconv2d(ctypes.byref(dm), _dev(V, torch.bfloat16, "V"),
                                          _dev(conv_w, torch.float32, "conv_w"),
                                          _dev(out, torch.bfloat16, "out"), _stream()), "ttt_shortconv2d")
    return out


def write(K, V, conv_w, theta0, lr: float, steps: int, dims, theta_out=None, workspace=None) -> torch.Tensor:
    """theta* after `steps` SGD steps on the TTT loss (Eq. 3); returns theta_out."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta0) if theta_out is None else theta_out
    ws = make_workspace(dm, OP_WRITE, K.device) if workspace is None else workspace
    _check(load_library().ttt_write(ctypes.byref(dm), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V"),
                                    _dev(conv_w, torch.float32, "conv_w"), _dev(theta0, torch.float32, "theta0"),
                                    float(lr), int(steps), _dev(theta_out, torch.float32, "theta_out"),
                                    ws.data_ptr(), ws.numel(), _stream()), "ttt_write")
    return theta_out


def grad(K, Vp, theta, dims, out=None, workspace=None) -> torch.Tensor:
    """d/dtheta of (1/2) sum_i ||T_theta(k_i) - v'_i||^2 over the tokens of (K, Vp) (Eq. 5 summand sum)."""
    dm = Dims.of(dims)
    out = torch.empty_like(theta) if out is None else out
    ws = make_workspace(dm, OP_WRITE, K.device) if workspace is None else workspace
    _check(load_library().ttt_grad(ctypes.byref(dm), _dev(K, torch.bfloat16, "K"), _dev(Vp, torch.bfloat16, "Vp"),
                                   _dev(theta, torch.float32, "theta"), _dev(out, torch.float32, "grad"),
                                   ws.data_ptr(), ws.numel(), _stream()), "ttt_grad")
    return out


def sgd_update(theta_in, grads, scale: float, dims, theta_out=None) -> torch.Tensor:
    """theta_out = theta_in - scale * sum_r grads[r] (rows of `grads` summed in order); returns theta_out."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta_in) if theta_out is None else theta_out
    if grads.numel() % theta_in.numel() != 0:
        raise ValueError("grads must hold whole gradients of theta's size")
    n_grads = grads.numel() // theta_in.numel()
    _check(load_library().ttt_sgd_update(ctypes.byref(dm), _dev(theta_in, torch.float32, "theta_in"),
                                         _dev(grads, torch.float32, "grads"), int(n_grads), float(scale),
                                         _dev(theta_out, torch.float32, "theta_out"), _stream()), "ttt_sgd_update")
    return theta_out


def write_muon(K, V, conv_w, theta0, lr: float, steps: int, dims, theta_out=None, workspace=None) -> torch.Tensor:
    """theta* after `steps` Muon steps on the dot-product loss (the pages' inner loop)."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta0) if theta_out is None else theta_out
    ws = make_workspace(dm, OP_WRITE, K.device) if workspace is None else workspace
    _check(load_library().ttt_write_muon(ctypes.byref(dm), _dev(K, torch.bfloat16, "K"),
                                         _dev(V, torch.bfloat16, "V"), _dev(conv_w, torch.float32, "conv_w"),
                                         _dev(theta0, torch.float32, "theta0"), float(lr), int(steps),
                                         _dev(theta_out, torch.float32, "theta_out"), ws.data_ptr(), ws.numel(),
                                         _stream()), "ttt_write_muon")
    return theta_out


def layer_muon(Q, K, V, conv_w, theta0, lr: float, steps: int, dims, theta_out=None, O=None,
               workspace=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The layer with the pages' inner loop (dot-product loss, Muon); returns (theta*, O)."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta0) if theta_out is None else theta_out
    O = torch.empty_like(Q) if O is None else O
    ws = make_workspace(dm, OP_LAYER, Q.device) if workspace is None else workspace
    _check(load_library().ttt_layer_muon(ctypes.byref(dm), _dev(Q, torch.bfloat16, "Q"),
                                         _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V"),
                                         _dev(conv_w, torch.float32, "conv_w"), _dev(theta0, torch.float32, "theta0"),
                                         float(lr), int(steps), _dev(theta_out, torch.float32, "theta_out"),
                                         _dev(O, torch.bfloat16, "O"), ws.data_ptr(), ws.numel(), _stream()),
           "ttt_layer_muon")
    return theta_out, O


def grad_dot(K, Vp, theta, dims, out=None, workspace=None) -> torch.Tensor:
    """d/dtheta of -sum_i <T_theta(k_i), v'_i> over the tokens of (K, Vp)."""
    dm = Dims.of(dims)
    out = torch.empty_like(theta) if out is None else out
    ws = make_workspace(dm, OP_WRITE, K.device) if workspace is None else workspace
    _check(load_library().ttt_grad_dot(ctypes.byref(dm), _dev(K, torch.bfloat16, "K"),
                                       _dev(Vp, torch.bfloat16, "Vp"), _dev(theta, torch.float32, "theta"),
                                       _dev(out, torch.float32, "grad"), ws.data_ptr(), ws.numel(), _stream()),
           "ttt_grad_dot")
    return out


def muon_update(theta_in, grads, lr: float, dims, theta_out=None) -> torch.Tensor:
    """theta_out = theta_in - lr * NS5(sum_r grads[r]) per weight matrix; returns theta_out."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta_in) if theta_out is None else theta_out
    if grads.numel() % theta_in.numel() != 0:
        raise ValueError("grads must hold whole gradients of theta's size")
    _check(load_library().ttt_muon_update(ctypes.byref(dm), _dev(theta_in, torch.float32, "theta_in"),
                                          _dev(grads, torch.float32, "grads"), int(grads.numel() // theta_in.numel()),
                                          float(lr), _dev(theta_out, torch.float32, "theta_out"), _stream()),
           "ttt_muon_update")
    return theta_out


def read(Q, theta, dims, O=None, workspace=None) -> torch.Tensor:
    """O = T_theta(Q) (Eq. 4) with frozen theta."""
    dm = Dims.of(dims)
    O = torch.empty_like(Q) if O is None else O
    ws = make_workspace(dm, OP_READ, Q.device) if workspace is None else workspace
    _check(load_library().ttt_read(ctypes.byref(dm), _dev(Q, torch.bfloat16, "Q"),
                                   _dev(theta, torch.float32, "theta"), _dev(O, torch.bfloat16, "O"),
                                   ws.data_ptr(), ws.numel(), _stream()), "ttt_read")
    return O


def layer(Q, K, V, conv_w, theta0, lr: float, steps: int, dims, theta_out=None, O=None,
          workspace=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The whole TTT layer; returns (theta*, O)."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta0) if theta_out is None else theta_out
    O = torch.empty_like(Q) if O is None else O
    ws = make_workspace(dm, OP_LAYER, Q.device) if workspace is None else workspace
    _check(load_library().ttt_layer(ctypes.byref(dm), _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"),
                                    _dev(V, torch.bfloat16, "V"), _dev(conv_w, torch.float32, "conv_w"),
                                    _dev(theta0, torch.float32, "theta0"), float(lr), int(steps),
                                    _dev(theta_out, torch.float32, "theta_out"), _dev(O, torch.bfloat16, "O"),
                                    ws.data_ptr(), ws.numel(), _stream()), "ttt_layer")
    return theta_out, O


def attention(X, Wq, Wk, Wv, Wo, conv_w, theta0, lr: float, steps: int, dims, inner: int = INNER_SGD,
              theta_out=None, out=None, workspace=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The attention layer with the TTT layer inside: q = L2(X Wq), k = L2(X Wk), v = X Wv,
    the layer (inner loop `inner`), out = O Wo.  X, out: bf16 [n, C]; W*: bf16 [C, C].
    Returns (theta*, out)."""
    dm = Dims.of(dims)
    theta_out = torch.empty_like(theta0) if theta_out is None else theta_out
    out = torch.empty_like(X) if out is None else out
    ws = make_workspace(dm, OP_ATTENTION, X.device) if workspace is None else workspace
    _check(load_library().ttt_attention(ctypes.byref(dm), _dev(X, torch.bfloat16, "X"),
                                        _dev(Wq, torch.bfloat16, "Wq"), _dev(Wk, torch.bfloat16, "Wk"),
                                        _dev(Wv, torch.bfloat16, "Wv"), _dev(Wo, torch.bfloat16, "Wo"),
                                        _dev(conv_w, torch.float32, "conv_w"), _dev(theta0, torch.float32, "theta0"),
                                        float(lr), int(steps), int(inner),
                                        _dev(theta_out, torch.float32, "theta_out"), _dev(out, torch.bfloat16, "out"),
                                        ws.data_ptr(), ws.numel(), _stream()), "ttt_attention")
    return theta_out, out


def gemm_bf16(A: torch.Tensor, B: torch.Tensor, a_t: bool = False, b_t: bool = False,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """C = op(A) op(B) on the library's tensor-core GEMM; op(X) = X.T when the flag is set
    (the tensor then holds the transpose).  bf16 in and out, FP32 accumulation."""
    for t, nm in ((A, "A"), (B, "B")):
        if t.dim() != 2:
            raise ValueError(f"{nm} must be 2-D")
    M, K = (A.shape[1], A.shape[0]) if a_t else (A.shape[0], A.shape[1])
    K2, N = (B.shape[1], B.shape[0]) if b_t else (B.shape[0], B.shape[1])
    if K != K2:
        raise ValueError("inner dimensions differ")
    out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device) if out is None else out
    _check(load_library().ttt_gemm_bf16(M, N, K, _dev(A, torch.bfloat16, "A"), A.shape[1], int(a_t),
                                        _dev(B, torch.bfloat16, "B"), B.shape[1], int(b_t),
                                        _dev(out, torch.bfloat16, "out"), out.shape[1], _stream()),
           "ttt_gemm_bf16")
    return out


def _host(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor of {dtype}")
    return t.data_ptr()


def layer_host(Q, K, V, conv_w, theta0, lr: float, steps: int, dims, theta_out, O, workspace) -> None:
    """ttt_layer on host (preferably pinned) tensors; enqueued on the current stream."""
    dm = Dims.of(dims)
    _check(load_library().ttt_layer_host(ctypes.byref(dm), _host(Q, torch.bfloat16, "Q"),
                                         _host(K, torch.bfloat16, "K"), _host(V, torch.bfloat16, "V"),
                                         _host(conv_w, torch.float32, "conv_w"),
                                         _host(theta0, torch.float32, "theta0"), float(lr), int(steps),
                                         _host(theta_out, torch.float32, "theta_out"),
                                         _host(O, torch.bfloat16, "O"), workspace.data_ptr(), workspace.numel(),
                                         _stream()), "ttt_layer_host")


def check_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream and return the workspace's device status (0 = ok)."""
    return int(load_library().ttt_check_status(ctypes.c_void_p(workspace.data_ptr()), _stream()))


def set_wait_limit(clocks: int) -> None:
    """Limit (SM clocks) of every bounded wait in kernels launched from now on; 0 = built-in."""
    _check(load_library().ttt_set_wait_limit(int(clocks)), "ttt_set_wait_limit")


def profile_start() -> None:
    """Start recording a CUDA event pair around every kernel the library launches."""
    _check(load_library().ttt_profile_start(), "ttt_profile_start")


def profile_stop() -> dict:
    """Stop recording; return {kernel name: {"launches": L, "total_ms": T}} (synchronises the events)."""
    lib = load_library()
    kt = KernelTimes()
    _check(lib.ttt_profile_stop(ctypes.byref(kt)), "ttt_profile_stop")
    out = {lib.ttt_kernel_name(k).decode(): {"launches": int(kt.launches[k]), "total_ms": float(kt.total_ms[k])}
           for k in range(KERNEL_KINDS)}
    out["_dropped"] = int(kt.dropped)
    return out
