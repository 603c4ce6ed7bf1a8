"""GPU checks of the library's tensor-core GEMM (ttt_gemm_bf16, the kernel
behind the projections and the wide-head path) through the C ABI, against a
float64 product of the same bf16 values.

Every operand layout (A as [M][K] or its transpose, B as [K][N] or its
transpose), ragged M, N and K (a partial 128 x 256 tile, a partial 64-deep K
step), several tiles and waves, and a padded leading dimension.  Bound per
element: one bf16 rounding of the result (half an ulp, 2^-9 relative) plus
FP32 accumulation error, at most K * 2^-24 of sum_k |a_ik b_kj| (generous)."""
import numpy as np
import pytest
import torch

from test_layer_reconstruction_b200 import ttt

pytestmark = pytest.mark.gpu


def _check(M, N, K, a_t, b_t, seed, lda_pad=0):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    ref = A.double() @ B.double()
    mag = A.double().abs() @ B.double().abs()
    Ad = (A.t() if a_t else A).contiguous()
    if lda_pad:
        Ad = torch.nn.functional.pad(Ad, (0, lda_pad))
    Bd = (B.t() if b_t else B).contiguous()
    Ad, Bd = Ad.cuda(), Bd.cuda()
    if lda_pad:
        # a view with the padded row pitch: pass the padded tensor and slice the logical columns
        C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        lib = ttt.load_library()
        import ctypes
        rc = lib.ttt_gemm_bf16(M, N, K, ctypes.c_void_p(Ad.data_ptr()), Ad.shape[1], int(a_t),
                               ctypes.c_void_p(Bd.data_ptr()), Bd.shape[1], int(b_t), ctypes.c_void_p(C.data_ptr()),
                               N, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
    else:
        C = ttt.gemm_bf16(Ad, Bd, a_t=a_t, b_t=b_t)
    torch.cuda.synchronize()
    got = C.double().cpu()
    bound = ref.abs() * 2.0 ** -8 + mag * K * 2.0 ** -24 + 1e-30
    assert torch.all((got - ref).abs() <= bound), float(((got - ref).abs() / bound).max())


@pytest.mark.parametrize("a_t,b_t", [(False, False), (False, True), (True, False), (True, True)])
def test_every_layout_ragged(a_t, b_t):
    _check(296, 264, 200, a_t, b_t, seed=1)


@pytest.mark.parametrize("a_t,b_t", [(False, False), (True, True)])
def test_several_waves(a_t, b_t):
    _check(2176, 1024, 1024, a_t, b_t, seed=2)


def test_single_element_and_tiny_k():
    _check(1, 8, 8, False, False, seed=3)
    _check(8, 16, 3, True, False, seed=4)


def test_padded_leading_dimension():
    _check(130, 64, 72, False, True, seed=5, lda_pad=8)


def test_bad_arguments_are_refused():
    A = torch.zeros(4, 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ttt.TTTError) as e:
        ttt.gemm_bf16(A, torch.zeros(8, 6, dtype=torch.bfloat16, device="cuda"))   # N not a multiple of 8
    assert e.value.status == -2
