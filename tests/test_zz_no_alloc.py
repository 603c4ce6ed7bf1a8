"""ttt_read_noalloc: the read for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (an allocator that forbids new device
allocations, or all device memory already handed to a pool the caller does
not control).  For them the library offers a read whose scratch is a fixed
array inside the library.  This test calls it through the C ABI twice in a
row and checks each result against ttt_read with a caller-allocated
workspace, reads the call's device status through ttt_read_noalloc_status
after each call, checks that the second call allocates no device memory
through the caller's allocator, and checks that shapes beyond the fixed
scratch are refused before anything runs.  It lives in its own file,
collected last, and passes alone or after the other tests.
"""
import ctypes

import pytest
import torch

from test_layer_reconstruction_b200 import inputs as tin
from test_layer_reconstruction_b200 import ttt
from ttt_testlib import TOL_O, bf16_inputs, normwise, to_device

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(lib, cfg, Q, theta, O):
    dm = ttt.Dims.of(cfg)
    return lib.ttt_read_noalloc(ctypes.byref(dm), ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(theta.data_ptr()),
                                ctypes.c_void_p(O.data_ptr()), _stream())


def test_read_noalloc_matches_read_twice():
    lib = ttt.load_library()
    cases = [tin.LayerConfig("na1", 3, 37, 37, 5, 4, 64, 256, 1, 0.1, 21),
             tin.LayerConfig("na2", 2, 8, 8, 0, 1, 16, 32, 1, 0.1, 22)]
    for cfg in cases:
        inp = bf16_inputs(tin.make_inputs(cfg))
        dev = to_device(inp)
        ref = ttt.read(dev["Q"], dev["theta"], cfg).float().cpu().numpy()
        outs = [torch.full_like(dev["Q"], float("nan")) for _ in range(2)]
        torch.cuda.synchronize()
        for i, O in enumerate(outs):
            before = torch.cuda.memory_allocated()
            assert _noalloc(lib, cfg, dev["Q"], dev["theta"], O) == 0
            assert lib.ttt_read_noalloc_status(_stream()) == 0
            if i == 1:
                # the first call on a device may set up the array's address; later ones allocate nothing
                assert torch.cuda.memory_allocated() == before
            got = O.float().cpu().numpy()
            assert normwise(got, ref) <= TOL_O


def test_read_noalloc_rejects_shapes_beyond_its_scratch():
    lib = ttt.load_library()
    # 64 heads x (W13 + W2 bf16 images of 256 x 64) = 6 MiB > 4 MiB of fixed scratch
    cfg = tin.LayerConfig("na_big", 1, 2, 2, 0, 64, 64, 256, 1, 0.1, 23)
    Q = torch.zeros(cfg.n, cfg.heads, cfg.d, dtype=torch.bfloat16, device="cuda")
    theta = torch.zeros(3 * cfg.heads * cfg.d * cfg.h, dtype=torch.float32, device="cuda")
    O = torch.empty_like(Q)
    assert _noalloc(lib, cfg, Q, theta, O) == -4
    assert lib.ttt_read_noalloc_status(_stream()) == 0
