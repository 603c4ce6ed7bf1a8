"""The guard-band helpers of the GPU canary tests, checked on CPU with fake
writers: an in-bounds writer leaves the canaries intact, a one-element
overrun on either side is detected, and payloads keep the 256-byte alignment
the library's workspace needs."""
import torch

from ttt_testlib import GUARD, guarded, guards_intact


def test_in_bounds_write_keeps_guards_and_poison_is_overwritten():
    out, buf = guarded((3, 5, 8), torch.bfloat16, "cpu", fill=float("nan"))
    assert torch.isnan(out.float()).all()
    out.copy_(torch.ones_like(out))
    assert guards_intact(buf) and not torch.isnan(out.float()).any()


def test_overrun_on_either_side_is_detected():
    for shift in (-1, 1):
        out, buf = guarded((4, 4), torch.float32, "cpu")
        flat = buf.view(torch.uint8)
        if shift < 0:
            flat[GUARD - 1] = 0
        else:
            flat[GUARD + out.numel() * 4] = 0
        assert not guards_intact(buf)


def test_payload_alignment():
    out, buf = guarded((1000,), torch.uint8, "cpu")
    assert (out.data_ptr() - buf.data_ptr()) % 256 == 0
