"""The guard-band helpers the GPU tests use instead of a memory sanitizer,
checked on the CPU: writes inside the view leave the guards intact, a write
one element past either end is caught."""
import torch

from tests.helpers import guarded, guards_intact


def test_guard_bands_catch_writes_past_either_end():
    for dtype in (torch.bfloat16, torch.float32):
        buf, t = guarded((2, 3, 5, 16), dtype, "cpu")
        assert t.is_contiguous() and t.shape == (2, 3, 5, 16) and t.dtype == dtype
        assert t.data_ptr() % 16 == buf.data_ptr() % 16
        t.fill_(1.0)
        assert guards_intact(buf)
        flat = buf[4096 - t.element_size():4096 + t.numel() * t.element_size() + t.element_size()].view(dtype)
        flat[-1] = 2.0   # one element past the end
        assert not guards_intact(buf)
        buf2, t2 = guarded((4, 8), dtype, "cpu")
        buf2[4096 - 1] = 0  # one byte before the start
        assert not guards_intact(buf2)
