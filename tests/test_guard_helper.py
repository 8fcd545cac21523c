"""The guard-region helper of the GPU out-of-bounds tests, checked on the CPU: writes that
stay inside the tensor leave the guards intact, and a write one element past either end is
detected; the tensor keeps its shape, dtype and a 256-byte aligned offset."""

import torch

from dsa_testutil import GUARD_BYTES, Guarded


def test_in_bounds_writes_keep_the_guards():
    for shape, dtype in [((4, 128, 512), torch.int16), ((3, 4095), torch.float32),
                         ((7, 2048), torch.int32), ((1000,), torch.uint8)]:
        g = Guarded(shape, dtype, "cpu", fill=0)
        assert tuple(g.t.shape) == shape and g.t.dtype == dtype and g.t.is_contiguous()
        assert (g.t.data_ptr() - g.buf.data_ptr()) == GUARD_BYTES
        assert (g.t.data_ptr() - g.buf.data_ptr()) % 256 == 0
        g.t.view(-1).fill_(7)
        assert g.intact()


def test_writes_past_either_end_are_detected():
    g = Guarded((5, 33), torch.float32, "cpu")
    flat = g.buf[GUARD_BYTES:GUARD_BYTES + g.nbytes + 4].view(torch.float32)
    flat[-1] = 1.0  # one element past the end
    assert not g.intact()
    g = Guarded((5, 33), torch.float32, "cpu")
    g.buf[GUARD_BYTES - 1] = 0  # the byte just before the start
    assert not g.intact()
