"""The guard-byte helper the GPU canary tests use, checked on CPU tensors: a write
inside the buffer leaves the guards intact, a write one byte past either end does not."""
import torch

from tests.harness import Guarded


def test_guards_detect_writes_just_outside():
    for dtype, shape in ((torch.float16, (3, 5, 8)), (torch.uint8, (7, 16)), (torch.int32, (1,))):
        g = Guarded(shape, dtype, "cpu", init=torch.zeros(shape, dtype=dtype))
        assert g.t.shape == shape and g.t.dtype == dtype and g.t.is_contiguous()
        assert g.t.data_ptr() % 256 == g.raw.data_ptr() % 256
        g.t.fill_(1)
        assert g.intact()
        g.raw[Guarded.GUARD - 1] = 0                     # the byte before the buffer
        assert not g.intact()
        g.raw[Guarded.GUARD - 1] = Guarded.PATTERN
        assert g.intact()
        g.raw[Guarded.GUARD + g.n] = 0                   # the byte after it
        assert not g.intact()
