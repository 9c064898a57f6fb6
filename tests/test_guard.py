"""The guard-band helper (tests/guard.py) on the CPU: views have the asked
shape and dtype, writes inside the tensor leave the guards alone, and a
write just past either end is seen."""

import pytest
import torch

from tests import guard


@pytest.mark.parametrize("shape,dtype", [((2, 3, 300, 128), torch.bfloat16), ((2, 3, 129), torch.float32),
                                         ((5, 7, 64), torch.float16), ((1000,), torch.uint8)])
def test_guarded_views(shape, dtype):
    t, buf = guard.guarded(shape, dtype, "cpu")
    assert tuple(t.shape) == shape and t.dtype == dtype and t.is_contiguous()
    assert t.data_ptr() - buf.data_ptr() == guard.GUARD and t.data_ptr() % 16 == buf.data_ptr() % 16
    t.fill_(1)
    assert guard.intact(buf)
    end = guard.GUARD + t.numel() * t.element_size()
    buf[end] = 0  # one byte past the end
    assert not guard.intact(buf)
    buf[end] = guard.FILL
    buf[guard.GUARD - 1] = 0  # one byte before the start
    assert not guard.intact(buf)
