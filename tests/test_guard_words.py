"""The canary-guarded output buffers the GPU tests use catch writes past either end (CPU check)."""
import pytest
import torch

from helpers import CANARY_PAD, Guarded


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.uint8])
def test_guard_words_catch_overruns(dtype):
    g = Guarded((3, 5), dtype, device="cpu")
    g.t.fill_(1)
    g.check("interior writes only")
    assert g.t.data_ptr() % 256 == g._buf.data_ptr() % 256  # the pad keeps the interior's alignment
    g._buf[CANARY_PAD + g._n] = 0  # one byte past the end
    with pytest.raises(AssertionError):
        g.check("overrun")
    g2 = Guarded((4,), dtype, device="cpu")
    g2._buf[CANARY_PAD - 1] = 0  # one byte before the start
    with pytest.raises(AssertionError):
        g2.check("underrun")
