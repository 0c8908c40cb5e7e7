"""The canary helpers themselves, on the CPU: a write inside the handed-out
tensor leaves every sentinel intact; a write one element outside it, on
either side or into a padding head, is caught."""

import torch

from tests.canary_util import Canvas, HeadCanvas


def test_canvas_detects_writes_past_either_end():
    for dtype in (torch.bfloat16, torch.float32, torch.uint8):
        c = Canvas((3, 5, 7), dtype, "cpu")
        assert c.t.is_contiguous() and c.t.shape == (3, 5, 7)
        c.t.zero_()
        assert c.intact()
        c.base[c.m + c.n] = 1
        assert not c.intact()
        c = Canvas((3, 5, 7), dtype, "cpu")
        c.base[c.m - 1] = 1
        assert not c.intact()
    c = Canvas((64,), torch.float32, "cpu")
    assert c.t.data_ptr() % 16 == c.base.data_ptr() % 16  # the margin keeps the interior's alignment


def test_head_canvas_detects_writes_into_neighbour_heads():
    c = HeadCanvas(2, 3, 4, 64, "cpu")
    assert c.t.shape == (2, 3, 4, 64) and c.t.stride() == (3 * 6 * 64, 6 * 64, 64, 1)
    c.t.zero_()
    assert c.intact()
    c.base[1, 2, 5, 0] = 1  # the padding head after the last one
    assert not c.intact()
    c = HeadCanvas(2, 3, 4, 64, "cpu")
    c.base[0, 0, 0, 63] = 1  # the padding head before the first one
    assert not c.intact()
