"""The guard-region helper used by the GPU out-of-bounds tests, checked on the CPU: a view
keeps its shape, dtype and alignment, writes inside it leave the guards intact, and one
element written just past either end is caught."""
import pytest

from _canary import GUARD, PATTERN, guarded_empty, guards_intact

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.uint8])
@pytest.mark.parametrize("shape", [(7, 3, 40), (13, 24), (1,), (0, 24)])
def test_view_shape_alignment_and_clean_writes(dtype, shape):
    buf, v = guarded_empty(shape, dtype, "cpu")
    assert tuple(v.shape) == shape and v.dtype == dtype and v.is_contiguous()
    if v.numel():                                # an empty view reports a null data pointer
        assert (v.data_ptr() - buf.data_ptr()) == GUARD and v.data_ptr() % 16 == buf.data_ptr() % 16
    assert guards_intact(buf)
    v.fill_(3)                                   # every byte of the output written
    assert guards_intact(buf)
    assert (buf.view(torch.uint8)[:GUARD] == PATTERN).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_one_element_past_either_end_is_caught(dtype):
    es = torch.empty((), dtype=dtype).element_size()
    g = GUARD // es
    for where in (g - 1, g + 5 * 24):            # just before the view, just after it
        buf, v = guarded_empty((5, 24), dtype, "cpu")
        v.fill_(1)
        buf[where] = 2
        assert not guards_intact(buf), where


def test_far_writes_inside_the_guard_are_caught():
    buf, v = guarded_empty((4, 8), torch.float32, "cpu")
    buf.view(torch.uint8)[-1] = 0
    assert not guards_intact(buf)
    buf, v = guarded_empty((4, 8), torch.float32, "cpu")
    buf.view(torch.uint8)[0] = 0
    assert not guards_intact(buf)
