"""The canary-band check that every GPU test runs around its outputs
(tests/gpu_util.GuardedAllocator), exercised on the CPU: writes inside a
buffer pass, a write one byte before or after it is found, and the binding
routes its allocations through the hook."""
import pytest
import torch

from gpu_util import GuardedAllocator


def test_in_bounds_writes_pass():
    a = GuardedAllocator()
    t = a((3, 5), torch.float32, torch.device("cpu"))
    t.fill_(1.0)
    u = a((7,), torch.uint8, torch.device("cpu"))
    u[:] = 0
    a.check()
    assert a.checked == 2


@pytest.mark.parametrize("where", ["before", "after"])
def test_stray_byte_is_found(where):
    a = GuardedAllocator()
    t = a((4, 4), torch.uint8, torch.device("cpu"))
    buf, n, _ = a.bufs[0]
    assert t.data_ptr() == buf.data_ptr() + a.BAND
    if where == "before":
        buf[a.BAND - 1] = 0       # the byte just before the output
    else:
        buf[a.BAND + n] = 0       # the byte just after it
    with pytest.raises(AssertionError, match=f"1 bytes {where}"):
        a.check()


def test_alignment_of_inner_view():
    a = GuardedAllocator()
    t = a((33,), torch.bfloat16, torch.device("cpu"))
    buf = a.bufs[0][0]
    assert (t.data_ptr() - buf.data_ptr()) % 256 == 0


def test_binding_uses_the_hook():
    mxq = pytest.importorskip("nvfp4_block_scaled_sm_b200")
    seen = []

    def alloc(shape, dtype, device):
        seen.append((shape, dtype))
        return torch.empty(shape, dtype=dtype)

    prev = mxq.set_output_allocator(alloc)
    try:
        t = mxq._empty((2, 3), torch.uint8, "cpu")
        z = mxq._zeros(4, torch.float32, "cpu")
    finally:
        assert mxq.set_output_allocator(prev) is alloc
    assert seen == [((2, 3), torch.uint8), ((4,), torch.float32)]
    assert t.shape == (2, 3) and float(z.abs().sum()) == 0.0


def test_nvtx_wrapping_keeps_the_api():
    mxq = pytest.importorskip("nvfp4_block_scaled_sm_b200")
    assert mxq.mxfp8_quantize.__name__ == "mxfp8_quantize"
    assert "MXFP8 rowwise quantize" in mxq.mxfp8_quantize.__doc__
    assert mxq.set_nvtx(False) is False and mxq.set_nvtx(False) is False
