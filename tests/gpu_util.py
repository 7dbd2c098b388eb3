"""Helpers for the GPU parity tests: host<->device moves and byte-exact
comparison with a readable report of the first mismatches."""
import numpy as np
import torch


def dev(a: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> bf16 CUDA tensor; float32 -> fp32."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    if a.dtype == np.uint8:
        return torch.from_numpy(a).cuda()
    assert a.dtype == np.float32
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy: uint8 as is, bf16 as uint16 bits, fp32 as uint32 bits."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def assert_same(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got)
    want = np.asarray(want)
    if want.dtype == np.float32:
        want = want.view(np.uint32)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        n = bad.shape[0]
        show = [(tuple(int(i) for i in b), int(got[tuple(b)]), int(want[tuple(b)]))
                for b in bad[:8]]
        raise AssertionError(f"{what}: {n} mismatching entries; first (index, gpu, oracle): {show}")
