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


class GuardedAllocator:
    """Output allocator for the binding's ``set_output_allocator`` hook that
    places every buffer between two guard bands of ``BAND`` canary bytes
    inside one larger allocation. A kernel that writes past either end of an
    output lands in a band of the same allocation, which does not fault;
    ``check()`` then finds the changed canary bytes. This is the bounds check
    that runs in place of a memory checker tool.

    The band is a multiple of 256 bytes, so the inner view keeps the
    allocation's alignment."""

    BAND = 4096
    CANARY = 0xA5

    def __init__(self, hold_bytes: int = 8 << 30):
        self.bufs = []          # (uint8 buffer, inner bytes, description)
        self.held = 0
        self.hold_bytes = hold_bytes
        self.checked = 0

    def __call__(self, shape, dtype, device):
        itemsize = torch.empty((), dtype=dtype).element_size()
        n = itemsize
        for d in shape:
            n *= int(d)
        if self.held + n > self.hold_bytes:
            self.check()
        buf = torch.full((2 * self.BAND + n,), self.CANARY, dtype=torch.uint8, device=device)
        self.bufs.append((buf, n, f"{tuple(shape)} {dtype}"))
        self.held += n
        return buf[self.BAND:self.BAND + n].view(dtype).view(shape)

    def check(self):
        """Raises if any guard byte of a buffer allocated so far changed;
        releases the buffers."""
        if torch.cuda.is_available():
            torch.cuda.synchronize()
        bad = []
        for buf, n, what in self.bufs:
            bands = torch.cat((buf[:self.BAND], buf[self.BAND + n:]))
            hit = torch.nonzero(bands != self.CANARY).flatten()
            if hit.numel():
                first = int(hit[0])
                where = (f"{self.BAND - first} bytes before" if first < self.BAND
                         else f"{first - self.BAND + 1} bytes after")
                bad.append(f"{what}: {hit.numel()} guard bytes changed, first {where} the buffer")
        self.checked += len(self.bufs)
        self.bufs, self.held = [], 0
        if bad:
            raise AssertionError("write outside an output buffer: " + "; ".join(bad))


def guarded_empty(alloc: GuardedAllocator, shape, dtype, device="cuda") -> torch.Tensor:
    """A tensor from ``alloc`` for tests that call the C ABI directly."""
    return alloc(tuple(shape), dtype, torch.device(device))


def oracle_map(fn, items, threads=None):
    """[fn(item) for item in items] on host threads. The oracle's C calls
    release the interpreter lock (ctypes), so the single-threaded oracle runs
    on several cores at once, one item per call."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    items = list(items)
    n = threads or max(1, min(32, len(os.sched_getaffinity(0)), len(items)))
    with ThreadPoolExecutor(n) as ex:
        return list(ex.map(fn, items))
