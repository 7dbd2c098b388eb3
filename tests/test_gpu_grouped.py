"""Grouped MX quantize (one launch over a stack of expert weights) on the GPU,
bit-exact against the oracle's per-expert quantize: the stacked call with
device row offsets (and its per-expert swizzled scales), the pointer-list
call, and the single-tensor call on the flattened stack."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, guarded_empty, host, oracle_map

pytestmark = pytest.mark.gpu


@pytest.mark.slow
def test_expert_stack_full_size():
    """64 experts of 2048 x 7168: every expert's codes, scales and swizzled
    scales against the oracle, through the stacked call, the pointer-list call
    and the flattened single-tensor call."""
    xs = W.experts()                                  # [64, 2048, 7168] bf16
    want = oracle_map(lambda x: oracle.mxfp8_quantize(x), xs)
    xd = dev(xs)
    q, s, z = mxq.mxfp8_quantize_grouped(xd, swizzled=True)
    assert q.shape == (64, 2048, 7168) and s.shape == (64, 2048, 224)
    qh, sh, zh = host(q), host(s), host(z)
    blk = 2048 * 224
    for e, (qo, so) in enumerate(want):
        assert_same(qh[e], qo, f"expert {e} qweight")
        assert_same(sh[e], so, f"expert {e} scale")
        assert_same(zh[e * blk:(e + 1) * blk], oracle.swizzle_scales(so), f"expert {e} swizzled")
    del q, s, z
    qf, sf = mxq.mxfp8_quantize(xd.view(-1, 7168))
    qfh, sfh = host(qf).reshape(64, 2048, 7168), host(sf).reshape(64, 2048, 224)
    for e, (qo, so) in enumerate(want):
        assert_same(qfh[e], qo, f"flattened call, expert {e} qweight")
        assert_same(sfh[e], so, f"flattened call, expert {e} scale")
    del qf, sf
    ql, sl = mxq.mxfp8_quantize_grouped(list(xd.unbind(0)))
    qlh, slh = host(ql).reshape(64, 2048, 7168), host(sl).reshape(64, 2048, 224)
    for e, (qo, so) in enumerate(want):
        assert_same(qlh[e], qo, f"pointer-list call, expert {e} qweight")
        assert_same(slh[e], so, f"pointer-list call, expert {e} scale")


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("offsets_on_device", [False, True])
def test_stacked_ragged_offsets_with_empty_experts(fmt, offsets_on_device):
    rows = [3, 0, 257, 1, 0, 64, 1000, 128, 0]
    N = 192
    parts = [W.linear_weight(seed=100 + i, M=max(r, 1), N=N)[:r] for i, r in enumerate(rows)]
    x = np.concatenate(parts, 0)
    offs = np.concatenate([[0], np.cumsum(rows)]).astype(np.int64)
    ro = torch.from_numpy(offs).cuda() if offsets_on_device else offs.tolist()
    quant = mxq.mxfp8_quantize_grouped if fmt == "mxfp8" else mxq.mxfp4_quantize_grouped
    oq = oracle.mxfp8_quantize_grouped if fmt == "mxfp8" else oracle.mxfp4_quantize_grouped
    qo, so, zo = oq(parts, swizzled=True)
    q, s = quant(dev(x), row_offsets=ro)
    assert_same(host(q), qo, f"{fmt} stacked codes")
    assert_same(host(s), so, f"{fmt} stacked scales")
    q, s, z = quant(dev(x), row_offsets=ro, swizzled=True)
    assert_same(host(q), qo, f"{fmt} stacked codes (swizzled call)")
    assert_same(host(s), so, f"{fmt} stacked scales (swizzled call)")
    # with device offsets the buffer is sized by the bound; the rest is unwritten
    assert_same(host(z)[:zo.size], zo, f"{fmt} per-expert swizzled scales")


def test_stacked_fp32_and_odd_scale_columns():
    rows = [40, 0, 129, 7]
    N = 32 * 7                                        # 7 scale columns: one padding column
    rng = np.random.default_rng(61)
    parts = [(rng.standard_t(3, (r, N)) * 0.5).astype(np.float32) for r in rows]
    x = np.concatenate(parts, 0)
    offs = np.concatenate([[0], np.cumsum(rows)]).tolist()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    qo, so, zo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    assert_same(host(q), qo, "fp32 stacked codes")
    assert_same(host(s), so, "fp32 stacked scales")
    assert_same(host(z), zo, "fp32 per-expert swizzled scales")


@pytest.mark.parametrize("S", [132, 256, 4])
def test_stacked_swizzle_through_the_staged_tile(S):
    """Scale widths with S % 4 == 0 go through the gather's shared-memory tile
    in chunks of 128 columns: S = 132 gives a full chunk and a 4-column
    remainder, S = 256 two full chunks, S = 4 one 4-column chunk. Ragged
    experts (one empty, partial 128-row blocks) and the single-tensor form of
    the same gather on the whole stack."""
    rows = [130, 0, 1, 255, 128, 3]
    N = 32 * S
    parts = [W.linear_weight(seed=300 + i, M=max(r, 1), N=N)[:r] for i, r in enumerate(rows)]
    x = np.concatenate(parts, 0)
    offs = np.concatenate([[0], np.cumsum(rows)]).tolist()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    qo, so, zo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    assert_same(host(q), qo, f"S={S} stacked codes")
    assert_same(host(s), so, f"S={S} stacked scales")
    assert_same(host(z), zo, f"S={S} per-expert swizzled scales")
    assert_same(host(mxq.swizzle_scales(s)), oracle.swizzle_scales(so), f"S={S} whole-stack swizzle")


def _stacked_swizzled_raw():
    f = ctypes.CDLL(mxq.library_path).mxfp8_quantize_grouped_swizzled
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [vp, i32, i32, vp, i64, i64, vp, vp, vp, i64, vp]
    f.restype = i32
    return f


def test_offsets_outside_the_rules_are_clamped(guard_bands):
    """Device offsets that fall back or pass M_total act as their clamped,
    non-decreasing form, and an undersized swizzled buffer is not written
    past its end (the guard bands around it stay intact)."""
    f = _stacked_swizzled_raw()
    M, N = 100, 64
    x = W.linear_weight(seed=70, M=M, N=N)
    bad = torch.tensor([7, 50, 30, 200, -5], dtype=torch.int64, device="cuda")
    clamped = [0, 50, 50, 100, 100]                   # entries 0 and E taken as 0 and M
    parts = [x[a:b] for a, b in zip(clamped[:-1], clamped[1:])]
    qo, so, zo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    xd = dev(x)
    sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for cap in (zo.size, zo.size // 2 + 3):
        q = guarded_empty(guard_bands, (M, N), torch.uint8)
        s = guarded_empty(guard_bands, (M, N // 32), torch.uint8)
        z = guarded_empty(guard_bands, (cap,), torch.uint8)
        st = f(ctypes.c_void_p(xd.data_ptr()), 0, 4, ctypes.c_void_p(bad.data_ptr()), M, N,
               ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(s.data_ptr()),
               ctypes.c_void_p(z.data_ptr()), cap, sp)
        assert st == 0
        assert_same(host(q), qo, "codes")
        assert_same(host(s), so, "scales")
        assert_same(host(z), zo[:cap], f"swizzled scales, {cap}-byte buffer")
        guard_bands.check()


def test_ragged_list_with_empty_experts():
    rows = [3, 0, 257, 1, 0, 64, 1000]
    xs = [W.linear_weight(seed=100 + i, M=max(r, 1), N=192)[:r] for i, r in enumerate(rows)]
    q, s = mxq.mxfp8_quantize_grouped([dev(x) for x in xs])
    qo, so = oracle.mxfp8_quantize_grouped(xs)
    assert_same(host(q), qo, "ragged qweight")
    assert_same(host(s), so, "ragged scale")


def test_many_experts_and_fp32():
    xs = [(np.random.default_rng(200 + e).standard_normal((e % 7 + 1, 64)) * (e + 1)).astype(np.float32)
          for e in range(100)]
    q, s = mxq.mxfp8_quantize_grouped([dev(x) for x in xs])
    qo, so = oracle.mxfp8_quantize_grouped(xs)
    assert_same(host(q), qo, "100 experts qweight")
    assert_same(host(s), so, "100 experts scale")
    x = np.concatenate(xs, 0)
    offs = np.concatenate([[0], np.cumsum([a.shape[0] for a in xs])]).tolist()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    qo, so, zo = oracle.mxfp8_quantize_grouped(xs, swizzled=True)
    assert_same(host(q), qo, "100 stacked experts qweight")
    assert_same(host(z), zo, "100 stacked experts swizzled")


def test_max_experts_stacked():
    E = 1024
    rows = [(e * 37) % 5 for e in range(E)]
    parts = [W.linear_weight(seed=7, M=max(r, 1), N=64)[:r] for r in rows]
    x = np.concatenate(parts, 0)
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(rows)]).astype(np.int64)).cuda()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    qo, so, zo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    assert_same(host(q), qo, "1024 experts qweight")
    assert_same(host(s), so, "1024 experts scale")
    assert_same(host(z)[:zo.size], zo, "1024 experts swizzled")


def test_single_expert_matches_plain_call():
    x = W.planted()
    qg, sg = mxq.mxfp8_quantize_grouped([dev(x)])
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(host(qg), qo, "E=1 qweight")
    assert_same(host(sg), so, "E=1 scale")


def test_too_many_experts_rejected():
    x = torch.zeros(1, 32, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_quantize_grouped([x] * 1025)
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_quantize_grouped(torch.zeros(1025, 1, 32, dtype=torch.bfloat16, device="cuda"))
