"""Pins of the oracle's NVFP4 quantize with one global scale per slice of rows
("Add FP8, NVFP4, and QARL training and export": per-slice / per-expert
global scales, per-half gate/up scales during QAT, one shared scale per
expert at export).

* Per slice, the torch fp32 formulation (refs.nvfp4_quantize_torch) run on
  that slice's rows alone, concatenated.
* One slice is the single-tensor quantize.
* Power-of-two equivariance: scaling one slice by 2^k scales its global scale
  by 2^k and changes no code, no block scale and no other slice.
* Per-half against shared: the half holding the expert's amax gets the
  shared scale and the shared result; the other half gets a smaller global
  scale and block scales at least as large.
"""
import numpy as np
import pytest

import refs
import workloads as W


def _torch_per_slice(x, rows):
    out_p, out_b, out_g = [], [], []
    r0 = 0
    for r in rows:
        if r:
            p, b, g = refs.nvfp4_quantize_torch(x[r0:r0 + r])
        else:
            p = np.zeros((0, x.shape[1] // 2), np.uint8)
            b = np.zeros((0, x.shape[1] // 16), np.uint8)
            g = np.float32(0)
        out_p.append(p)
        out_b.append(b)
        out_g.append(np.float32(g))
        r0 += r
    return np.concatenate(out_p), np.concatenate(out_b), np.array(out_g, np.float32)


@pytest.mark.parametrize("rows", [[64], [16, 0, 48], [1, 31, 32], [8] * 8])
def test_matches_torch_per_slice(orc, rows):
    x = W.experts(seed=81, E=1, M=sum(rows), N=256)[0]
    p, b, g = orc.nvfp4_quantize_sliced(x, rows)
    pt, bt, gt = _torch_per_slice(x, rows)
    assert np.array_equal(g.view(np.uint32), gt.view(np.uint32))
    assert np.array_equal(b, bt) and np.array_equal(p, pt)


def test_one_slice_is_single_tensor(orc):
    x = W.nvfp4_tensor(seed=82, M=96, N=512)
    p, b, g = orc.nvfp4_quantize_sliced(x, [96])
    p1, b1, g1 = orc.nvfp4_quantize(x)
    assert g[0] == g1 and np.array_equal(p, p1) and np.array_equal(b, b1)
    gs = np.float32([0.0123])
    p, b, _ = orc.nvfp4_quantize_sliced(x, [96], global_scales=gs)
    p1, b1, _ = orc.nvfp4_quantize(x, global_scale=gs[0])
    assert np.array_equal(p, p1) and np.array_equal(b, b1)


def test_power_of_two_equivariance(orc):
    xs = W.experts(seed=83, E=4, M=32, N=128)
    x = xs.reshape(-1, 128)
    rows = [32] * 4
    p, b, g = orc.nvfp4_quantize_sliced(x, rows)
    xf = refs.bf16_bits_to_f64(x)
    xf[32:64] *= 8.0                               # slice 1 times 2^3 (exact in bf16)
    y = W.to_bf16_bits(xf.astype(np.float32))
    p2, b2, g2 = orc.nvfp4_quantize_sliced(y, rows)
    assert g2[1] == np.float32(g[1] * 8)
    assert np.array_equal(np.delete(g2, 1), np.delete(g, 1))
    assert np.array_equal(p2, p) and np.array_equal(b2, b)


def test_slices_are_independent(orc):
    x = W.experts(seed=84, E=3, M=16, N=64).reshape(-1, 64).copy()
    p, b, g = orc.nvfp4_quantize_sliced(x, [16, 16, 16])
    x[20, 5] = W.bits_of([1000.0])[0]              # a new amax inside slice 1
    p2, b2, g2 = orc.nvfp4_quantize_sliced(x, [16, 16, 16])
    assert g2[0] == g[0] and g2[2] == g[2] and g2[1] != g[1]
    keep = np.r_[0:16, 32:48]
    assert np.array_equal(p2[keep], p[keep]) and np.array_equal(b2[keep], b[keep])


def test_per_half_against_shared(orc):
    """Fused gate/up rows of 4 experts, gate and up halves of different
    magnitude: per-half scales (QAT) against one shared scale (export)."""
    E, I, H = 4, 16, 128
    rng = np.random.default_rng(85)
    x = np.empty((E, 2 * I, H), np.float32)
    for e in range(E):
        x[e, :I] = rng.standard_normal((I, H)) * 0.02 * (e + 1)
        x[e, I:] = rng.standard_normal((I, H)) * 0.005 * (e + 1)
    xb = W.to_bf16_bits(x).reshape(-1, H)
    ph, bh, gh = orc.nvfp4_quantize_sliced(xb, [I] * (2 * E))
    ps, bs, gs = orc.nvfp4_quantize_sliced(xb, [2 * I] * E)
    for e in range(E):
        gate = slice(2 * e * I, 2 * e * I + I)
        up = slice(2 * e * I + I, 2 * (e + 1) * I)
        assert gh[2 * e] == gs[e] and gh[2 * e + 1] < gs[e]
        assert np.array_equal(ph[gate], ps[gate]) and np.array_equal(bh[gate], bs[gate])
        assert np.all(bh[up] >= bs[up])              # E4M3 codes of positive scales order like values


def test_bad_slices(orc):
    x = np.zeros((8, 32), np.uint16)
    with pytest.raises(ValueError):
        orc.nvfp4_quantize_sliced(x, [4, 5])
    with pytest.raises(ValueError):
        orc.nvfp4_quantize_sliced(x, [10, -2])
