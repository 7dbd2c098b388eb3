"""The oracle's codecs against ml_dtypes, an independent library
implementation of the OCP formats: every decode table (E4M3, E2M1, E8M0), and
round-to-nearest-even casts of finite in-range values. ml_dtypes is used only
where its behaviour is the OCP definition: decode, and casts of values inside
the format's range (its saturation and NaN handling are not relied on)."""
import ml_dtypes
import numpy as np
import pytest


def _same(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])


def test_e4m3_decode_table(orc):
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert _same([orc.e4m3_decode(c) for c in range(256)], lib)


def test_e2m1_decode_table(orc):
    lib = np.array([float(ml_dtypes.float4_e2m1fn(v)) for v in
                    [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]])
    ours = np.array([orc.e2m1_decode(c) for c in range(16)])
    assert _same(ours, lib)
    # and the code order: code c decodes to the c-th value above
    assert np.array_equal(np.signbit(ours[8:]), np.ones(8, bool))


def test_e8m0_decode_table(orc):
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert _same([orc.e8m0_value(b) for b in range(256)], lib)


@pytest.mark.parametrize("seed", [0, 1])
def test_e4m3_rne_casts_in_range(orc, seed):
    rng = np.random.default_rng(seed)
    # finite fp32 values of |v| <= 448: random magnitudes over the whole E4M3
    # range, exact code values, and every midpoint between neighbouring codes
    codes = np.arange(0, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = (codes[:-1] + codes[1:]) / 2
    v = np.concatenate([np.exp2(rng.uniform(-14, np.log2(448), 20000)) * rng.choice([-1, 1], 20000),
                        codes, -codes, mids, -mids]).astype(np.float32)
    v = v[np.abs(v) <= 448]
    lib = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ours = orc.e4m3_encode_array(v.astype(np.float64))
    assert np.array_equal(ours, lib)


def test_e2m1_rne_casts_in_range(orc):
    rng = np.random.default_rng(2)
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = (vals[:-1] + vals[1:]) / 2
    v = np.concatenate([rng.uniform(-6, 6, 20000), vals, -vals, mids, -mids]).astype(np.float32)
    lib = np.array([float(ml_dtypes.float4_e2m1fn(x)) for x in v])
    ours = np.array([orc.e2m1_decode(int(c)) for c in orc.e2m1_encode_array(v.astype(np.float64))])
    assert _same(np.abs(ours), np.abs(lib))
    nz = lib != 0
    assert np.array_equal(np.sign(ours[nz]), np.sign(lib[nz]))
