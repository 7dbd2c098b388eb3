"""The NVFP4 block pass decides E2M1 codes without a division: with r an
approximate reciprocal of eff (within 1 ulp of 1/eff, the documented bound of
rcp.approx.f32), it takes lo = fl(x * fl(r (1 - 2^-20))) and
hi = fl(x * fl(r (1 + 2^-20))); when E2M1(lo) == E2M1(hi) that code is used,
otherwise the block is recomputed with IEEE divisions. This checks on the CPU,
in fp32 arithmetic, that an agreeing bracket always gives the oracle's
E2M1(fl(x / eff)), for fp32- and bf16-like numerators placed at and around
every midpoint, and that exact ties never agree (so they always take the exact
path)."""
import numpy as np

MID = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def f32(v):
    return np.float32(v)


def test_agreeing_bracket_equals_oracle(orc):
    rng = np.random.default_rng(0)
    agreed = split = ties = 0
    for _ in range(40000):
        c = int(rng.integers(0, 7))
        eff = f32(np.exp2(rng.uniform(-90, 90)) * rng.uniform(1, 2))
        base = np.array([f32(eff * f32(MID[c]))], np.float32).view(np.uint32)[0]
        if rng.random() < 0.5:      # fp32-like numerator within a few ulps of eff * M
            xb = np.uint32(int(base) + int(rng.integers(-3, 4)))
        else:                       # bf16-like numerator (8 significant bits)
            xb = np.uint32((int(base) & 0xFFFF0000) + (int(rng.integers(0, 3)) << 16))
        x = np.array([xb], np.uint32).view(np.float32)[0] * f32(1 if rng.random() < 0.5 else -1)
        want = orc.e2m1_encode(float(f32(x / eff)))
        r = f32(f32(1.0) / eff)
        rbits = int(np.array([r], np.float32).view(np.uint32)[0]) + int(rng.integers(-1, 2))
        r = np.array([rbits], np.uint32).view(np.float32)[0]      # within 1 ulp
        lo = f32(x * f32(r * f32(0.99999904632568359375)))
        hi = f32(x * f32(r * f32(1.00000095367431640625)))
        cl, ch = orc.e2m1_encode(float(lo)), orc.e2m1_encode(float(hi))
        if f32(x / eff) == f32(MID[c]) * np.sign(x):
            ties += 1
            assert cl != ch, (x, eff)
        if cl == ch:
            agreed += 1
            assert cl == want, (x, eff, r)
        else:
            split += 1
    assert agreed > 10000 and split > 5000 and ties > 100
