"""Pins of the oracle's block-scaled MXFP8 product D = A B^T (the definition
the tensor-core GEMM is checked against).

* Identity: B = the E4M3 identity (code 0x38 = 1.0 on the diagonal, scale
  byte 127) gives D = the pinned dequantization of A.
* Closed form: all codes 1.0 gives D[m, n] = 32 * sum_g 2^(sa[m,g] + sb[n,g] - 254).
* Brute force: a scalar triple loop over codes and scale bytes on a tiny case.
* Transpose: swapping the operands transposes D.
"""
import numpy as np

import workloads as W


def _rand_operand(rng, rows, K, lo=118, hi=136):
    q = rng.integers(0, 256, (rows, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x38                      # no NaN codes
    s = rng.integers(lo, hi, (rows, K // 32), dtype=np.uint8)
    return q, s


def test_identity_gives_dequantized_a(orc):
    x = W.activation(seed=101, M=40, N=96)
    qa, sa = orc.mxfp8_quantize(x)
    K = 96
    qb = np.zeros((K, K), np.uint8)
    np.fill_diagonal(qb, 0x38)
    sb = np.full((K, K // 32), 127, np.uint8)
    d = orc.mxfp8_gemm(qa, sa, qb, sb)
    want = orc.mxfp8_dequantize(qa, sa, out="f32").astype(np.float64)
    assert np.array_equal(d, want)


def test_all_ones_closed_form(orc):
    rng = np.random.default_rng(102)
    M, N, K = 5, 7, 160
    qa = np.full((M, K), 0x38, np.uint8)
    qb = np.full((N, K), 0x38, np.uint8)
    sa = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    sb = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    d = orc.mxfp8_gemm(qa, sa, qb, sb)
    for m in range(M):
        for n in range(N):
            want = 32 * sum(2.0 ** (int(sa[m, g]) + int(sb[n, g]) - 254) for g in range(K // 32))
            assert d[m, n] == want


def test_brute_force_tiny(orc):
    rng = np.random.default_rng(103)
    M, N, K = 3, 2, 64
    qa, sa = _rand_operand(rng, M, K)
    qb, sb = _rand_operand(rng, N, K)
    d = orc.mxfp8_gemm(qa, sa, qb, sb)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                a = orc.e4m3_decode(int(qa[m, k])) * orc.e8m0_value(int(sa[m, k // 32]))
                b = orc.e4m3_decode(int(qb[n, k])) * orc.e8m0_value(int(sb[n, k // 32]))
                acc += a * b
            assert abs(d[m, n] - acc) <= 1e-12 * abs(acc) + 1e-300


def test_swap_operands_transposes(orc):
    rng = np.random.default_rng(104)
    qa, sa = _rand_operand(rng, 9, 96)
    qb, sb = _rand_operand(rng, 6, 96)
    assert np.array_equal(orc.mxfp8_gemm(qa, sa, qb, sb), orc.mxfp8_gemm(qb, sb, qa, sa).T)
