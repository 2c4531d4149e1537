"""Pins of the oracle's block-scaled FP4 GEMM (the consumer of the quantized
operands), checked against things other than itself.

Qiita note on NVFP4 training: Fprop multiplies X by W^T with both operands in
NVFP4, each block's E2M1 codes times its E4M3 block scale.  The oracle's
gemm_block_scaled is dequantize + a float64 matmul; these tests pin the
contraction (which index is summed, which operand is transposed), the scale
layouts and alpha.
"""
from fractions import Fraction

import numpy as np
import pytest

E2M1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6]                 # the E2M1 magnitudes (Glossary)
E4M3 = {0x30: 0.5, 0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x48: 4.0}   # a few E4M3 codes


def e2m1(code):
    v = Fraction(E2M1[code & 7]).limit_denominator()
    return -v if code & 8 else v


def codes(q, rows, cols):
    """[rows, cols] nibbles of packed codes (element 2j in the low nibble)."""
    out = np.zeros((rows, cols), np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


def pack(c):
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def test_exact_product_by_brute_force(orc):
    """Tiny linear-layout case summed with exact fractions from the value
    tables above: every term is dyadic, so the float64 oracle must be exact."""
    M, N, K = 3, 5, 32
    rng = np.random.default_rng(1)
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    keys = np.array(list(E4M3))
    sa = rng.choice(keys, (M, K // 16)).astype(np.uint8)
    sb = rng.choice(keys, (N, K // 16)).astype(np.uint8)
    got = orc.gemm_block_scaled(pack(ca), sa.ravel(), pack(cb), sb.ravel(), M, N, K,
                                scale_layout=orc.SCALE_LINEAR)
    for m in range(M):
        for n in range(N):
            want = sum(e2m1(int(ca[m, k])) * Fraction(E4M3[int(sa[m, k // 16])]) *
                       e2m1(int(cb[n, k])) * Fraction(E4M3[int(sb[n, k // 16])]) for k in range(K))
            assert Fraction(got[m, n]) == want, (m, n)


@pytest.mark.parametrize("layout", [0, 1])
def test_one_hot_b_selects_columns_of_a(orc, layout):
    """B row n holds the code of 1.0 at column k_n and zeros elsewhere, scale
    1.0: then C[:, n] is column k_n of dequantized A (M != N catches a swapped
    operand, distinct k_n a wrong contraction index)."""
    M, N, K = 256, 128, 512
    rng = np.random.default_rng(2)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    sfa = rng.integers(0x20, 0x50, orc.scale_bytes(M, K // 16, layout), dtype=np.uint8)
    kn = rng.permutation(K)[:N]
    cb = np.zeros((N, K), np.uint8)
    cb[np.arange(N), kn] = 0x2
    sfb = np.full(orc.scale_bytes(N, K // 16, layout), 0x38, np.uint8)
    c = orc.gemm_block_scaled(qa, sfa, pack(cb), sfb, M, N, K, scale_layout=layout)
    a = orc.dequantize(orc.FMT_NVFP4, qa, sfa, M, K, 1, 16, s_dec=1.0, scale_layout=layout)
    np.testing.assert_array_equal(c, a[:, kn].astype(np.float64))


def test_layouts_agree_and_alpha_scales(orc):
    """The same block scales stored linearly or in the 128x4 tiles give the
    same product; alpha multiplies it."""
    M, N, K = 128, 256, 256
    rng = np.random.default_rng(3)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qb = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    la = rng.integers(0x20, 0x48, (M, K // 16), dtype=np.uint8)
    lb = rng.integers(0x20, 0x48, (N, K // 16), dtype=np.uint8)

    def swz(lin, rows, cols):
        out = np.zeros(orc.scale_bytes(rows, cols, 1), np.uint8)
        for r in range(rows):
            for c in range(cols):
                out[orc.scale_offset(r, c, rows, cols, 1)] = lin[r, c]
        return out

    c_lin = orc.gemm_block_scaled(qa, la.ravel(), qb, lb.ravel(), M, N, K,
                                  scale_layout=orc.SCALE_LINEAR)
    c_swz = orc.gemm_block_scaled(qa, swz(la, M, K // 16), qb, swz(lb, N, K // 16), M, N, K,
                                  scale_layout=orc.SCALE_SWIZZLED)
    np.testing.assert_array_equal(c_lin, c_swz)
    c_q = orc.gemm_block_scaled(qa, la.ravel(), qb, lb.ravel(), M, N, K, alpha=0.25,
                                scale_layout=orc.SCALE_LINEAR)
    np.testing.assert_array_equal(c_q, c_lin * 0.25)


def test_mxfp4_operands_by_brute_force(orc):
    """MXFP4 operands: 32-value blocks with E8M0 scales 2^(s - 127); the exact
    product from the E2M1 table and powers of two."""
    M, N, K = 2, 3, 64
    rng = np.random.default_rng(4)
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = rng.integers(120, 134, (M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 134, (N, K // 32), dtype=np.uint8)
    got = orc.gemm_block_scaled(pack(ca), sa.ravel(), pack(cb), sb.ravel(), M, N, K,
                                fmt=orc.FMT_MXFP4, scale_layout=orc.SCALE_LINEAR)
    for m in range(M):
        for n in range(N):
            want = sum(e2m1(int(ca[m, k])) * Fraction(2) ** (int(sa[m, k // 32]) - 127) *
                       e2m1(int(cb[n, k])) * Fraction(2) ** (int(sb[n, k // 32]) - 127)
                       for k in range(K))
            assert Fraction(got[m, n]) == want, (m, n)


def test_if4_operand_by_brute_force(orc):
    """An IF4 A operand (scale bit 7 set: INT4 block, k in two's complement,
    value RN(RN(k * RN(6/7)) * S)) against an NVFP4 B operand, 16-value
    blocks: the exact sum of the products of those binary32 values."""
    M, N, K = 2, 3, 64
    rng = np.random.default_rng(5)
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    ca[ca == 8] = 9                                   # -8 is not an INT4 code
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    keys = np.array(list(E4M3))
    sa = rng.choice(keys, (M, K // 16)).astype(np.uint8)
    sa[:, ::2] |= 0x80                                # every other A block is INT4
    sb = rng.choice(keys, (N, K // 16)).astype(np.uint8)
    got = orc.gemm_block_scaled(pack(ca), sa.ravel(), pack(cb), sb.ravel(), M, N, K,
                                fmt=orc.FMT_IF4, scale_layout=orc.SCALE_LINEAR)
    c67 = np.float32(6.0) / np.float32(7.0)

    def a_value(m, k):
        s = int(sa[m, k // 16])
        S = np.float32(E4M3[s & 0x7F])
        c = int(ca[m, k])
        if s & 0x80:
            kk = c - 16 if c & 8 else c
            return Fraction(float(np.float32(np.float32(kk) * c67) * S))
        return e2m1(c) * Fraction(float(S))

    for m in range(M):
        for n in range(N):
            terms = [a_value(m, k) * e2m1(int(cb[n, k])) * Fraction(E4M3[int(sb[n, k // 16])])
                     for k in range(K)]
            # each product is exact in float64; only the K - 1 additions round
            bound = sum(abs(t) for t in terms) * K * Fraction(1, 2 ** 53)
            assert abs(Fraction(got[m, n]) - sum(terms)) <= bound, (m, n)
