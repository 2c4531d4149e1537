"""Host-side checks of arithmetic shortcuts the CUDA kernels take (CPU only).

The kernels are compared with the oracle bit for bit on the GPU; these tests
pin the shortcuts themselves over every input they can meet, which no finite
GPU test can enumerate.
"""
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def div_exe(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("div") / "div_check")
    flags = ["-O2", "-ffp-contract=off"]
    # use the hardware FMA when the host has one (fmaf is correctly rounded either way)
    probe = subprocess.run(["gcc", "-mfma", "-x", "c", "-", "-o", "/dev/null"],
                           input="int main(){return 0;}", text=True, capture_output=True)
    if probe.returncode == 0:
        flags.append("-mfma")
    subprocess.check_call(["gcc", *flags, os.path.join(HERE, "div_check.c"), "-o", exe, "-lm"])
    return exe


@pytest.mark.parametrize("d,floor", [("6", -125), ("7.5", -122), ("28", -122)])
def test_division_by_the_grid_maximum_is_the_ieee_quotient(div_exe, d, floor):
    """Markstein's corrected product equals RN(y/d) for every float y >= 2^floor
    (checked over all finite non-negative bit patterns), for the FP4 maximum 6
    and the FP6 maxima 7.5 (E2M3) and 28 (E3M2).  Below 2^-125 the quotient
    by 6 is subnormal and rounds to E4M3 code 0; the FP6 kernels divide with
    IEEE division below 2^-122."""
    out = subprocess.run([div_exe, "0", "0x7F800000", d], capture_output=True, text=True,
                         check=True).stdout.split()
    bad, worst = int(out[0]), float(out[1])
    assert worst < 2.0 ** floor, worst
    assert bad < (1 << 24)                  # only the subnormal-quotient range differs


def test_magic_number_rounding_is_round_half_even():
    """IF4's INT4 step: RN(t + 1.5*2^23) - 1.5*2^23 == rint(t) for |t| < 7.5,
    including every tie j + 1/2."""
    t = np.concatenate([np.linspace(-7.5, 7.5, 200_001, dtype=np.float32)[1:-1],
                        np.arange(-7, 7, dtype=np.float32) + np.float32(0.5)])
    t = t[np.abs(t) < 7.5]
    magic = np.float32(12582912.0)
    s = (t + magic).astype(np.float32)
    assert np.array_equal((s - magic).astype(np.float32), np.rint(t))
    assert np.array_equal(s.view(np.uint32) & 0xF,
                          (np.rint(t).astype(np.int64) & 0xF).astype(np.uint32))


def test_magic_number_low_bits_are_the_int4_nibble():
    """IF4's INT4 nibble: for an integer-valued k in [-8, 7], RN(k + 1.5*2^23)
    is exact and its low four bits are k in two's complement."""
    k = np.arange(-8, 8, dtype=np.float32)
    s = (k + np.float32(12582912.0)).astype(np.float32)
    assert np.array_equal((s - np.float32(12582912.0)).astype(np.float32), k)
    assert np.array_equal(s.view(np.uint32) & 0xF, (k.astype(np.int64) & 0xF).astype(np.uint32))


def test_magic_number_rint_and_int6_group_packing():
    """IF6's INT6 step: RN(t + 1.5*2^23) - 1.5*2^23 == rint(t) for |t| <= 31.25
    (every tie j + 1/2 included), and four such words summed with weights 64^i,
    minus (0x4B400000 - 32) * (1 + 64 + 64^2 + 64^3), XOR 0x820820, is the
    24-bit group of the four 6-bit two's-complement codes."""
    magic = np.float32(12582912.0)
    t = np.concatenate([np.linspace(-31.25, 31.25, 400_001, dtype=np.float32),
                        np.arange(-31, 31, dtype=np.float32) + np.float32(0.5)])
    s_ = (t + magic).astype(np.float32)
    assert np.array_equal((s_ - magic).astype(np.float32), np.rint(t))
    rng = np.random.default_rng(0)
    k = np.concatenate([rng.integers(-31, 32, (20000, 4)),
                        np.array([[-31, -31, -31, -31], [31, 31, 31, 31], [0, -1, 1, -31]])])
    bits = (k.astype(np.float32) + magic).astype(np.float32).view(np.uint32).astype(np.uint64)
    acc = (((bits[:, 3] * 64 + bits[:, 2]) * 64 + bits[:, 1]) * 64 + bits[:, 0]) % 2**32
    bias = ((0x4B400000 - 32) * (1 + 64 + 4096 + 262144)) % 2**32
    got = ((acc - bias) % 2**32) ^ 0x820820
    want = sum((k[:, i] & 0x3F).astype(np.uint64) << (6 * i) for i in range(4))
    assert np.array_equal(got, want)


def test_if3_fp3_by_three_comparisons():
    """IF3's FP3 step: with s1 = [a > 0.5], s2 = [a >= 1.5], s3 = [a > 3] the
    index s1 + s2 + s3 and value s1 + s2 + 2 s3 are the nearest E2M0 magnitude
    (0, 1, 2, 4; ties to the even index; saturating) by exhaustive search."""
    grid = np.array([0.0, 1.0, 2.0, 4.0])
    a = np.concatenate([np.linspace(0, 8, 400_001, dtype=np.float32),
                        np.float32([0.5, 1.5, 3.0, np.nextafter(np.float32(0.5), 1),
                                    np.nextafter(np.float32(1.5), 0),
                                    np.nextafter(np.float32(3.0), 4), 1e30])])
    d = np.abs(a.astype(np.float64)[:, None] - grid[None, :])
    # among the nearest magnitudes (two only at a tie) take the even index
    best = np.argmin(np.where(d == d.min(1, keepdims=True), np.arange(4) % 2, 9), axis=1)
    best[a >= 4] = 3                                # saturation (float64 distances tie at 1e30)
    s1, s2, s3 = (a > 0.5), (a >= 1.5), (a > 3.0)
    idx = s1.astype(int) + s2 + s3
    assert np.array_equal(idx, best)
    assert np.array_equal(s1 + s2.astype(float) + 2 * s3, grid[best])


def test_if3_group_packing_and_pair_store():
    """IF3's packing: eight words RN(n + 1.5*2^23) (n the FP3 index, or k in
    -3..3) summed with weights 8^j, minus 0x4B400000 (or 0x4B400000 - 4) times
    0x249249, give the 24-bit group (FP3: plus the sign bits shifted into bit
    2; INT3: XOR 0x924924 for two's complement); a pair of blocks' groups go
    out as three little-endian words holding 12 consecutive code bytes, and
    three 16-bit loads give a block's two groups back."""
    magic = np.float32(12582912.0)
    w = np.array([8 ** j for j in range(8)], dtype=np.uint64)
    kocts = 0x249249
    rng = np.random.default_rng(1)
    n = rng.integers(0, 4, (5000, 8))
    sg = rng.integers(0, 2, (5000, 8))
    bits = (n.astype(np.float32) + magic).astype(np.float32).view(np.uint32).astype(np.uint64)
    acc = ((bits + 4 * sg.astype(np.uint64)) * w).sum(axis=1) % 2**32
    got_fp = (acc - (0x4B400000 * kocts) % 2**32) % 2**32
    assert np.array_equal(got_fp, ((n + 4 * sg).astype(np.uint64) * w).sum(axis=1))
    t = np.concatenate([np.linspace(-3.25, 3.25, 100_001, dtype=np.float32),
                        np.float32([-2.5, -1.5, -0.5, 0.5, 1.5, 2.5])])
    assert np.array_equal(((t + magic).astype(np.float32) - magic).astype(np.float32), np.rint(t))
    k = np.concatenate([rng.integers(-3, 4, (5000, 8)), np.full((1, 8), -3), np.full((1, 8), 3)])
    bits = (k.astype(np.float32) + magic).astype(np.float32).view(np.uint32).astype(np.uint64)
    acc = (bits * w).sum(axis=1) % 2**32
    got_int = ((acc - ((0x4B400000 - 4) * kocts) % 2**32) % 2**32) ^ 0x924924
    assert np.array_equal(got_int, ((k & 7).astype(np.uint64) * w).sum(axis=1))
    # the pair store and the dequantizer's reassembly
    for ga0, ga1, gb0, gb1 in rng.integers(0, 1 << 24, (200, 4)).tolist():
        w0 = (ga0 | ga1 << 24) & 0xFFFFFFFF
        w1 = (ga1 >> 8 | gb0 << 16) & 0xFFFFFFFF
        w2 = (gb0 >> 16 | gb1 << 8) & 0xFFFFFFFF
        out = b"".join(v.to_bytes(4, "little") for v in (w0, w1, w2))
        want = b"".join(g.to_bytes(3, "little") for g in (ga0, ga1, gb0, gb1))
        assert out == want
        for blk in (out[:6], out[6:]):
            h0, h1, h2 = (int.from_bytes(blk[2 * i:2 * i + 2], "little") for i in range(3))
            g0, g1 = (h0 | h1 << 16) & 0xFFFFFF, (h1 >> 8) | (h2 << 8)
            assert blk == g0.to_bytes(3, "little") + g1.to_bytes(3, "little")


def test_if4_split_tables_sum_to_k():
    """The IF4 GEMM's split: for every INT4 nibble n (k in two's complement)
    the two E2M1 codes of the tables the split kernel uses add up to k."""
    part1, part2 = 0xACDEEFFF77665420, 0x0000A0AC20200000
    e2m1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6]

    def value(code):
        return -e2m1[code & 7] if code & 8 else e2m1[code & 7]

    for n in range(16):
        k = n - 16 if n & 8 else n
        c1, c2 = (part1 >> (4 * n)) & 0xF, (part2 >> (4 * n)) & 0xF
        assert value(c1) + value(c2) == k, (n, c1, c2)


def test_rint_ties_go_to_even():
    """rint (the kernels' cvt.rni) on the INT4 ties t = j + 0.5."""
    t = np.arange(-7, 7, dtype=np.float32) + np.float32(0.5)
    assert np.all(np.rint(t) % 2 == 0)


@pytest.mark.parametrize("method", [0, 1, 2, 3])
def test_stochastic_rounding_fixed_point_method(tmp_path, method):
    """The kernels' stochastic rounding methods (0: integer codes, 1: rounded
    values then the round-to-nearest conversion, 2: the same after scaling
    by 2^-126, which needs no range test, 3: method 2 with the product
    saturated at 1 and the low bits dropped by a truncating conversion
    instead of a mask) equal the oracle's rule
    (round the magnitude up iff u < t * 2^16) on every u for values around
    each E2M1 grid point and midpoint, and on 4M random pairs."""
    exe = str(tmp_path / "sr_check")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-frounding-math",
                           os.path.join(HERE, "sr_check.c"),
                           os.path.join(os.path.dirname(HERE), "oracle", "fp4q_oracle.c"),
                           "-o", exe, "-lm"])
    out = subprocess.run([exe, "4000000", str(method)], capture_output=True, text=True,
                         check=True)
    assert int(out.stdout.strip()) == 0


def _rht_source():
    return open(os.path.join(HERE, "..", "fp4_block_scaled_04_b200", "csrc", "rht.cu")).read()


def test_rht_philox_table_layout():
    """The per-warp Philox table of the SR transform: the four words of the
    call for token t and column octet o at byte (2 t + o) * 16 + (t / 16) * 16.
    Entries do not overlap and fit the table. The eight 16-byte writes of a
    quarter warp (tokens 16 g + i, g = 0..7, fixed i and o) hit eight distinct
    bank groups. The table fits in one BF16 input stage of the tile."""
    src = _rht_source()
    assert "constexpr int kPTabBytes = (2 * 127 + 1) * 16 + (127 / 16) * 16 + 16;" in src
    assert "ptab_off(int t, int o) { return (2 * t + o) * 16 + (t >> 4) * 16; }" in src
    assert "constexpr int kUnits = 128 * 4 + 16;" in src
    size = (2 * 127 + 1) * 16 + (127 // 16) * 16 + 16
    off = lambda t, o: (2 * t + o) * 16 + (t >> 4) * 16
    spans = sorted((off(t, o), off(t, o) + 16) for t in range(128) for o in range(2))
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= size <= (128 * 4 + 16) * 8     # one stage: kUnits units of 8 bytes
    for i in range(16):
        for o in range(2):
            assert len({(off(16 * g + i, o) // 16) % 8 for g in range(8)}) == 8, (i, o)
