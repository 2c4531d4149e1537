"""GPU parity: the CUDA library (called through its C ABI) against the oracle.

Every output -- packed codes, scale bytes (including IF4 flags), tensor
scales, dequantized values and the exposed RHT intermediate -- must match the
oracle bit for bit on the same seeded inputs.  Small shapes span several
tiles and ragged tails; the full-size cases use the benchmark workloads and
the same calls bench.py times.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def bits(x: torch.Tensor) -> np.ndarray:
    """CPU numpy view for the oracle: BF16 -> uint16 bit patterns, FP32 as is."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16).copy()
    return x.numpy().copy()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_same(name, got, want):
    got = np.asarray(got).reshape(-1)
    want = np.asarray(want).reshape(-1)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), want.view(np.uint32)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (f"{name}: {bad.size} of {got.size} differ; first at {bad[:8]}: "
                           f"gpu {got[bad[:8]]} oracle {want[bad[:8]]}")


def randmat(rows, cols, dtype, seed, scale_spread=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    if scale_spread and rows * cols > 0:
        # per-row magnitudes over many binades, a few outliers, exact zeros,
        # negative zeros and tiny values
        x *= torch.exp2(torch.randint(-20, 12, (rows, 1), generator=g).float())
        flat = x.view(-1)
        n = flat.numel()
        idx = torch.randint(0, n, (max(1, n // 97),), generator=g)
        flat[idx] *= 300.0
        flat[torch.randint(0, n, (max(1, n // 53),), generator=g)] = 0.0
        flat[torch.randint(0, n, (max(1, n // 61),), generator=g)] = -0.0
        flat[torch.randint(0, n, (max(1, n // 71),), generator=g)] *= 1e-30
    return x.to(dtype)


SHAPES_16 = [(16, 16), (48, 80), (80, 144), (208, 336)]
DTYPES = [torch.bfloat16, torch.float32]


# ------------------------------------------------------------------ amax

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (130, 272), (1000, 64)])
def test_amax(orc, dtype, shape):
    x = randmat(*shape, dtype, seed=1)
    got = fq.fp4q_amax(x.to(DEV))
    assert_same("amax", host(got), np.array([orc.amax(bits(x))], np.float32))


def test_amax_strided_input(orc):
    base = randmat(64, 96, torch.bfloat16, seed=2).to(DEV)
    x = base[:, 16:80]                       # ld = 96, cols = 64
    got = fq.fp4q_amax(x)
    assert_same("amax", host(got), np.array([orc.amax(bits(x))], np.float32))


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("where", ["first", "last", "middle"])
def test_amax_position_and_stride(orc, dtype, where):
    """The maximum in the first, last or a middle chunk, for a contiguous
    tensor spanning several grid-stride steps and for a strided view."""
    base = randmat(2304, 640, dtype, seed=3, scale_spread=False)
    pos = {"first": (0, 0), "last": (2303, 639), "middle": (1151, 333)}[where]
    base[pos] = -1000.0
    for x in (base, base[:, 64:576]):
        got = fq.fp4q_amax(x.to(DEV) if x is base else base.to(DEV)[:, 64:576])
        assert_same("amax", host(got), np.array([orc.amax(bits(x))], np.float32))


# ------------------------------------------------------------------ NVFP4

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", SHAPES_16)
@pytest.mark.parametrize("layouts", [1, 2, 3])
@pytest.mark.parametrize("rnd", [0, 1])
def test_nvfp4(orc, dtype, shape, layouts, rnd):
    x = randmat(*shape, dtype, seed=hash((shape, layouts)) & 0xFFFF)
    seed = 0x1234_5678_9ABC
    got = fq.fp4q_quantize_nvfp4(x.to(DEV), layouts=layouts, round=rnd, seed=seed)
    want = orc.quantize_nvfp4(bits(x), layouts=layouts, round=rnd, seed=seed)
    assert_same("s_dec", host(got["s_dec"]), want["s_dec"])
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        if k in want:
            assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("layouts", [1, 2, 3])
def test_nvfp4_swizzled_and_given_amax(orc, layouts):
    x = randmat(256, 128, torch.bfloat16, seed=5)
    amax = fq.fp4q_amax(x.to(DEV))
    got = fq.fp4q_quantize_nvfp4(x.to(DEV), layouts=layouts, amax=amax,
                                 scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_nvfp4(bits(x), layouts=layouts, amax=float(host(amax)[0]),
                              scale_layout=orc.SCALE_SWIZZLED)
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        if k in want:
            assert_same(k, host(got[k]), want[k])


def test_nvfp4_strided_input(orc):
    base = randmat(64, 160, torch.float32, seed=6).to(DEV)
    x = base[:, 32:128]
    got = fq.fp4q_quantize_nvfp4(x, layouts=3)
    want = orc.quantize_nvfp4(bits(x), layouts=3)
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("kind", ["zeros", "one_value", "negative_max", "tiny", "huge"])
def test_nvfp4_degenerate(orc, kind):
    x = torch.zeros(32, 64)
    if kind == "one_value":
        x[7, 9] = 3.0
    elif kind == "negative_max":
        x = randmat(32, 64, torch.float32, seed=7, scale_spread=False)
        x[3, 3] = -1000.0
    elif kind == "tiny":
        x = randmat(32, 64, torch.float32, seed=8, scale_spread=False) * 1e-38
    elif kind == "huge":
        x = randmat(32, 64, torch.float32, seed=9, scale_spread=False) * 1e37
    for dtype in DTYPES:
        xd = x.to(dtype)
        got = fq.fp4q_quantize_nvfp4(xd.to(DEV), layouts=3)
        want = orc.quantize_nvfp4(bits(xd), layouts=3)
        assert_same("s_dec", host(got["s_dec"]), want["s_dec"])
        for k in ("q_row", "sf_row", "q_col", "sf_col"):
            assert_same(f"{kind}/{k}", host(got[k]), want[k])


def wide_range(rows, cols, dtype, seed):
    """Values of about 100 and one of 4e10 at [0, 0].  The tensor scale
    s_enc = 2688 / amax is then so small that a block whose largest magnitude
    is a few hundred gets the scale code 0, whose factor is 0: its values
    encode as zeros, negative ones as -0 (code 8), under both roundings."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * 100.0
    x[0, 0] = 4e10
    return x.to(dtype)


@pytest.mark.parametrize("layouts", [1, 3])
@pytest.mark.parametrize("rnd", [0, 1])
def test_nvfp4_zero_scale_blocks(orc, layouts, rnd):
    for dtype in DTYPES:
        x = wide_range(64, 96, dtype, seed=41)
        got = fq.fp4q_quantize_nvfp4(x.to(DEV), layouts=layouts, round=rnd, seed=77)
        want = orc.quantize_nvfp4(bits(x), layouts=layouts, round=rnd, seed=77)
        assert (want["sf_row"] == 0).sum() > 0
        for k in ("s_dec", "q_row", "sf_row") + (("q_col", "sf_col") if layouts & 2 else ()):
            assert_same(f"{dtype}/{k}", host(got[k]), want[k])


@pytest.mark.parametrize("n", [16, 128])
@pytest.mark.parametrize("rnd", [0, 1])
def test_rht_zero_scale_blocks(orc, n, rnd):
    """The same through the transform: the huge value stays in column 0,
    whose blocks set the amax, and the other columns' blocks get scale 0."""
    dy = wide_range(256, 48, torch.bfloat16, seed=42)
    got = fq.fp4q_quantize_rht_sr(dy.to(DEV), n, round=rnd, seed=5)
    want = orc.quantize_rht(bits(dy), n, round=rnd, seed=5)
    assert (want["sf_t"] == 0).sum() > 0
    for k in ("s_dec", "q_t", "sf_t"):
        assert_same(k, host(got[k]), want[k])


def test_empty_inputs():
    x = torch.empty(0, 32, dtype=torch.bfloat16, device=DEV)
    out = fq.fp4q_quantize_nvfp4(x, layouts=3)
    assert float(out["s_dec"].cpu()[0]) == 1.0
    y = fq.fp4q_dequantize(fq.FMT_NVFP4, out["q_row"], out["sf_row"], 0, 32,
                           tensor_scale=out["s_dec"])
    assert y.shape == (0, 32)
    assert float(fq.fp4q_amax(x).cpu()[0]) == 0.0


def test_bad_arguments_return_status():
    import ctypes
    x = torch.zeros(32, 24, dtype=torch.bfloat16, device=DEV)   # cols % 16 != 0
    with pytest.raises(fq.Fp4qError) as e:
        fq.fp4q_quantize_nvfp4(x)
    assert e.value.status == 2
    out = torch.zeros(1, device=DEV)
    host_x = torch.zeros(16, 16)                                 # host memory is rejected
    st = fq.lib().fp4q_amax(ctypes.c_void_p(host_x.data_ptr()), 1, 16, 16, 16,
                            ctypes.c_void_p(out.data_ptr()), None)
    assert st == 1
    x = torch.zeros(32, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fq.Fp4qError) as e:                      # swizzle needs 128-row multiples
        fq.fp4q_quantize_nvfp4(x, scale_layout=fq.SCALE_SWIZZLED)
    assert e.value.status == 2
    torch.cuda.synchronize()


# ------------------------------------------------------------------ MXFP4

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(32, 32), (96, 160), (160, 96)])
@pytest.mark.parametrize("layouts", [1, 2, 3])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_mxfp4(orc, dtype, shape, layouts, mode):
    x = randmat(*shape, dtype, seed=11 + mode)
    got = fq.fp4q_quantize_mxfp4(x.to(DEV), layouts=layouts, e8m0_mode=mode)
    want = orc.quantize_mxfp4(bits(x), layouts=layouts, e8m0_mode=mode)
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        if k in want:
            assert_same(k, host(got[k]), want[k])


def test_mxfp4_swizzled(orc):
    x = randmat(256, 512, torch.bfloat16, seed=12)
    got = fq.fp4q_quantize_mxfp4(x.to(DEV), layouts=3, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_mxfp4(bits(x), layouts=3, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("q_row", "sf_row", "q_col", "sf_col"):
        assert_same(k, host(got[k]), want[k])


# ------------------------------------------------------------------ 2D

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (80, 144), (208, 336)])
def test_2d(orc, dtype, shape):
    w = randmat(*shape, dtype, seed=13)
    got = fq.fp4q_quantize_2d(w.to(DEV), with_1x16=True)
    want = orc.quantize_2d(bits(w), with_1x16=True)
    for k in ("s_dec", "q_w", "q_wt", "sf_tiles", "sf_w_1x16", "sf_wt_1x16"):
        assert_same(k, host(got[k]), want[k])


def test_2d_swizzled(orc):
    w = randmat(256, 512, torch.float32, seed=14)
    got = fq.fp4q_quantize_2d(w.to(DEV), with_1x16=True, scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_2d(bits(w), with_1x16=True, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("q_w", "q_wt", "sf_tiles", "sf_w_1x16", "sf_wt_1x16"):
        assert_same(k, host(got[k]), want[k])


# ------------------------------------------------------------------ RHT + SR

@pytest.mark.parametrize("n", [16, 128])
@pytest.mark.parametrize("rnd", [1, 0])
@pytest.mark.parametrize("shape", [(128, 8), (256, 72), (384, 200)])
def test_rht(orc, n, rnd, shape):
    dy = workloads.gradient(seed=21, tokens=shape[0], cols=shape[1])
    seed = 0xDEADBEEF01
    got = fq.fp4q_quantize_rht_sr(dy.to(DEV), n, round=rnd, seed=seed, want_rht=True)
    want = orc.quantize_rht(bits(dy), n, round=rnd, seed=seed, want_rht=True)
    assert_same("rht", host(got["rht"]), want["rht"])
    for k in ("s_dec", "q_t", "sf_t"):
        assert_same(k, host(got[k]), want[k])


def test_rht16_ragged_tokens(orc):
    dy = workloads.gradient(seed=22, tokens=144, cols=24)       # 144 = 128 + 16
    got = fq.fp4q_quantize_rht_sr(dy.to(DEV), 16, round=1, seed=3)
    want = orc.quantize_rht(bits(dy), 16, round=1, seed=3)
    for k in ("s_dec", "q_t", "sf_t"):
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("n", [16, 128])
def test_rht_amax_and_fp32_input(orc, n):
    dy = randmat(256, 128, torch.float32, seed=23, scale_spread=False)
    a = fq.fp4q_rht_amax(dy.to(DEV), n, seed=9)
    t = orc.rht(bits(dy), n, 9)
    assert_same("amax_rht", host(a), np.array([np.abs(t).max()], np.float32))
    got = fq.fp4q_quantize_rht_sr(dy.to(DEV), n, round=1, seed=9, amax_rht=a,
                                  scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_rht(bits(dy), n, round=1, seed=9, scale_layout=orc.SCALE_SWIZZLED)
    for k in ("s_dec", "q_t", "sf_t"):
        assert_same(k, host(got[k]), want[k])


# ------------------------------------------------------------------ IF4

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(1, 16), (48, 80), (257, 336)])
def test_if4(orc, dtype, shape):
    x = workloads.if4_blocks(seed=31, rows=shape[0], cols=shape[1]).to(dtype)
    got = fq.fp4q_quantize_if4(x.to(DEV))
    want = orc.quantize_if4(bits(x))
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("shape,layout", [((256, 32288), 0), ((2048, 2048), 1), ((2048, 2048), 0)])
def test_if4_lanes_walk_several_pairs(orc, shape, layout):
    """Shapes with more pairs of blocks than the grid has lanes. With 32288
    columns (1009 pairs per row, a prime that divides no full grid's stride)
    a lane's pair column changes from one pair to the next. With 2048
    columns the stride is a multiple of the pairs per row, so every lane
    stays on one pair column; the columns are also a multiple of 32, so the
    kernel's even form runs (no lone trailing block, both scale bytes of a
    pair in one store), in both scale layouts."""
    x = workloads.if4_blocks(seed=34, rows=shape[0], cols=shape[1])
    got = fq.fp4q_quantize_if4(x.to(DEV), scale_layout=layout)
    want = orc.quantize_if4(bits(x), scale_layout=layout)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])


def test_if4_spread_and_swizzled(orc):
    x = randmat(256, 256, torch.bfloat16, seed=32)
    got = fq.fp4q_quantize_if4(x.to(DEV), scale_layout=fq.SCALE_SWIZZLED)
    want = orc.quantize_if4(bits(x), scale_layout=orc.SCALE_SWIZZLED)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])


@pytest.mark.parametrize("layout", [0, 1])
def test_if4_scales_at_an_odd_address(orc, layout):
    """The scale matrix may start anywhere (the ABI asks 16-byte alignment of
    the codes only): the kernel's paired scale stores fall back to single
    bytes when it starts on an odd address."""
    x = randmat(256, 256, torch.bfloat16, seed=33)
    n = fq.fp4q_scale_bytes(256, 256, 16, layout)
    buf = torch.full((n + 2,), 0xAB, dtype=torch.uint8, device=DEV)
    out = {"s_dec": torch.empty(1, dtype=torch.float32, device=DEV),
           "q": torch.empty((256, 128), dtype=torch.uint8, device=DEV), "sf": buf[1:n + 1]}
    got = fq.fp4q_quantize_if4(x.to(DEV), scale_layout=layout, out=out)
    want = orc.quantize_if4(bits(x), scale_layout=layout)
    for k in ("s_dec", "q", "sf"):
        assert_same(k, host(got[k]), want[k])
    assert int(buf[0].item()) == 0xAB and int(buf[n + 1].item()) == 0xAB


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("cols", [256, 2048])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_dequant_all_formats(orc, out_dtype, cols):
    """Every format, both scale layouts, both output types.  With 2048
    columns (a multiple of 1024) the kernel's row-aligned form runs: a warp's
    step lies in one row, one scale offset and one bound test per step."""
    od = orc.FP32 if out_dtype == torch.float32 else orc.BF16
    R, C = 256, cols
    x = randmat(R, C, torch.bfloat16, seed=41).to(DEV)
    for layout in (fq.SCALE_LINEAR, fq.SCALE_SWIZZLED):
        nv = fq.fp4q_quantize_nvfp4(x, layouts=3, scale_layout=layout)
        y = fq.fp4q_dequantize(fq.FMT_NVFP4, nv["q_row"], nv["sf_row"], R, C,
                               tensor_scale=nv["s_dec"], scale_layout=layout, out_dtype=out_dtype)
        want = orc.dequantize(orc.FMT_NVFP4, host(nv["q_row"]), host(nv["sf_row"]), R, C,
                              s_dec=float(host(nv["s_dec"])[0]), scale_layout=layout, out_dtype=od)
        assert_same("nvfp4 deq", host(y), want)
        mx = fq.fp4q_quantize_mxfp4(x, layouts=1, scale_layout=layout)
        y = fq.fp4q_dequantize(fq.FMT_MXFP4, mx["q_row"], mx["sf_row"], R, C, 1, 32,
                               scale_layout=layout, out_dtype=out_dtype)
        want = orc.dequantize(orc.FMT_MXFP4, host(mx["q_row"]), host(mx["sf_row"]), R, C, 1,
                              32, scale_layout=layout, out_dtype=od)
        assert_same("mxfp4 deq", host(y), want)
        i4 = fq.fp4q_quantize_if4(x, scale_layout=layout)
        y = fq.fp4q_dequantize(fq.FMT_IF4, i4["q"], i4["sf"], R, C, tensor_scale=i4["s_dec"],
                               scale_layout=layout, out_dtype=out_dtype)
        want = orc.dequantize(orc.FMT_IF4, host(i4["q"]), host(i4["sf"]), R, C,
                              s_dec=float(host(i4["s_dec"])[0]), scale_layout=layout, out_dtype=od)
        assert_same("if4 deq", host(y), want)
    WC = 64 if cols == 256 else 1024
    w = randmat(128, WC, torch.float32, seed=42).to(DEV)
    q2 = fq.fp4q_quantize_2d(w)
    y = fq.fp4q_dequantize(fq.FMT_NVFP4, q2["q_w"], q2["sf_tiles"], 128, WC, 16, 16,
                           tensor_scale=q2["s_dec"], out_dtype=out_dtype)
    want = orc.dequantize(orc.FMT_NVFP4, host(q2["q_w"]), host(q2["sf_tiles"]), 128, WC, 16, 16,
                          s_dec=float(host(q2["s_dec"])[0]), out_dtype=od)
    assert_same("2d deq", host(y), want)


def test_dequant_arbitrary_bytes(orc):
    """Every code and every scale byte, including IF4 INT4 blocks."""
    g = torch.Generator().manual_seed(43)
    q = torch.randint(0, 256, (64, 128), generator=g, dtype=torch.int32).to(torch.uint8)
    sf = torch.randint(0, 256, (64 * 16,), generator=g, dtype=torch.int32).to(torch.uint8)
    sf[(sf & 0x7F) == 0x7F] = 0x7E          # 0x7F / 0xFF are E4M3 NaN
    s = torch.tensor([0.37], dtype=torch.float32)
    for fmt in (fq.FMT_NVFP4, fq.FMT_IF4):
        y = fq.fp4q_dequantize(fmt, q.to(DEV), sf.to(DEV), 64, 256, tensor_scale=s.to(DEV))
        want = orc.dequantize(fmt, q.numpy(), sf.numpy(), 64, 256, s_dec=0.37)
        assert_same(f"fmt {fmt}", host(y), want)
    sfm = torch.randint(0, 255, (64 * 8,), generator=g, dtype=torch.int32).to(torch.uint8)
    y = fq.fp4q_dequantize(fq.FMT_MXFP4, q.to(DEV), sfm.to(DEV), 64, 256, 1, 32)
    want = orc.dequantize(orc.FMT_MXFP4, q.numpy(), sfm.numpy(), 64, 256, 1, 32)
    assert_same("mx any", host(y), want)


# ------------------------------------------------------------------ format edges

def test_e2m1_and_e4m3_edges_through_the_abi(orc):
    """Blocks whose maximum is exactly 6 with amax = 2688 have s_enc = 1 and
    S = 1, so the element step sees x itself: every E2M1 tie, its float32
    neighbours, zeros of both signs and values beyond 6 reach the encoder."""
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    vals = []
    for p in ties:
        b = np.array([p], np.float32).view(np.int32)[0]
        vals += list(np.arange(b - 8, b + 9, dtype=np.int32).view(np.float32))
    vals += [0.0, -0.0, 1e-40, -1e-40, 5.999]
    vals = np.array(vals, np.float32)
    vals = np.concatenate([vals, -vals])
    vals = vals[np.abs(vals) <= 6.0]
    rows = []
    for i in range(0, len(vals), 15):
        chunk = np.zeros(15, np.float32)
        chunk[: len(vals[i:i + 15])] = vals[i:i + 15]
        rows.append(np.concatenate([[6.0], chunk]))
    # block maxima just above 6 keep S = 1, so v > 6 and the encoder saturates
    rows.append(np.array([6.2, 6.1, -6.2, 6.05] + [0.0] * 12, np.float32))
    rows.append(np.array([2688.0] + [0.0] * 15, np.float32))       # amax: s_enc = 1
    x = np.stack(rows).astype(np.float32)
    got = fq.fp4q_quantize_nvfp4(torch.from_numpy(x).to(DEV), layouts=1)
    want = orc.quantize_nvfp4(x, layouts=1)
    assert_same("q_row", host(got["q_row"]), want["q_row"])
    assert_same("sf_row", host(got["sf_row"]), want["sf_row"])
    # block scales over a sweep of block maxima: E4M3 rounding of RN(m/6)
    m = np.exp2(np.linspace(-14, 8.9, 4096)).astype(np.float32) * 6
    y = np.zeros((m.size + 1, 16), np.float32)
    y[:-1, 0] = m
    y[-1, 0] = 2688.0
    got = fq.fp4q_quantize_nvfp4(torch.from_numpy(y).to(DEV), layouts=1)
    want = orc.quantize_nvfp4(y, layouts=1)
    assert_same("scale sweep", host(got["sf_row"]), want["sf_row"])
    assert_same("scale sweep q", host(got["q_row"]), want["q_row"])
