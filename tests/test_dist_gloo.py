"""Multi-rank host logic, run as two ``gloo`` ranks on the CPU.

Checks what the several-GPU path adds around the kernels: the aligned row
shards, the 4-byte all-reduce MAX that gives every rank the whole tensor's
amax (the tensor-level scale of the Qiita NVFP4 note, "scaleの導出", comes
from the amax of the whole tensor), and the max-over-ranks step time.  The
per-rank quantizer here is the oracle, so the test needs no GPU: quantizing
each shard with the global amax must give exactly the slices of quantizing
the whole tensor.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp4_block_scaled_04_b200 import dist as fdist
from fp4_block_scaled_04_b200 import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _worker(rank, world_size, port, outdir):
    import oracle as orc

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world_size,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        rows, cols = 384, 128
        x = workloads.activation(rows=rows, cols=cols, seed=3)
        # one huge outlier in rank 1's rows: rank 0 alone would pick a smaller amax
        x[300, 5] = 4000.0
        xb = _bits(x)
        r0, r1 = fdist.shard_rows(rows, world_size, rank, align=128)
        shard = xb[r0:r1]

        local = torch.tensor([orc.amax(shard)], dtype=torch.float32)
        g = fdist.global_amax(local)
        whole_amax = orc.amax(xb)
        assert float(g.item()) == whole_amax

        mine = orc.quantize_nvfp4(shard, layouts=orc.ROWWISE | orc.COLWISE,
                                  amax=float(g.item()), scale_layout=orc.SCALE_SWIZZLED)
        full = orc.quantize_nvfp4(xb, layouts=orc.ROWWISE | orc.COLWISE,
                                  amax=whole_amax, scale_layout=orc.SCALE_SWIZZLED)
        assert mine["s_dec"] == full["s_dec"]
        np.testing.assert_array_equal(mine["q_row"], full["q_row"][r0:r1])
        # swizzled row scales: whole 128-row tiles are contiguous 512-byte runs
        per_tile = (cols // 16 // 4) * 512
        np.testing.assert_array_equal(
            mine["sf_row"].reshape(-1),
            full["sf_row"].reshape(-1)[(r0 // 128) * per_tile:(r1 // 128) * per_tile])
        # column-wise codes are the transpose: this shard owns byte columns r0/2..r1/2
        np.testing.assert_array_equal(mine["q_col"], full["q_col"][:, r0 // 2:r1 // 2])

        # step time: every rank reports the slowest rank's
        t = fdist.max_over_ranks(1.5 + rank)
        assert t == 1.5 + (world_size - 1)
        gbs = fdist.aggregate_gbs(1_000_000, world_size, 10, t)
        assert gbs == pytest.approx(world_size * 1e7 / (t * 1e-3) / 1e9)
        open(os.path.join(outdir, f"ok{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_quantize_matches_whole_tensor(orc):
    world_size = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(world_size, _free_port(), d), nprocs=world_size, join=True)
        assert sorted(os.listdir(d)) == ["ok0", "ok1"]


def test_shard_rows_partition():
    for rows, align in [(0, 16), (16, 16), (384, 128), (8192, 16), (14336, 128)]:
        for ws in (1, 2, 3, 4, 8):
            spans = [fdist.shard_rows(rows, ws, r, align) for r in range(ws)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            for a0, a1 in spans:
                assert a0 % align == 0 and a1 % align == 0 and a1 >= a0
            sizes = [a1 - a0 for a0, a1 in spans]
            assert max(sizes) - min(sizes) <= align


def test_shard_rows_rejects_bad_arguments():
    with pytest.raises(ValueError):
        fdist.shard_rows(100, 2, 0, align=16)
    with pytest.raises(ValueError):
        fdist.shard_rows(128, 2, 2, align=16)


def test_single_process_is_identity():
    a = torch.tensor([3.25], dtype=torch.float32)
    assert fdist.global_amax(a) is a and float(a.item()) == 3.25
    assert fdist.max_over_ranks(7.0) == 7.0
    with pytest.raises(ValueError):
        fdist.global_amax(torch.zeros(2))
