"""Row-parallel (tp) GEMM host logic on CPU: K-shard slicing of packed operands and of both
swizzled scale layouts against the oracle's own swizzle of the sliced scales, and a
world-size-2 gloo run of the row-parallel call (the local GEMM replaced by the oracle's)
against the oracle's row-parallel reading, plus the bench's max-over-ranks reduction."""
import importlib.util
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as orc
from nvfp4_block_scaled_10_b200 import SF_128x4, SF_8x4, tp, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_k_shard_bounds():
    assert tp.k_shard_bounds(8192, 0, 2) == (0, 4096)
    assert tp.k_shard_bounds(8192, 1, 2) == (4096, 8192)
    with pytest.raises(ValueError):
        tp.k_shard_bounds(192, 0, 2)  # 96-element shards are not whole 64-element steps


@pytest.mark.parametrize("layout,olayout", [(SF_128x4, orc.L128x4), (SF_8x4, orc.L8x4)])
@pytest.mark.parametrize("R,K", [(5, 256), (130, 512), (17, 1024)])
def test_shard_scales_match_oracle_swizzle(layout, olayout, R, K):
    lin = workloads.random_bytes((R, K // 16), R + K)
    full = torch.from_numpy(orc.swizzle(lin, olayout))
    for t in (2, 4):
        if K % (64 * t):
            continue
        for r in range(t):
            k0, k1 = tp.k_shard_bounds(K, r, t)
            want = orc.swizzle(np.ascontiguousarray(lin[:, k0 // 16:k1 // 16]), olayout)
            got = tp.shard_scales(full, R, K, layout, r, t).numpy()
            assert np.array_equal(got, want)


def test_shard_packed():
    q = torch.from_numpy(workloads.random_bytes((3, 512), 1))
    a, b = tp.shard_packed(q, 0, 2), tp.shard_packed(q, 1, 2)
    assert torch.equal(torch.cat([a, b], dim=1), q) and a.is_contiguous()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _operands(M=6, N=40, K=256):
    a = workloads.random_bytes((M, K // 2), 31)
    w = workloads.random_bytes((N, K // 2), 32)
    sa = workloads.random_bytes((M, K // 16), 33, 0x28, 0x48)
    sw = workloads.random_bytes((N, K // 16), 34, 0x28, 0x48)
    return a, sa, 3.0, w, sw, 40.0


def _rank_main(rank, world, port, outdir):
    import torch.distributed as dist

    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, sa, ga, w, sw, gw = _operands()
        K = 2 * a.shape[1]
        k0, k1 = tp.k_shard_bounds(K, rank, world)
        a_s, w_s = a[:, k0 // 2:k1 // 2], w[:, k0 // 2:k1 // 2]
        sa_s, sw_s = sa[:, k0 // 16:k1 // 16], sw[:, k0 // 16:k1 // 16]

        def cpu_gemm(*_args, out=None, **_kw):  # this rank's shard GEMM, by the oracle
            o = torch.from_numpy(orc.gemm(a_s, sa_s, ga, w_s, sw_s, gw).view(np.float16).copy())
            if out is not None:
                out.copy_(o)
                return out
            return o

        got = tp.row_parallel_gemm(None, None, None, None, None, None, local_gemm=cpu_gemm)
        ms = bench.max_over_ranks(10.0 + rank, dist, "cpu")
        np.save(os.path.join(outdir, f"rank{rank}.npy"), got.view(torch.int16).numpy())
        np.save(os.path.join(outdir, f"ms{rank}.npy"), np.array([ms]))
    finally:
        dist.destroy_process_group()


def test_row_parallel_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    want = orc.gemm_row_parallel(*_operands(), tp=world)
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npy").view(np.uint16)
        assert np.array_equal(got, want)  # every rank holds the same summed output
        assert np.load(tmp_path / f"ms{r}.npy")[0] == 11.0  # the slowest rank's time


def test_job_throughput():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_throughput(2, 1.5, 10.0) == pytest.approx(300.0)  # 2 x 1.5 units / 10 ms
