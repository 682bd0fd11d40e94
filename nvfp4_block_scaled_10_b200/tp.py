"""Row-parallel (K-split) NVFP4 GEMM whose fp16 outputs are summed over the ranks: the tensor
parallelism of "Fused Nvfp4 GEMM All Reduce Plugin" (TensorRT-Edge-LLM C++ API, tp_size 2).

Each rank holds one K shard of the activation and of the weight (both quantized with the
full tensors' global scales, so a shard's block scales are the full scales' K columns). It
runs the block-scaled GEMM on its shard, which gives a rank-local fp16 [M, N], and the ranks
add those outputs with one NCCL all_reduce (for two ranks, the correctly rounded fp16 sum).

This is the unfused form: the GEMM kernel, then the collective on the same stream. A kernel
that stores its epilogue tiles into the peer's memory and reduces there needs two GPUs to
run and is not built.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import SF_128x4, SF_8x4, nvfp4_gemm


def k_shard_bounds(K: int, rank: int, tp: int) -> tuple[int, int]:
    """[k0, k1) of rank's K shard; every shard holds whole 64-element MMA steps."""
    if K % (64 * tp) != 0:
        raise ValueError(f"K = {K} does not split into {tp} shards of whole 64-element steps")
    ks = K // tp
    return rank * ks, (rank + 1) * ks


def shard_packed(q: torch.Tensor, rank: int, tp: int) -> torch.Tensor:
    """Rank's K shard of a packed E2M1 operand [rows, K/2] (contiguous copy)."""
    k0, k1 = k_shard_bounds(2 * q.shape[1], rank, tp)
    return q[:, k0 // 2:k1 // 2].contiguous()


def shard_scales(sf: torch.Tensor, rows: int, K: int, layout: int, rank: int,
                 tp: int) -> torch.Tensor:
    """Rank's K shard of a swizzled scale buffer. Both layouts store atoms of 4 scale columns
    (64 elements of K) in row-block-major order, so a K shard is the same atom columns of
    every row block: [row blocks, K/64, atom bytes] sliced on the middle axis."""
    k0, k1 = k_shard_bounds(K, rank, tp)
    rb, atom = (128, 512) if layout == SF_128x4 else (8, 32) if layout == SF_8x4 else (0, 0)
    if rb == 0:
        raise ValueError("shard_scales takes the 128x4 or the 8x4 layout")
    blocks = (rows + rb - 1) // rb
    return sf.view(blocks, K // 64, atom)[:, k0 // 64:k1 // 64, :].contiguous().view(-1)


def row_parallel_gemm(a_q, a_sf, a_g, w_q, w_sf, w_g, group=None, a_layout: int = SF_128x4,
                      out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      local_gemm=None) -> torch.Tensor:
    """This rank's shard GEMM (fp16 [M, N]), then the sum over the group's ranks in place.

    a_q, w_q: this rank's packed K shards; a_sf, w_sf: their swizzled scales; a_g, w_g: the
    full tensors' encode scales (device fp32 [1]). `local_gemm` replaces the shard GEMM (same
    signature as nvfp4_gemm); tests of the host logic pass one that runs on CPU.
    """
    gemm = nvfp4_gemm if local_gemm is None else local_gemm
    out = gemm(a_q, a_sf, a_g, w_q, w_sf, w_g, a_layout=a_layout, out=out, workspace=workspace)
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out
