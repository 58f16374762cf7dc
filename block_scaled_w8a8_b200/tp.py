"""Tensor- and expert-parallel forms of the block-scaled linear layer.

The block-wise INT8 page (section 3) fixes how a block-quantised weight may
be split over GPUs: every shard of the output dimension must be a multiple of
block_n, and, when the input dimension is split, every shard of it a multiple
of block_k, so that no weight block (and no 1 x block_k activation group) is
cut.  ``check_partition`` applies that rule (bq_check_tp_partition); the three
layer forms below then need no other care:

* column parallel (the output dimension N split): each GPU quantises the
  whole input and computes its N / world columns; the codes, scales and
  outputs are exactly those of the unsharded layer (optionally all-gathered);
* row parallel (the input dimension K split): each GPU quantises its K slice
  (its 1 x block_k groups are whole groups of the unsharded input, so the
  codes and scales are the unsharded ones), computes the unrounded fp32
  partial over its K-blocks (bq_gemm_partial), the partials are summed
  across GPUs in fp32 (all-reduce, or reduce-scatter over the token rows),
  and one kernel adds the bias and rounds once to bf16 (bq_finish_bf16): the
  layer is rounded exactly once, as unsharded;
* expert parallel MoE (the experts split): each GPU quantises its own tokens
  once, groups its (token, slot) rows by global expert (bq_moe_permute,
  bq_moe_quant_gather), sends each GPU the codes and scales of the rows routed
  to its experts (all-to-all: one byte per element instead of two), runs its
  experts on every received chunk (the fused w13 + SiLU requantisation and
  the w2 grouped GEMM), sends the outputs back, and combines each token's
  top-k rows with their routing weights (bq_moe_combine: fp32 sum, one bf16
  rounding).

Collectives go through torch.distributed (NCCL on GPUs, gloo on CPU).  Every
arithmetic step runs in a ``Local`` backend: the CUDA library by default
(``CudaLocal``); the CPU tests pass the oracle instead.  Tensor layouts are
the library's: activations bf16 [M, K], codes uint8, activation scales fp32
[Kb, M] (K-block-major), weight codes [N, K] with scales [ceil(N/bn), Kb].
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (INT8, check_tp_partition, finish_bf16, gemm, gemm_partial, grouped_gemm,
               grouped_gemm_silu_quant, moe_combine, moe_permute, moe_quant_gather, quant_act)


class CudaLocal:
    """The per-GPU steps, run by libbq's CUDA kernels."""

    def quant_act(self, x, group_k, dtype):
        return quant_act(x, group_k, dtype)

    def gemm(self, qa, sa, qw, sw, bn, bk, dtype, bias=None):
        return gemm(qa, sa, qw, sw, bn, bk, dtype, bias=bias)

    def gemm_partial(self, qa, sa, qw, sw, bn, bk, dtype):
        return gemm_partial(qa, sa, qw, sw, bn, bk, dtype)

    def finish_bf16(self, part, bias=None):
        return finish_bf16(part, bias)

    def moe_permute(self, ids, E):
        return moe_permute(ids, E)

    def moe_quant_gather(self, x, perm, topk, group_k, dtype):
        return moe_quant_gather(x, perm, topk, group_k, dtype)

    def w13_silu_quant(self, qa, sa, offsets, q13, s13, dtype):
        return grouped_gemm_silu_quant(qa, sa, offsets, q13, s13, dtype)

    def w2(self, qh, sh, offsets, q2, s2, dtype):
        return grouped_gemm(qh, sh, offsets, q2, s2, 128, 128, 0, dtype)

    def moe_combine(self, y, inv_perm, topk_w):
        return moe_combine(y, inv_perm, topk_w)


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def check_partition(world: int, input_size: int, input_size_per_partition: int,
                    output_partition_sizes, block_n: int = 128, block_k: int = 128):
    """The block-wise INT8 page's tensor-parallel rule (section 3)."""
    check_tp_partition(world, input_size, input_size_per_partition,
                       list(output_partition_sizes), block_n, block_k)


def column_parallel_linear(x, qw_shard, sw_shard, bias_shard=None, *, block_n=128, block_k=128,
                           dtype=INT8, group=None, gather=True, local=None):
    """y = x W^T with W's rows (the output columns) split evenly over the
    group: this rank holds rows [r N/w, (r + 1) N/w) of the codes, their
    scale rows and bias slice.  Returns this rank's bf16 [M, N/w] columns,
    or the whole [M, N] output when gather is set (all-gather)."""
    local = local or CudaLocal()
    world, _ = _world(group)
    n_local = qw_shard.shape[0]
    check_partition(world, x.shape[1], x.shape[1], [n_local] * world, block_n, block_k)
    qa, sa = local.quant_act(x, block_k, dtype)
    y = local.gemm(qa, sa, qw_shard, sw_shard, block_n, block_k, dtype, bias=bias_shard)
    if not gather or world == 1:
        return y
    parts = [torch.empty_like(y) for _ in range(world)]
    dist.all_gather(parts, y.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def row_parallel_linear(x_shard, qw_shard, sw_shard, bias=None, *, block_n=128, block_k=128,
                        dtype=INT8, group=None, scatter_rows=False, local=None):
    """y = x W^T with the input dimension K split evenly over the group: this
    rank holds x[:, Kr] and W[:, Kr] (Kr = [r K/w, (r + 1) K/w)) with the
    matching scale columns, and the whole bias.  The fp32 partials are summed
    over the group (all-reduce, or reduce-scatter over token rows when
    scatter_rows is set, leaving this rank rows [r M/w, (r + 1) M/w)), then
    the bias is added and the sum rounded once to bf16."""
    local = local or CudaLocal()
    world, _ = _world(group)
    M, k_local = x_shard.shape
    N = qw_shard.shape[0]
    check_partition(world, k_local * world, k_local, [N], block_n, block_k)
    qa, sa = local.quant_act(x_shard, block_k, dtype)
    part = local.gemm_partial(qa, sa, qw_shard, sw_shard, block_n, block_k, dtype)
    if world > 1:
        if scatter_rows:
            if M % world != 0:
                raise ValueError(f"scatter_rows needs M ({M}) divisible by the group size")
            out = torch.empty(M // world, N, dtype=part.dtype, device=part.device)
            dist.reduce_scatter_tensor(out, part.contiguous(), op=dist.ReduceOp.SUM, group=group)
            part = out
        else:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return local.finish_bf16(part, bias)


def _all_to_all_rows(send, counts_out, counts_in, group):
    """Rows of `send` (first dimension) go to rank d in chunks of
    counts_out[d]; returns the rows received, in rank order."""
    recv = send.new_empty((int(sum(counts_in)),) + tuple(send.shape[1:]))
    dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=list(counts_in),
                           input_split_sizes=list(counts_out), group=group)
    return recv


def expert_parallel_moe(x, topk_ids, topk_w, q13, s13, q2, s2, *, E, dtype=INT8, group=None,
                        local=None):
    """The MoE layer with its E experts split evenly over the group: this rank
    holds experts [r E/w, (r + 1) E/w) -- gate/up codes q13 [E/w, 2I, H] with
    scales s13 [E/w, 2 ceil(I/128), H/128], down codes q2 [E/w, H, I] with
    scales s2 -- and its own tokens x bf16 [T, H] routed by topk_ids int32
    [T, k] (global expert ids) with weights topk_w fp32 [T, k].  Returns this
    rank's bf16 [T, H] outputs."""
    local = local or CudaLocal()
    world, _ = _world(group)
    if E % world != 0:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    e_local = E // world
    T, H = x.shape
    topk = topk_ids.shape[1]
    # 1. group this rank's (token, slot) rows by global expert and quantise
    #    them once: rows for rank d's experts are one contiguous chunk
    offsets, perm, inv = local.moe_permute(topk_ids, E)
    qa, sa = local.moe_quant_gather(x, perm, topk, 128, dtype)
    off = offsets.to("cpu", torch.int64)
    bounds = [int(off[d * e_local]) for d in range(world)] + [int(off[E])]
    counts_out = [bounds[d + 1] - bounds[d] for d in range(world)]
    # per-destination expert offsets (relative to the chunk start)
    rel = torch.stack([off[d * e_local:(d + 1) * e_local + 1] - bounds[d] for d in range(world)])
    # 2. exchange row counts and expert offsets (on the collective's device),
    #    then codes and scales
    counts_t = torch.tensor(counts_out, dtype=torch.int64, device=x.device)
    counts_in_t = torch.empty_like(counts_t)
    dist.all_to_all_single(counts_in_t, counts_t, group=group)
    counts_in = [int(c) for c in counts_in_t.cpu()]
    rel = rel.to(x.device)
    rel_in = torch.empty_like(rel)
    dist.all_to_all_single(rel_in, rel.contiguous(), group=group)
    q_in = _all_to_all_rows(qa, counts_out, counts_in, group)
    s_in = _all_to_all_rows(sa.t().contiguous(), counts_out, counts_in, group)   # [rows, Kb]
    # 3. this rank's experts on every received chunk (rows grouped by expert)
    ys, start = [], 0
    for src in range(world):
        n = counts_in[src]
        if n == 0:
            ys.append(q_in.new_empty((0, H), dtype=torch.bfloat16))
            continue
        qa_c = q_in[start:start + n].contiguous()
        sa_c = s_in[start:start + n].t().contiguous()
        offs = rel_in[src].to(device=qa_c.device, dtype=torch.int32)
        qh, sh = local.w13_silu_quant(qa_c, sa_c, offs, q13, s13, dtype)
        ys.append(local.w2(qh, sh, offs, q2, s2, dtype))
        start += n
    y_local = torch.cat(ys, dim=0)
    # 4. outputs back to the ranks that own the tokens, in their row order
    y_back = _all_to_all_rows(y_local, counts_in, counts_out, group)
    # 5. weighted top-k combine: fp32 sum, one bf16 rounding
    return local.moe_combine(y_back, inv, topk_w)
