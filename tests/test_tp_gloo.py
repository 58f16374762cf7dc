"""Tensor- and expert-parallel layer forms (block_scaled_w8a8_b200.tp) with two
ranks over gloo on CPU.

Each rank builds the same seeded weights, keeps its shard, and runs the
sharded layer; the local steps run in the CPU oracle (injected as the
``local`` backend: the tests exercise the sharding, the partition rule and
the collectives, while the CUDA kernels behind the default backend have their
own GPU parity tests).  Results are compared with the unsharded oracle layer:
  * column parallel: bit-identical (every output column is computed the same);
  * row parallel: the fp32 partials of the two K halves are summed and
    rounded once, so the result lies within the GEMM tolerance of the
    unsharded fp64 result (and within one bf16 ulp of it);
  * expert parallel MoE: every row meets the same codes, expert weights and
    combine as unsharded, so the result is bit-identical."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


class OracleLocal:
    """The per-GPU steps of tp.py, computed by the CPU oracle on torch CPU
    tensors in the library's layouts (scales [Kb, rows])."""

    def __init__(self, oracle):
        self.o = oracle

    def quant_act(self, x, group_k, dtype):
        q, s = self.o.quant_act(_bits(x), group_k, dtype)
        return torch.from_numpy(q), torch.from_numpy(np.ascontiguousarray(s.T))

    def gemm(self, qa, sa, qw, sw, bn, bk, dtype, bias=None):
        out = self.o.gemm(qa.numpy(), sa.numpy().T, qw.numpy(), sw.numpy(), bn, bk, dtype,
                          bias_bf16=None if bias is None else _bits(bias))
        return _bf16(self.o.bf16_from_f64(out))

    def gemm_partial(self, qa, sa, qw, sw, bn, bk, dtype):
        out = self.o.gemm(qa.numpy(), sa.numpy().T, qw.numpy(), sw.numpy(), bn, bk, dtype)
        return torch.from_numpy(out.astype(np.float32))

    def finish_bf16(self, part, bias=None):
        v = part.numpy().astype(np.float64)
        if bias is not None:
            v = v + self.o.bf16_to_f64(_bits(bias))[None, :]
        return _bf16(self.o.bf16_from_f64(v))

    def moe_permute(self, ids, E):
        off, perm, inv = self.o.moe_permute(ids.numpy(), E)
        return (torch.from_numpy(off.astype(np.int32)), torch.from_numpy(perm.astype(np.int32)),
                torch.from_numpy(inv.astype(np.int32)))

    def moe_quant_gather(self, x, perm, topk, group_k, dtype):
        rows = perm.numpy() // topk
        return self.quant_act(x[torch.from_numpy(rows.astype(np.int64))], group_k, dtype)

    def w13_silu_quant(self, qa, sa, offsets, q13, s13, dtype):
        I = q13.shape[1] // 2
        y = self.o.grouped_gemm(qa.numpy(), sa.numpy().T, offsets.numpy(), q13.numpy(),
                                s13.numpy(), 128, 128, dtype, seam=I)
        h = self.o.silu_mul(self.o.bf16_from_f64(y), I)
        return self.quant_act(_bf16(h), 128, dtype)

    def w2(self, qh, sh, offsets, q2, s2, dtype):
        y = self.o.grouped_gemm(qh.numpy(), sh.numpy().T, offsets.numpy(), q2.numpy(),
                                s2.numpy(), 128, 128, dtype)
        return _bf16(self.o.bf16_from_f64(y))

    def moe_combine(self, y, inv_perm, topk_w):
        return _bf16(self.o.moe_combine(_bits(y), inv_perm.numpy(), topk_w.numpy()))


def _worker(rank, world, port, case, q):
    try:
        import sys
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import torch.distributed as dist
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bq_synth
        import oracle
        from block_scaled_w8a8_b200 import tp
        loc = OracleLocal(oracle)
        res = {}
        if case in ("column", "row"):
            M, N, K = 19, 512, _linear_k(world)
            x = bq_synth.activations(M, K, 3, 7, 20.0)
            w = bq_synth.weights(N, K, 0.02, 4).numpy()
            bias = bq_synth.activations(1, N, 5)[0]
            qw, sw = oracle.quant_weight(w, 128, 128, oracle.INT8)
            qw, sw = torch.from_numpy(qw), torch.from_numpy(sw)
            if case == "column":
                n = N // world
                y = tp.column_parallel_linear(
                    x, qw[rank * n:(rank + 1) * n].contiguous(),
                    sw[rank * n // 128:(rank + 1) * n // 128].contiguous(),
                    bias[rank * n:(rank + 1) * n].contiguous(), group=None, local=loc)
            else:
                k = K // world
                y = tp.row_parallel_linear(
                    x[:, rank * k:(rank + 1) * k].contiguous(),
                    qw[:, rank * k:(rank + 1) * k].contiguous(),
                    sw[:, rank * k // 128:(rank + 1) * k // 128].contiguous(), bias,
                    group=None, local=loc)
                ms = _scatter_rows(world)
                y2 = tp.row_parallel_linear(
                    x[:ms, rank * k:(rank + 1) * k].contiguous(),
                    qw[:, rank * k:(rank + 1) * k].contiguous(),
                    sw[:, rank * k // 128:(rank + 1) * k // 128].contiguous(), bias,
                    group=None, scatter_rows=True, local=loc)
                res["scattered"] = _bits(y2)
            res["y"] = _bits(y)
        elif case == "moe":
            T, H, I, E, topk = 24, 256, 256, 4, 2
            x = bq_synth.activations(T, H, 10 + rank)      # each rank's own tokens
            ids, tw = oracle.moe_route(bq_synth.router_logits(T, E, 20 + rank).numpy(), topk)
            w13 = [bq_synth.weights(2 * I, H, 0.02, 30 + e).numpy() for e in range(E)]
            w2 = [bq_synth.weights(H, I, 0.02, 40 + e).numpy() for e in range(E)]
            qs13 = [oracle.quant_weight_gate_up(w, I, 128, 128, oracle.INT8) for w in w13]
            qs2 = [oracle.quant_weight(w, 128, 128, oracle.INT8) for w in w2]
            el = E // world
            mine = range(rank * el, (rank + 1) * el)
            q13 = torch.from_numpy(np.stack([qs13[e][0] for e in mine]))
            s13 = torch.from_numpy(np.stack([qs13[e][1] for e in mine]))
            q2 = torch.from_numpy(np.stack([qs2[e][0] for e in mine]))
            s2 = torch.from_numpy(np.stack([qs2[e][1] for e in mine]))
            y = tp.expert_parallel_moe(x, torch.from_numpy(ids), torch.from_numpy(tw), q13, s13,
                                       q2, s2, E=E, group=None, local=loc)
            # unsharded: all E experts on this rank's tokens
            allq13 = torch.from_numpy(np.stack([a for a, _ in qs13]))
            alls13 = torch.from_numpy(np.stack([b for _, b in qs13]))
            allq2 = torch.from_numpy(np.stack([a for a, _ in qs2]))
            alls2 = torch.from_numpy(np.stack([b for _, b in qs2]))
            off, perm, inv = loc.moe_permute(torch.from_numpy(ids), E)
            qa, sa = loc.moe_quant_gather(x, perm, topk, 128, oracle.INT8)
            qh, sh = loc.w13_silu_quant(qa, sa, off, allq13, alls13, oracle.INT8)
            yr = loc.w2(qh, sh, off, allq2, alls2, oracle.INT8)
            ref = loc.moe_combine(yr, inv, torch.from_numpy(tw))
            res["y"], res["ref"] = _bits(y), _bits(ref)
        dist.destroy_process_group()
        q.put((rank, res, None))
    except Exception as e:                          # report instead of hanging the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))


def _linear_k(world):
    """K of the linear cases: K / world must be a whole number of 128-blocks."""
    return 768 if world == 2 else 1024


def _scatter_rows(world):
    """Token rows of the reduce-scatter case: a multiple of the group size."""
    return 18 if world == 2 else 16


def _run(case, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, res, err = q.get(timeout=240)
        assert err is None, err
        out[rank] = res
    for p in procs:
        p.join(timeout=60)
    return out


def _reference_linear(world=2):
    import bq_synth
    import oracle
    M, N, K = 19, 512, _linear_k(world)
    x = bq_synth.activations(M, K, 3, 7, 20.0)
    w = bq_synth.weights(N, K, 0.02, 4).numpy()
    bias = _bits(bq_synth.activations(1, N, 5)[0])
    qa, sa = oracle.quant_act(_bits(x), 128, oracle.INT8)
    qw, sw = oracle.quant_weight(w, 128, 128, oracle.INT8)
    return oracle.gemm(qa, sa, qw, sw, 128, 128, oracle.INT8, bias_bf16=bias)


def test_column_parallel_matches_unsharded_bit_for_bit():
    import oracle
    out = _run("column")
    ref = oracle.bf16_from_f64(_reference_linear())
    for rank in (0, 1):
        assert np.array_equal(out[rank]["y"], ref)


def test_row_parallel_rounds_once_after_the_fp32_sum():
    import oracle
    out = _run("row")
    ref64 = _reference_linear()
    for rank in (0, 1):
        got = oracle.bf16_to_f64(out[rank]["y"])
        d = got - ref64
        assert np.abs(d).max() <= 1e-2 * np.abs(ref64).max()
        assert np.linalg.norm(d) <= 2e-3 * np.linalg.norm(ref64)
        # one rounding of a sum within fp32 error: at most one bf16 ulp away
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref64), 1e-30))) - 7)
        assert np.all(np.abs(d) <= ulp + 1e-30)
        # the reduce-scatter form leaves rank r the rows [9 r, 9 r + 9)
        assert np.array_equal(out[rank]["scattered"], out[rank]["y"][9 * rank:9 * rank + 9])


def test_expert_parallel_moe_matches_unsharded_bit_for_bit():
    out = _run("moe")
    for rank in (0, 1):
        assert np.array_equal(out[rank]["y"], out[rank]["ref"])


def test_partition_rule_rejects_cut_blocks():
    from block_scaled_w8a8_b200 import tp, BqError
    tp.check_partition(2, 1024, 512, [256, 256])
    with pytest.raises(BqError):
        tp.check_partition(2, 1024, 512, [200, 312])       # output shard not a block_n multiple
    with pytest.raises(BqError):
        tp.check_partition(2, 640, 320, [256])              # input shard not a block_k multiple


def test_four_ranks():
    """The same three forms over four gloo ranks: column and expert parallel
    (one expert per rank, so some ranks receive no rows from others) equal the
    unsharded layer bit for bit; row parallel sums four fp32 partials and
    rounds once (within one bf16 ulp), and its reduce-scatter leaves rank r
    rows [4 r, 4 r + 4)."""
    import oracle
    ref64 = _reference_linear(4)
    out = _run("column", world=4)
    for rank in range(4):
        assert np.array_equal(out[rank]["y"], oracle.bf16_from_f64(ref64))
    out = _run("row", world=4)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref64), 1e-30))) - 7)
    for rank in range(4):
        d = oracle.bf16_to_f64(out[rank]["y"]) - ref64
        assert np.all(np.abs(d) <= ulp + 1e-30)
        assert np.array_equal(out[rank]["scattered"], out[rank]["y"][4 * rank:4 * rank + 4])
    out = _run("moe", world=4)
    for rank in range(4):
        assert np.array_equal(out[rank]["y"], out[rank]["ref"])
