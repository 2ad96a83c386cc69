"""The multi-GPU bench path on CPU: two gloo ranks, token-sharded replicas.

Each rank times its own batch; the job's device time is the slowest rank's,
and throughput counts the tokens of every rank (weak scaling, no collective on
the data path, only the max-reduce of the timings)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms_local = [12.0, 15.5][rank]
    ms, value = bench.combine_ranks(ms_local, tokens_per_rank=1000, steps=4, world=world, device="cpu")
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 15.5
        assert value == pytest.approx(1000 * 2 * 4 / 15.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    ms, value = bench.combine_ranks(10.0, 500, 3, 1)
    assert ms == 10.0 and value == pytest.approx(500 * 3 / 10e-3)


def test_launch_count_per_step():
    import bench
    import combine_router_gemm_softmax_b200 as M
    assert bench.launches(M.config(64, 128, 8, 2, 128)) == 6
    # CTA-pair GEMM tiles (AUTO's choice here) are one launch per GEMM too
    cfg = M.config(4096, 1024, 8, 2, 3584)
    assert M.moe_gemm_tiles_used(cfg) == M.MOE_GEMM_TILES_PAIR and bench.launches(cfg) == 6
    # combine fused into the down projection (opt-in): no combine kernel
    assert bench.launches(M.config(64, 128, 8, 2, 128, combine="fused")) == 5
    # MXFP8: the row copy is replaced by the dispatch that quantises the rows
    assert bench.launches(M.config(64, 128, 8, 2, 128, precision="mxfp8")) == 6
    assert bench.launches(M.config(64, 128, 8, 2, 128, expert_kind="identity")) == 4
    assert bench.launches(M.config(64, 128, 8, 2, 128, expert_kind="scale")) == 5
    assert bench.launches(M.config(64, 32, 4, 2, 64, dtype="f32")) == 7
    assert bench.launches(M.config(65536, 128, 256, 2, 128)) == 7      # 256 * 512 chunks: separate scan
    assert bench.launches(M.config(8192, 2048, 128, 8, 768)) == 6      # 128 * 64 chunks: scan inside rank
    assert bench.launches(M.config(64, 128, 8, 4, 128, capacity=20, layout="padded")) == 7  # + padding fill
    assert bench.launches(M.config(64, 128, 8, 4, 128, capacity=0, layout="padded")) == 6
