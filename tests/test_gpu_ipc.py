"""The fused wgrad + reduce-scatter through CUDA IPC: two processes, each a
data-parallel rank owning half of an FP32 main gradient, map each other's
shard (exchange_shards over a gloo group) and add their wgrad products into
both.  With one GPU available both processes share it; nothing in them
waits on the other's kernels (the reductions are atomic and the ranks meet
only on the host, after synchronizing their own streams)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

N, K, M = 512, 384, 256


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank):
    from blockwise_fp8_pretraining_b200 import synthetic as syn

    g = syn.generator(9100 + rank)
    return syn.normal_bf16((M, N), 1e-3, g), syn.activation_bf16(M, K, 4, 30.0, g)


def _start():
    return np.random.default_rng(17).normal(scale=0.01, size=(N, K)).astype(np.float32)


def _rank(rank, world, port, results):
    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import blockwise_fp8_pretraining_b200 as fp8
    from blockwise_fp8_pretraining_b200 import synthetic as syn

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        rows = N // world
        local = torch.from_numpy(_start()[rank * rows:(rank + 1) * rows].copy()).cuda()
        shards = fp8.exchange_shards(local)
        dy, x = _inputs(rank)
        _, _, dyqT, sdyT = fp8.fp8_quantize_act_1x128(dy.cuda(), fp8.COLWISE)
        _, _, xqT, sxT = fp8.fp8_quantize_act_1x128(x.cuda(), fp8.COLWISE)
        fp8.fp8_block_gemm_wgrad_reduce_scatter_f32(dyqT, sdyT, xqT, sxT, shards)
        torch.cuda.synchronize()
        dist.barrier()                      # every rank's additions are done
        results[rank] = local.cpu().numpy().tolist()
        del shards
        torch.cuda.synchronize()
        dist.barrier()                      # peers' mappings released before the owners free
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_scatter_through_ipc():
    import torch.multiprocessing as mp

    import oracle
    from blockwise_fp8_pretraining_b200 import synthetic as syn

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = {r: np.array(results[r]) for r in range(world)}
    running = _start().astype(np.float64)
    tol = np.zeros((N, K))
    for r in range(world):
        dy, x = _inputs(r)
        dyqT, sdyT = oracle.quantize_act_colwise(syn.bf16_bits(dy))
        xqT, sxT = oracle.quantize_act_colwise(syn.bf16_bits(x))
        running, bound = oracle.gemm_wgrad_accum(dyqT, sdyT, xqT, sxT, running)
        tol += 2e-3 * bound + 1e-6 + 2.0 ** -24 * np.abs(running)
    rows = N // world
    for r in range(world):
        sl = slice(r * rows, (r + 1) * rows)
        err = np.abs(got[r] - running[sl])
        assert np.all(err <= tol[sl]), f"rank {r}: {int((err > tol[sl]).sum())} elements outside the bound"
