"""The multi-rank (N > 1) host path on CPU with gloo, world size 2: token sharding,
the Wgrad all-reduce, the NVFP4 global amax option, max-over-ranks timing, and a
rank that fails before a collective. The per-rank compute stands in with the CPU
oracle (the CUDA kernels are covered by the -m gpu tests)."""
import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp4_block_scaled_deterministic_b200 import dp, synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port, timeout_s=30):
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=timeout_s))


def _wgrad_worker(rank, world, port, fmt, out_q):
    try:
        import sys
        sys.path.insert(0, ROOT)
        import oracle
        _init(rank, world, port)
        M, N, K = 128, 64, 96
        X = synthetic.normal(M, K, 1.0, seed=3, outlier_frac=0.02, outlier_mult=50.0)
        dY = synthetic.heavy_tailed_grad(M, N, seed=4)
        a, b = dp.token_shard(M, rank, world)
        Xs, dYs = X[a:b].contiguous(), dY[a:b].contiguous()
        if fmt == oracle.NVFP4:
            # global tensor amax: each rank's amax of its rotated shard, max over ranks
            amax = torch.tensor([oracle.rotate(dYs, 16, oracle.COL).__abs__().max(),
                                 oracle.rotate(Xs, 16, oracle.COL).__abs__().max()],
                                dtype=torch.float32)
            dp.allreduce_amax_(amax)
            out_q.put((rank, "amax", amax.numpy().tolist()))
        qa = oracle.quantize(dYs, fmt, 16, oracle.COL)
        qb = oracle.quantize(Xs, fmt, 16, oracle.COL)
        part = oracle.gemm_f64(oracle.dequantize(*qa[:3], fmt), oracle.dequantize(*qb[:3], fmt))
        t = torch.from_numpy(part)
        work = dp.allreduce_wgrad(t, async_op=True)
        work.wait()
        slowest = dp.max_over_ranks(float(rank + 1), "cpu")
        out_q.put((rank, "dW", t.numpy(), slowest))
        dist.barrier()
        dist.destroy_process_group()
    except Exception:
        out_q.put((rank, "error", traceback.format_exc()))


def _run(fn, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    # drain the queue while the ranks run: a child that has put items exits only after
    # they are read, so joining first would wait out the whole timeout
    import queue
    import time
    results = []
    deadline = time.monotonic() + 120
    while time.monotonic() < deadline and any(p.is_alive() for p in procs):
        try:
            results.append(q.get(timeout=0.2))
        except queue.Empty:
            pass
    for p in procs:
        p.join(timeout=max(0.0, deadline - time.monotonic()))
    while True:
        try:
            results.append(q.get(timeout=0.2))
        except queue.Empty:
            break
    for p in procs:
        if p.is_alive():
            p.kill()
    return results


@pytest.mark.parametrize("fmt", [0])
def test_dp_wgrad_equals_single_rank_wgrad(orc, fmt):
    res = _run(_wgrad_worker, 2, fmt)
    errs = [r for r in res if r[1] == "error"]
    assert not errs, errs[0][2]
    dws = [r for r in res if r[1] == "dW"]
    assert len(dws) == 2
    M, N, K = 128, 64, 96
    X = synthetic.normal(M, K, 1.0, seed=3, outlier_frac=0.02, outlier_mult=50.0)
    dY = synthetic.heavy_tailed_grad(M, N, seed=4)
    qa = orc.quantize(dY, fmt, 16, orc.COL)
    qb = orc.quantize(X, fmt, 16, orc.COL)
    full = orc.gemm_f64(orc.dequantize(*qa[:3], fmt), orc.dequantize(*qb[:3], fmt))
    for r in dws:
        assert np.allclose(r[2], full, rtol=1e-12, atol=1e-12)
        assert r[3] == 2.0  # max over ranks of (rank + 1)
    assert np.array_equal(dws[0][2], dws[1][2])


def test_nvfp4_global_amax_matches_single_rank(orc):
    res = _run(_wgrad_worker, 2, 1)
    errs = [r for r in res if r[1] == "error"]
    assert not errs, errs[0][2]
    amaxes = [r[2] for r in res if r[1] == "amax"]
    assert len(amaxes) == 2 and amaxes[0] == amaxes[1]
    M, N, K = 128, 64, 96
    X = synthetic.normal(M, K, 1.0, seed=3, outlier_frac=0.02, outlier_mult=50.0)
    dY = synthetic.heavy_tailed_grad(M, N, seed=4)
    full_dy = orc.quantize(dY, 1, 16, orc.COL)[3]
    full_x = orc.quantize(X, 1, 16, orc.COL)[3]
    assert np.float32(amaxes[0][0]) == np.float32(full_dy)
    assert np.float32(amaxes[0][1]) == np.float32(full_x)


def _failing_worker(rank, world, port, out_q):
    try:
        _init(rank, world, port, timeout_s=5)
        if rank == 1:
            raise RuntimeError("rank 1 fails before its collective")
        t = torch.ones(4)
        try:
            dist.all_reduce(t)
            out_q.put((rank, "no-error"))
        except Exception as e:  # the peer never joins: the collective must end in an error
            out_q.put((rank, "collective-error", type(e).__name__))
    except RuntimeError as e:
        out_q.put((rank, "raised", str(e)))


def test_rank_failure_surfaces_as_collective_error():
    res = _run(_failing_worker, 2)
    kinds = {r[0]: r[1] for r in res}
    assert kinds.get(1) == "raised"
    assert kinds.get(0) == "collective-error"


def test_token_shard():
    assert dp.token_shard(8192, 0, 2) == (0, 4096)
    assert dp.token_shard(8192, 7, 8) == (7168, 8192)
    with pytest.raises(ValueError):
        dp.token_shard(8192 + 32, 0, 2)
    with pytest.raises(ValueError):
        dp.token_shard(64, 2, 2)
