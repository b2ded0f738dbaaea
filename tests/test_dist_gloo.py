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


def _partial_dw(oracle, X, dY, rank, world, fmt):
    """This rank's fp32 partial dW: the oracle's Wgrad of its token shard (the GPU GEMM
    writes fp32 dW)."""
    a, b = dp.token_shard(X.shape[0], rank, world)
    Xs, dYs = X[a:b].contiguous(), dY[a:b].contiguous()
    qa = oracle.quantize(dYs, fmt, 16, oracle.COL)
    qb = oracle.quantize(Xs, fmt, 16, oracle.COL)
    part = oracle.gemm_f64(oracle.dequantize(*qa[:3], fmt), oracle.dequantize(*qb[:3], fmt))
    return part.astype(np.float32), (Xs, dYs)


def _inputs(M=128, N=64, K=96):
    X = synthetic.normal(M, K, 1.0, seed=3, outlier_frac=0.02, outlier_mult=50.0)
    dY = synthetic.heavy_tailed_grad(M, N, seed=4)
    return X, dY


def _wgrad_worker(rank, world, port, fmt, out_q):
    try:
        import sys
        sys.path.insert(0, ROOT)
        import oracle
        _init(rank, world, port)
        X, dY = _inputs()
        part, (Xs, dYs) = _partial_dw(oracle, X, dY, rank, world, fmt)
        if fmt == oracle.NVFP4:
            # global tensor amax: each rank's amax of its rotated shard, max over ranks
            amax = torch.tensor([oracle.rotate(dYs, 16, oracle.COL).__abs__().max(),
                                 oracle.rotate(Xs, 16, oracle.COL).__abs__().max()],
                                dtype=torch.float32)
            dp.allreduce_amax_(amax)
            out_q.put((rank, "amax", amax.numpy().tolist()))
        t = torch.from_numpy(part.copy())
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


@pytest.mark.parametrize("world", [2, 4])
def test_dp_wgrad_is_the_rank_ordered_sum(orc, world):
    """The reduced dW equals, bit for bit, the sum of the ranks' fp32 partials added in
    rank order, on every rank and on two runs; it is within fp32 rounding of the
    single-rank Wgrad over all tokens."""
    fmt = 0
    runs = []
    for _ in range(2):
        res = _run(_wgrad_worker, world, fmt)
        errs = [r for r in res if r[1] == "error"]
        assert not errs, errs[0][2]
        dws = sorted((r for r in res if r[1] == "dW"), key=lambda r: r[0])
        assert len(dws) == world
        assert all(r[3] == float(world) for r in dws)  # max over ranks of (rank + 1)
        runs.append([r[2] for r in dws])
    X, dY = _inputs()
    acc = _partial_dw(orc, X, dY, 0, world, fmt)[0].copy()
    for r in range(1, world):
        acc += _partial_dw(orc, X, dY, r, world, fmt)[0]  # one fp32 rounding per addition
    for run in runs:
        for d in run:
            assert d.dtype == np.float32 and np.array_equal(d.view(np.uint32), acc.view(np.uint32))
    qa = orc.quantize(dY, fmt, 16, orc.COL)
    qb = orc.quantize(X, fmt, 16, orc.COL)
    full = orc.gemm_f64(orc.dequantize(*qa[:3], fmt), orc.dequantize(*qb[:3], fmt))
    assert np.linalg.norm(acc - full) <= 1e-6 * np.linalg.norm(full)


def test_rank_ordered_sum_is_sequential():
    parts = torch.tensor([[1.0], [2.0 ** -24], [2.0 ** -24]], dtype=torch.float32)
    # ((1 + 2^-24) + 2^-24) = 1 in fp32 (each tie rounds to even); 1 + (2^-24 + 2^-24) would not
    assert dp.rank_ordered_sum_(parts).item() == 1.0
    assert dp.rank_ordered_sum_(parts.flip(0)).item() == 1.0 + 2.0 ** -23


def test_nvfp4_global_amax_matches_single_rank(orc):
    res = _run(_wgrad_worker, 2, 1)
    errs = [r for r in res if r[1] == "error"]
    assert not errs, errs[0][2]
    amaxes = [r[2] for r in res if r[1] == "amax"]
    assert len(amaxes) == 2 and amaxes[0] == amaxes[1]
    X, dY = _inputs()
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
