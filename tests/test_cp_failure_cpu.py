"""Failure of a rank during the context-parallel decode step, on the CPU with
two gloo ranks and a short process-group timeout (5 s).  Rank 1 fails on the
host before the step's first collective, either by leaving (its process
ends) or by never arriving (it stalls).  Rank 0's step must then end with an
error from its collective within a bounded time, not wait for good.  The
step's kernels are the numpy stand-ins of test_cp_cpu.py; no GPU is used."""
import datetime
import os
import socket
import time

import pytest

PG_TIMEOUT_S = 5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, port, mode, res):
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for x in (root, os.path.join(root, "tests")):
        sys.path.insert(0, x)
    from chunk_sparse_long_b200 import cp, hils
    import test_cp_cpu as t
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=PG_TIMEOUT_S))
    if rank == 1:
        if mode == "stall":
            time.sleep(PG_TIMEOUT_S + 10)    # never reaches the exchange in time
        os._exit(0)                          # leaves without the step
    p = t._problem()
    cfg = hils.HilsConfig(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, t.CHUNK, p.top_k,
                          p.calib_rank, p.dtype)
    shard = hils.Cache(None, 0, None, t.SPLIT, None,
                       torch.full((p.batch,), p.seq_len, dtype=torch.int32))
    q = torch.from_numpy(p.q[:, p.seq_len - 1].copy())
    out = torch.zeros((p.batch, p.n_q_heads, p.head_dim), dtype=torch.float32)
    dec = cp.Decoder(cfg, shard, 0, kernels=t.FakeKernels(p, 0, t.SPLIT), device="cpu")
    t0 = time.monotonic()
    try:
        dec.step(q, None, None, None, None, out)
        res.put(("completed", time.monotonic() - t0))
    except Exception as e:   # the collective's error
        res.put((type(e).__name__, time.monotonic() - t0))
    res.close()
    res.join_thread()        # the result is in the pipe before the process ends
    os._exit(0)


@pytest.mark.parametrize("mode", ["leave", "stall"])
def test_step_ends_with_an_error_when_a_rank_fails(mode):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        kind, elapsed = q.get(timeout=120)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert kind != "completed", "the step finished without its peer"
    assert elapsed < PG_TIMEOUT_S + 30, elapsed
