"""The multi-process path of bench.py, on the CPU with the gloo backend
(world size 2): the barrier, the max-over-ranks step time and the whole-job
weak-scaling throughput, and the per-rank input seeds (each rank runs its own
independent sequence; the path has no data exchange)."""
import datetime
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import hils_inputs as hi
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        barrier, maxreduce = bench.dist_ops("gloo", "cpu")
        barrier()
        step_ms = 10.0 + rank          # the ranks' own step times
        worst = maxreduce(step_ms)
        value = bench.weak_scaling_value(131072, world, worst)
        # the seed offset of each rank gives it its own sequence
        w = hi.WORKLOADS["prefill_128k_gqa"]
        q0 = hi.normal(w.seed + rank, hi.TID_Q, 0, 8, 1.0, hi.DT_F32)
        out.put((rank, worst, value, q0.tolist()))
        barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_step_time_and_scale_weakly():
    import torch.multiprocessing as mp
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
    (r0, worst0, v0, q00), (r1, worst1, v1, q01) = res
    assert worst0 == worst1 == 11.0            # the slowest rank sets the step time
    assert v0 == v1 == pytest.approx(131072 * 2 / 11.0e-3)
    assert q00 != q01                          # independent inputs per rank


def test_weak_scaling_value_is_units_over_slowest_step():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.weak_scaling_value(1000, 1, 1.0) == pytest.approx(1e6)
    assert bench.weak_scaling_value(1000, 8, 2.0) == pytest.approx(4e6)


def test_reference_arm_runs_on_rank_0_only():
    """Under torchrun the reference arm (the oracle on host cores) runs on rank
    0 alone; the other ranks leave at once, with status 0 and no output, and
    touch neither CUDA nor a process group (this runs on a CPU-only host)."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
