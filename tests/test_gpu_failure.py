"""Failure detection on the GPU: a kernel that gives up on a bounded wait
reports HILS_ERR_TIMEOUT, and the context stays usable.

The test lowers the wait limit of the kernels' pipeline waits to 1 ns through
the testing hook, so that the prefill kernels give up while their pipelines are
still filling: the attention kernel's MMA thread, for one, starts out waiting
for its first tile and gives up after a few hundred idle polls.  The kernels'
waits for their own copies and products in flight keep their full limit, so
they exit with nothing left running.  No fault, trap or endless loop is
involved.
"""
import numpy as np
import pytest
import torch

import hils_inputs as hi
from problem import random_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from chunk_sparse_long_b200 import build, hils
    build.build()
    hils.load()


def test_prefill_gives_up_on_a_short_wait_limit_and_recovers():
    import gpu_util as gu
    from chunk_sparse_long_b200 import hils
    from problem import run_oracle
    p = random_problem(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, chunk_size=64, top_k=8,
                       calib_rank=32, seq_len=1500, dtype=hi.DT_BF16, seed=2, spare_pages=3)
    dp = gu.DevProblem(p)
    hils.set_wait_limit_ns(1)
    try:
        with pytest.raises(hils.HilsError) as e:
            gu.run_prefill(dp)
        assert e.value.status == 5, e.value          # HILS_ERR_TIMEOUT
        assert "bounded wait" in str(e.value)
    finally:
        hils.set_wait_limit_ns(0)
    hils.device_status()                            # the error word was cleared
    # the next call runs normally and is correct
    out, idx, w = gu.run_prefill(dp)
    orc = run_oracle(p)
    qr, rb, rh, rp = p.rows()

    def rerun(rows, forced):
        from oracle import oracle
        from problem import ocfg
        return oracle.hils_rows(ocfg(p), qr[rows], rb[rows], rh[rows], rp[rows], p.A, p.B,
                                p.pages, p.block_table, p.landmarks, forced)
    gu.compare(idx.cpu().numpy(), w.cpu().numpy(), gu.to_f64(out).reshape(-1, p.head_dim), orc,
               rerun, p.dtype)
