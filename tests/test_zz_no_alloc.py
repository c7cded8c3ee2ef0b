"""hils_decode_noalloc gives the same results as hils_decode.

hils_decode_noalloc serves callers that cannot allocate device memory (a host
engine's plugin that is given only inputs and outputs, or a service that must
not allocate while serving): its scratch is an array built into the library.
Here both entry points run the same two decode steps in a row, each on its
own copy of the cache, and their outputs must agree within the decode
tolerance (bf16 outputs max-abs <= 2e-2; in practice identical).  This file
is collected last on purpose.
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


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    import gpu_util as gu
    from chunk_sparse_long_b200 import hils
    p = random_problem(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, chunk_size=64, top_k=8,
                       calib_rank=16, seq_len=1400, dtype=hi.DT_BF16, seed=31, spare_pages=2)
    ref = gu.DevProblem(p)     # runs hils_decode with a caller workspace
    na = gu.DevProblem(p)      # runs hils_decode_noalloc
    t0 = 1300
    for dp in (ref, na):
        dp.seq_lens.fill_(t0)
    nbytes = hils.workspace_size(ref.cfg, hils.OP_DECODE, 1, p.max_chunks)
    assert 0 < nbytes <= hils.decode_noalloc_capacity()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    Kd, Vd = gu.dev(p.K), gu.dev(p.V)
    B, Hq, d, k = p.batch, p.n_q_heads, p.head_dim, p.top_k
    for t in (t0, t0 + 1):
        q = ref.q[:, t].contiguous()
        kn, vn = Kd[:, t].contiguous(), Vd[:, t].contiguous()
        res = []
        for dp, fn in ((ref, "ws"), (na, "noalloc")):
            out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
            idx = torch.empty((B, Hq, k), dtype=torch.int32, device="cuda")
            w = torch.empty((B, Hq, k), dtype=torch.float32, device="cuda")
            if fn == "ws":
                hils.decode(dp.cfg, q, kn, vn, dp.A, dp.B, dp.cache, out, idx, w, ws, nbytes)
            else:
                hils.decode_noalloc(dp.cfg, q, kn, vn, dp.A, dp.B, dp.cache, out, idx, w)
            hils.device_status()
            res.append((idx.cpu().numpy(), w.cpu().numpy(), gu.to_f64(out)))
        (i0, w0, o0), (i1, w1, o1) = res
        np.testing.assert_array_equal(i1, i0)
        np.testing.assert_allclose(w1, w0, rtol=0, atol=1e-5)
        assert np.abs(o1 - o0).max() <= 2e-2
    assert ref.seq_lens.cpu().tolist() == na.seq_lens.cpu().tolist() == [t0 + 2] * B


def test_noalloc_rejects_configurations_beyond_its_scratch():
    from chunk_sparse_long_b200 import hils
    cfg = hils.HilsConfig(64, 64, 64, 128, 64, 32, 16, hils.HILS_BF16)
    big = 1 << 20
    assert hils.workspace_size(cfg, hils.OP_DECODE, 1, big) > hils.decode_noalloc_capacity()
    fake = 1 << 20
    cache = hils.Cache(fake, 1, fake, big, fake, fake)
    with pytest.raises(hils.HilsError) as e:
        hils.decode_noalloc(cfg, fake, None, None, fake, fake, cache, fake, None, None)
    assert e.value.status == 3 and "built-in" in str(e.value)


def test_noalloc_clears_counters_left_by_a_larger_configuration():
    """Every call starts from what the previous call left in the built-in
    scratch.  A large configuration fills the start of the array with its
    candidate lists; a small one that follows keeps its completion counters at
    an offset inside that region, so it is correct only because the call
    clears them first.  Its results must equal hils_decode on a zeroed
    workspace."""
    import gpu_util as gu
    from chunk_sparse_long_b200 import hils
    big = random_problem(batch=2, n_q_heads=32, n_kv_heads=4, head_dim=64, chunk_size=64,
                         top_k=32, calib_rank=8, seq_len=36000, dtype=hi.DT_BF16, seed=33,
                         spare_pages=2)
    small = random_problem(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, chunk_size=64,
                           top_k=4, calib_rank=8, seq_len=300, dtype=hi.DT_BF16, seed=34,
                           spare_pages=2)
    nb_big = hils.workspace_size(gu.cfg_of(big), hils.OP_DECODE, 1, big.max_chunks)
    nb_small = hils.workspace_size(gu.cfg_of(small), hils.OP_DECODE, 1, small.max_chunks)
    assert nb_small < nb_big // 8 < hils.decode_noalloc_capacity()

    def one_step(p, dp, noalloc):
        t = p.seq_len - 1
        dp.seq_lens.fill_(t + 1)
        B, Hq, d, k = p.batch, p.n_q_heads, p.head_dim, p.top_k
        q = dp.q[:, t].contiguous()
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((B, Hq, k), dtype=torch.int32, device="cuda")
        w = torch.empty((B, Hq, k), dtype=torch.float32, device="cuda")
        if noalloc:
            hils.decode_noalloc(dp.cfg, q, None, None, dp.A, dp.B, dp.cache, out, idx, w)
        else:
            nb = hils.workspace_size(dp.cfg, hils.OP_DECODE, 1, p.max_chunks)
            ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
            hils.decode(dp.cfg, q, None, None, dp.A, dp.B, dp.cache, out, idx, w, ws, nb)
        hils.device_status()
        return idx.cpu().numpy(), w.cpu().numpy(), gu.to_f64(out)

    one_step(big, gu.DevProblem(big), noalloc=True)     # leaves candidate keys in the scratch
    dps = gu.DevProblem(small)
    i1, w1, o1 = one_step(small, dps, noalloc=True)
    i0, w0, o0 = one_step(small, dps, noalloc=False)
    np.testing.assert_array_equal(i1, i0)
    np.testing.assert_allclose(w1, w0, rtol=0, atol=1e-5)
    assert np.abs(o1 - o0).max() <= 2e-2
