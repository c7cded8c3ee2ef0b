"""GPU parity of the C-ABI library against the CPU oracle on small seeded problems.

Sizes span several tiles (128-row selection tiles, 64-key chunks, 128-pair
attention tiles) with ragged tails; cases cover GQA, both head sizes, both
storage types, fewer visible chunks than k, top-1, chunked prefill
(q_pos0 > 0), no calibration, and decode steps that append tokens and cross a
chunk boundary.  Tolerances: chunk indices bit-exact where the oracle's gap
exceeds 1e-5; outputs max-abs <= 1e-3 (float32 storage) or <= 2e-2 (bf16);
fusion weights within 1e-5.
"""
import numpy as np
import pytest
import torch

import hils_inputs as hi
from problem import ocfg, random_problem, to_f64

pytestmark = pytest.mark.gpu

F32, BF16 = hi.DT_F32, hi.DT_BF16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from chunk_sparse_long_b200 import build, hils
    build.build()
    hils.load()


def _gu():
    import gpu_util
    return gpu_util


PREFILL_CASES = {
    # the tiny float32 correctness workload: B1 H2 d64 L1024 S64 k4 r8, seed 0
    "tiny_f32_workload": dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, top_k=4,
                              calib_rank=8, seq_len=1024, dtype=F32, seed=0),
    "bf16_d64_ragged_b2": dict(batch=2, n_q_heads=4, n_kv_heads=4, head_dim=64, top_k=5,
                               calib_rank=16, seq_len=1000, dtype=BF16, seed=1),
    "bf16_d128_gqa": dict(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, top_k=8,
                          calib_rank=32, seq_len=1500, dtype=BF16, seed=2),
    "f32_d128_gqa": dict(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=128, top_k=6,
                         calib_rank=4, seq_len=777, dtype=F32, seed=3),
    "k_exceeds_visible_chunks": dict(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, top_k=16,
                                     calib_rank=8, seq_len=300, dtype=BF16, seed=4),
    "top1": dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, top_k=1, calib_rank=8,
                 seq_len=400, dtype=BF16, seed=5),
    "top32_max": dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, top_k=32, calib_rank=64,
                      seq_len=3000, dtype=BF16, seed=6),
    "chunked_prefill": dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, top_k=4,
                            calib_rank=8, seq_len=1300, q_pos0=700, dtype=BF16, seed=7),
    "no_calibration": dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=128, top_k=4,
                           calib_rank=0, seq_len=520, dtype=BF16, seed=8),
    "single_chunk": dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, top_k=4, calib_rank=8,
                         seq_len=37, dtype=F32, seed=9),
}


def _oracle_rerun(p):
    from oracle import oracle
    qr, rb, rh, rp = p.rows()

    def rerun(rows, forced):
        return oracle.hils_rows(ocfg(p), qr[rows], rb[rows], rh[rows], rp[rows], p.A, p.B, p.pages,
                                p.block_table, p.landmarks, forced)
    return rerun


@pytest.mark.parametrize("name", sorted(PREFILL_CASES))
def test_prefill_matches_oracle(name):
    gu = _gu()
    from problem import run_oracle
    p = random_problem(chunk_size=64, spare_pages=3, **PREFILL_CASES[name])
    dp = gu.DevProblem(p)
    out, idx, w = gu.run_prefill(dp, ws_pad=512)
    orc = run_oracle(p)
    rep = gu.compare(idx.cpu().numpy(), w.cpu().numpy(), gu.to_f64(out).reshape(-1, p.head_dim),
                     orc, _oracle_rerun(p), p.dtype)
    print(name, rep)


@pytest.mark.parametrize("dtype,head_dim", [(BF16, 128), (BF16, 64), (F32, 64)])
def test_prefill_tied_scores_keep_the_lowest_chunks(dtype, head_dim):
    """Every chunk of a KV head carries the same landmark, so all of a row's
    scores tie and the order (score desc, index asc) fixes the selection:
    idx = [own, 0, 1, .., k-2] (fewer when fewer chunks are visible), with
    uniform weights.  At 8192 positions a row sees up to 127 candidates, more
    than a collection buffer holds, so the cut of a full buffer to its best
    k-1 runs on every long row."""
    gu = _gu()
    p = random_problem(chunk_size=64, batch=1, n_q_heads=4, n_kv_heads=2, head_dim=head_dim,
                       top_k=32, calib_rank=8, seq_len=8192, dtype=dtype, seed=21)
    p.landmarks[:] = p.landmarks[:, :1]
    dp = gu.DevProblem(p)
    out, idx, w = gu.run_prefill(dp)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    _, _, _, rp = p.rows()
    own = rp // 64
    n_sel = np.minimum(own, p.top_k - 1)
    exp = np.full(idx.shape, -1, dtype=np.int32)
    exp[:, 0] = own
    for r in range(idx.shape[0]):
        exp[r, 1:1 + n_sel[r]] = np.arange(n_sel[r])
    np.testing.assert_array_equal(idx, exp)
    exp_w = np.where(exp >= 0, 1.0 / (1 + n_sel)[:, None], 0.0)
    np.testing.assert_allclose(w, exp_w, rtol=0, atol=1e-6)
    # outputs against the oracle on every 16th row
    from oracle import oracle
    qr, rb, rh, rp = p.rows()
    sel = np.arange(0, qr.shape[0], 16)
    orc = oracle.hils_rows(ocfg(p), qr[sel], rb[sel], rh[sel], rp[sel], p.A, p.B, p.pages,
                           p.block_table, p.landmarks)
    np.testing.assert_array_equal(orc["idx"], exp[sel])

    def rerun(rows, forced):
        s_ = sel[rows]
        return oracle.hils_rows(ocfg(p), qr[s_], rb[s_], rh[s_], rp[s_], p.A, p.B, p.pages,
                                p.block_table, p.landmarks, forced)
    rep = gu.compare(idx[sel], w[sel], gu.to_f64(out).reshape(-1, p.head_dim)[sel], orc, rerun,
                     p.dtype)
    print(rep)


def test_prefill_outputs_only_4_byte_aligned():
    """idx and w need only int32 / float alignment: views one element into
    larger buffers must receive exactly what aligned buffers receive."""
    gu = _gu()
    from chunk_sparse_long_b200 import hils
    p = random_problem(chunk_size=64, **PREFILL_CASES["bf16_d128_gqa"])   # k = 8
    dp = gu.DevProblem(p)
    out, idx, w = gu.run_prefill(dp)
    rows = p.batch * p.q_len * p.n_q_heads
    ibuf = torch.full((rows * p.top_k + 1,), -7, dtype=torch.int32, device="cuda")
    wbuf = torch.full((rows * p.top_k + 1,), -7.0, dtype=torch.float32, device="cuda")
    idx_u, w_u = ibuf[1:].view(rows, p.top_k), wbuf[1:].view(rows, p.top_k)
    assert idx_u.data_ptr() % 16 == 4 and w_u.data_ptr() % 16 == 4
    out2 = torch.empty_like(out)
    nbytes = hils.workspace_size(dp.cfg, hils.OP_PREFILL, p.q_len, p.max_chunks)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    hils.prefill(dp.cfg, dp.q, p.q_len, p.q_pos0, dp.A, dp.B, dp.cache, out2, idx_u, w_u, ws, nbytes)
    hils.device_status()
    assert int(ibuf[0]) == -7 and float(wbuf[0]) == -7.0
    assert torch.equal(idx_u, idx) and torch.equal(w_u, w)
    # the bf16 output sums a row's k shares by atomic additions in no fixed
    # order, so two runs agree to the rounding of those additions only
    assert float((out2.float() - out.float()).abs().max()) <= 2e-2


@pytest.mark.parametrize("name", ["tiny_f32_workload", "bf16_d128_gqa", "chunked_prefill"])
def test_score_and_topk_match_oracle(name):
    gu = _gu()
    from chunk_sparse_long_b200 import hils
    from oracle import oracle
    p = random_problem(chunk_size=64, **PREFILL_CASES[name])
    dp = gu.DevProblem(p)
    n_cols = p.max_chunks
    rows = p.batch * p.q_len * p.n_q_heads
    scores = torch.empty((rows, n_cols), dtype=torch.float32, device="cuda")
    hils.score(dp.cfg, dp.q, p.q_len, p.q_pos0, dp.A, dp.B, dp.cache, scores, n_cols)
    idx = torch.empty((rows, p.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((rows, p.top_k), dtype=torch.float32, device="cuda")
    hils.topk(dp.cfg, scores, p.q_len, p.q_pos0, n_cols, idx, w)
    hils.device_status()
    qr, rb, rh, rp = p.rows()
    s_or = oracle.scores_rows(ocfg(p), qr, rb, rh, rp, p.A, p.B, p.landmarks, p.max_chunks, n_cols)
    s_gpu = scores.cpu().numpy().astype(np.float64)
    assert (np.isinf(s_or) == np.isinf(s_gpu)).all()
    fin = np.isfinite(s_or)
    np.testing.assert_allclose(s_gpu[fin], s_or[fin], rtol=1e-5, atol=2e-5)
    # selection on identical inputs (the GPU's float32 scores) must be bit-exact
    oi, ow, _ = oracle.topk_rows(s_gpu, rp, 64, p.top_k)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)
    np.testing.assert_allclose(w.cpu().numpy(), ow, rtol=0, atol=2e-6)


def _decode_problem(batch, n_q_heads, n_kv_heads, head_dim, top_k, calib_rank, t0, steps, dtype,
                    seed):
    p = random_problem(batch=batch, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=head_dim,
                       chunk_size=64, top_k=top_k, calib_rank=calib_rank,
                       seq_len=t0 + 7 * (batch - 1) + steps, dtype=dtype, seed=seed, spare_pages=2)
    t0s = [t0 + 7 * b for b in range(batch)]
    return p, t0s


@pytest.mark.parametrize("case", [
    dict(batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, top_k=4, calib_rank=8, t0=1000,
         steps=70, dtype=BF16, seed=11),
    dict(batch=3, n_q_heads=8, n_kv_heads=2, head_dim=128, top_k=6, calib_rank=16, t0=2000,
         steps=20, dtype=BF16, seed=12),
    dict(batch=2, n_q_heads=2, n_kv_heads=2, head_dim=64, top_k=16, calib_rank=8, t0=100,
         steps=40, dtype=F32, seed=13),
    # every landmark of a KV head the same: all scores tie, so each step must
    # keep chunks 0 .. k-2; 516+ chunks span two scan ranges at d=64 bf16
    dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, top_k=16, calib_rank=8, t0=33000,
         steps=12, dtype=BF16, seed=14, tied=True),
])
def test_decode_steps_match_oracle(case):
    """Each step appends (k_t, v_t) and attends at t; step s of sequence b is
    row t = t0_b + s of the prefill over the same tokens."""
    gu = _gu()
    from chunk_sparse_long_b200 import hils
    from oracle import oracle
    case = dict(case)
    tied = case.pop("tied", False)
    p, t0s = _decode_problem(**case)
    if tied:
        p.landmarks[:] = p.landmarks[:, :1]
    dp = gu.DevProblem(p)
    # the device cache starts with only the first t0_b tokens of each sequence
    pages = p.pages.copy()
    for b, t0 in enumerate(t0s):
        for t in range(t0, p.seq_len):
            pg = p.block_table[b, t // 64]
            pages[pg, :, :, t % 64, :] = 0
    dp.pages.copy_(gu.dev(pages))
    dp.seq_lens.copy_(torch.tensor(t0s, dtype=torch.int32))
    nbytes = hils.workspace_size(dp.cfg, hils.OP_DECODE, 1, p.max_chunks)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    steps = case["steps"]
    B, Hq, Hkv, d, k = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.top_k
    odt = torch.float32 if p.dtype == F32 else torch.bfloat16
    outs = torch.empty((steps, B, Hq, d), dtype=odt, device="cuda")
    idxs = torch.empty((steps, B, Hq, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((steps, B, Hq, k), dtype=torch.float32, device="cuda")
    qdev = dp.q                    # [B][L][Hq][d] (all positions)
    Kd, Vd = gu.dev(p.K), gu.dev(p.V)
    for s in range(steps):
        ts = [t0 + s for t0 in t0s]
        q = torch.stack([qdev[b, ts[b]] for b in range(B)]).contiguous()
        kn = torch.stack([Kd[b, ts[b]] for b in range(B)]).contiguous()
        vn = torch.stack([Vd[b, ts[b]] for b in range(B)]).contiguous()
        hils.decode(dp.cfg, q, kn, vn, dp.A, dp.B, dp.cache, outs[s], idxs[s], wts[s], ws, nbytes)
    hils.device_status()
    assert dp.seq_lens.cpu().tolist() == [t0 + steps for t0 in t0s]
    # oracle rows: (step, b, h) at t = t0_b + step, on the full (appended) cache
    sb, bb, hb = np.meshgrid(np.arange(steps), np.arange(B), np.arange(Hq), indexing="ij")
    rb, rh = bb.reshape(-1).astype(np.int32), hb.reshape(-1).astype(np.int32)
    rp = (np.array(t0s)[rb] + sb.reshape(-1)).astype(np.int64)
    qr = p.q[rb, rp, rh]
    orc = oracle.hils_rows(ocfg(p), qr, rb, rh, rp, p.A, p.B, p.pages, p.block_table, p.landmarks)

    def rerun(rows, forced):
        return oracle.hils_rows(ocfg(p), qr[rows], rb[rows], rh[rows], rp[rows], p.A, p.B, p.pages,
                                p.block_table, p.landmarks, forced)
    if tied:
        own = rp // 64
        n_sel = np.minimum(own, k - 1)
        exp = np.full((rp.shape[0], k), -1, dtype=np.int32)
        exp[:, 0] = own
        for r in range(rp.shape[0]):
            exp[r, 1:1 + n_sel[r]] = np.arange(n_sel[r])
        np.testing.assert_array_equal(idxs.cpu().numpy().reshape(-1, k), exp)
        np.testing.assert_array_equal(orc["idx"], exp)
    rep = gu.compare(idxs.cpu().numpy().reshape(-1, k), wts.cpu().numpy().reshape(-1, k),
                     gu.to_f64(outs).reshape(-1, d), orc, rerun, p.dtype)
    print(case, rep)


def test_decode_equals_prefill_rows_on_gpu():
    """Decode at t (cache already holding token t) equals prefill row t."""
    gu = _gu()
    from chunk_sparse_long_b200 import hils
    p = random_problem(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=64, chunk_size=64, top_k=6,
                       calib_rank=8, seq_len=900, dtype=BF16, seed=21)
    dp = gu.DevProblem(p)
    out_p, idx_p, w_p = gu.run_prefill(dp)
    nbytes = hils.workspace_size(dp.cfg, hils.OP_DECODE, 1, p.max_chunks)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for t in (0, 63, 64, 500, 899):
        dp.seq_lens.fill_(t + 1)
        out = torch.empty((1, 4, 64), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((1, 4, 6), dtype=torch.int32, device="cuda")
        w = torch.empty((1, 4, 6), dtype=torch.float32, device="cuda")
        q = dp.q[:, t].contiguous()
        hils.decode(dp.cfg, q, None, None, dp.A, dp.B, dp.cache, out, idx, w, ws, nbytes)
        hils.device_status()
        np.testing.assert_array_equal(idx.cpu().numpy().reshape(4, 6),
                                      idx_p.cpu().numpy().reshape(900, 4, 6)[t])
        np.testing.assert_allclose(w.cpu().numpy().reshape(4, 6),
                                   w_p.cpu().numpy().reshape(900, 4, 6)[t], atol=1e-6)
        # both paths are checked against the oracle elsewhere at max-abs 2e-2; here the
        # CUDA-core decode and the tensor-core prefill (bf16 P, bf16 sums) agree to 2e-2
        np.testing.assert_allclose(gu.to_f64(out).reshape(4, 64),
                                   gu.to_f64(out_p).reshape(900, 4, 64)[t], atol=2e-2)


def test_bad_block_table_entry_reports_device_error():
    """A block-table entry outside the page pool is caught by the kernels'
    bounds check: the access is skipped and the device error word is set."""
    gu = _gu()
    from chunk_sparse_long_b200 import hils
    p = random_problem(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, chunk_size=64, top_k=4,
                       calib_rank=8, seq_len=512, dtype=BF16, seed=22)
    dp = gu.DevProblem(p)
    dp.bt[0, 3] = p.pages.shape[0] + 5
    with pytest.raises(hils.HilsError) as e:
        gu.run_prefill(dp)
    assert e.value.status == 6
    hils.device_status()           # cleared after being reported
