"""Context-parallel decode kernels (hils_decode_cp_*) on one GPU: two shards of
the chunk range, each a cache of its own over the same page pool, stand in for
two GPUs; the test itself plays the collectives (stacking the shards' key
lists and own scores, summing their weighted outputs).  Every appending step
must match the oracle's decode row under the usual selection rule, and both
shards' seq_lens must advance.  One more case runs the whole range as a
single shard through chunk_sparse_long_b200.cp.Decoder."""
import numpy as np
import pytest
import torch

from problem import ocfg, random_problem
import hils_inputs as hi

pytestmark = pytest.mark.gpu
BF16, F32 = hi.DT_BF16, hi.DT_F32


def _gu():
    import gpu_util
    return gpu_util


def _setup(batch, n_q_heads, n_kv_heads, head_dim, top_k, calib_rank, t0, steps, dtype, seed):
    gu = _gu()
    p = random_problem(batch=batch, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
                       head_dim=head_dim, chunk_size=64, top_k=top_k, calib_rank=calib_rank,
                       seq_len=t0 + 7 * (batch - 1) + steps, dtype=dtype, seed=seed,
                       calib_std=0.2, spare_pages=2)
    t0s = [t0 + 7 * b for b in range(batch)]
    pages = p.pages.copy()
    for b, t in enumerate(t0s):       # the cache starts with the first t0_b tokens
        for x in range(t, p.seq_len):
            pages[p.block_table[b, x // 64], :, :, x % 64, :] = 0
    return gu, p, t0s, gu.dev(pages)


def _shard(gu, p, pages, lo, hi_, t0s):
    from chunk_sparse_long_b200 import hils
    bt = gu.dev(np.ascontiguousarray(p.block_table[:, lo:hi_]))
    lm = gu.dev(np.ascontiguousarray(p.landmarks[:, lo:hi_]))
    sl = torch.tensor(t0s, dtype=torch.int32, device="cuda")
    cache = hils.Cache(pages, p.pages.shape[0], bt, hi_ - lo, lm, sl)
    nbytes = hils.workspace_size(gu.cfg_of(p), hils.OP_DECODE, 1, hi_ - lo)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    return cache, (bt, lm, sl, ws, nbytes)


def _oracle_check(gu, p, t0s, steps, idxs, wts, outs):
    from oracle import oracle
    B, Hq, d, k = p.batch, p.n_q_heads, p.head_dim, p.top_k
    sb, bb, hb = np.meshgrid(np.arange(steps), np.arange(B), np.arange(Hq), indexing="ij")
    rb, rh = bb.reshape(-1).astype(np.int32), hb.reshape(-1).astype(np.int32)
    rp = (np.array(t0s)[rb] + sb.reshape(-1)).astype(np.int64)
    qr = p.q[rb, rp, rh]
    orc = oracle.hils_rows(ocfg(p), qr, rb, rh, rp, p.A, p.B, p.pages, p.block_table, p.landmarks)

    def rerun(rows, forced):
        return oracle.hils_rows(ocfg(p), qr[rows], rb[rows], rh[rows], rp[rows], p.A, p.B, p.pages,
                                p.block_table, p.landmarks, forced)
    return gu.compare(idxs.cpu().numpy().reshape(-1, k), wts.cpu().numpy().reshape(-1, k),
                      gu.to_f64(outs).reshape(-1, d), orc, rerun, p.dtype), orc


@pytest.mark.parametrize("case", [
    dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, top_k=8, calib_rank=8, t0=3000,
         steps=6, dtype=BF16, seed=31),
    dict(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=128, top_k=16, calib_rank=16, t0=1500,
         steps=4, dtype=F32, seed=32),
])
def test_two_shards_match_oracle(case):
    from chunk_sparse_long_b200 import hils
    gu, p, t0s, pages = _setup(**case)
    split = p.max_chunks // 2
    shards = [_shard(gu, p, pages, 0, split, t0s), _shard(gu, p, pages, split, p.max_chunks, t0s)]
    bases = [0, split]
    cfg = gu.cfg_of(p)
    steps = case["steps"]
    B, Hq, Hkv, d, k = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.top_k
    K = max(k - 1, 1)
    odt = torch.float32 if p.dtype == F32 else torch.bfloat16
    outs = torch.empty((steps, B, Hq, d), dtype=odt, device="cuda")
    scratch = torch.empty((B, Hq, d), dtype=odt, device="cuda")
    idxs = torch.empty((steps, B, Hq, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((steps, B, Hq, k), dtype=torch.float32, device="cuda")
    qdev, Kd, Vd = gu.dev(p.q), gu.dev(p.K), gu.dev(p.V)
    A, Bm = gu.dev(p.A), gu.dev(p.B)
    for s in range(steps):
        ts = [t0 + s for t0 in t0s]
        q = torch.stack([qdev[b, ts[b]] for b in range(B)]).contiguous()
        kn = torch.stack([Kd[b, ts[b]] for b in range(B)]).contiguous()
        vn = torch.stack([Vd[b, ts[b]] for b in range(B)]).contiguous()
        keys = torch.zeros((2, B, Hq, K), dtype=torch.int64, device="cuda")
        own = torch.empty((2, B, Hq), dtype=torch.float32, device="cuda")
        for r, (cache, (_, _, _, ws, nbytes)) in enumerate(shards):
            hils.decode_cp_candidates(cfg, q, kn, vn, A, Bm, cache, bases[r], keys[r], own[r], ws,
                                      nbytes)
        hils.decode_cp_select(cfg, 2, keys, own, shards[0][1][2], True, idxs[s], wts[s])
        total = torch.zeros((B, Hq, d), dtype=torch.float32, device="cuda")
        for r, (cache, _) in enumerate(shards):
            part = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
            hils.decode_cp_attend(cfg, q, kn, vn, cache, bases[r], idxs[s], wts[s], part)
            total += part
        hils.decode_cp_finish(cfg, total, outs[s], shards[0][1][2], True)
        hils.decode_cp_finish(cfg, total, scratch, shards[1][1][2], True)
    hils.device_status()
    for _, (_, _, sl, _, _) in shards:
        assert sl.cpu().tolist() == [t0 + steps for t0 in t0s]
    rep, orc = _oracle_check(gu, p, t0s, steps, idxs, wts, outs)
    # both shards contributed selected chunks
    sel = orc["idx"][:, 1:]
    assert (sel[sel >= 0] < split).any() and (sel[sel >= 0] >= split).any()
    print(case, rep)


def test_one_shard_through_decoder_matches_oracle():
    from chunk_sparse_long_b200 import cp
    gu, p, t0s, pages = _setup(batch=2, n_q_heads=4, n_kv_heads=4, head_dim=64, top_k=4,
                               calib_rank=8, t0=900, steps=3, dtype=BF16, seed=33)
    cache, _ = _shard(gu, p, pages, 0, p.max_chunks, t0s)
    cfg = gu.cfg_of(p)
    dec = cp.Decoder(cfg, cache, 0)
    B, Hq, d, k, steps = p.batch, p.n_q_heads, p.head_dim, p.top_k, 3
    outs = torch.empty((steps, B, Hq, d), dtype=torch.bfloat16, device="cuda")
    idxs = torch.empty((steps, B, Hq, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((steps, B, Hq, k), dtype=torch.float32, device="cuda")
    qdev, Kd, Vd = gu.dev(p.q), gu.dev(p.K), gu.dev(p.V)
    A, Bm = gu.dev(p.A), gu.dev(p.B)
    for s in range(steps):
        ts = [t0 + s for t0 in t0s]
        q = torch.stack([qdev[b, ts[b]] for b in range(B)]).contiguous()
        kn = torch.stack([Kd[b, ts[b]] for b in range(B)]).contiguous()
        vn = torch.stack([Vd[b, ts[b]] for b in range(B)]).contiguous()
        i, w = dec.step(q, kn, vn, A, Bm, outs[s])
        idxs[s].copy_(i)
        wts[s].copy_(w)
    from chunk_sparse_long_b200 import hils
    hils.device_status()
    rep, _ = _oracle_check(gu, p, t0s, steps, idxs, wts, outs)
    print(rep)
