"""Context-parallel decode (chunk_sparse_long_b200.cp) over two gloo ranks on
the CPU.  The ranks split the chunks of every sequence; each runs the step's
collectives (all-gather of the best k-1 keys and own-chunk scores, all-reduce
of the weighted outputs) around a stand-in for the library's four kernels,
written here in numpy (float64 scores from the oracle, float64 per-chunk
attention).  The step must reproduce the oracle's unsharded decode row: the
same selection, weights and output.  The GPU kernels behind the same step are
checked in tests/test_gpu_cp.py."""
import datetime
import os
import socket

import numpy as np

CHUNK = 8
SPLIT = 12          # rank 0 holds chunks 0..11, rank 1 the rest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _problem():
    from problem import random_problem
    import hils_inputs as hi
    return random_problem(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=16, chunk_size=CHUNK,
                          top_k=4, calib_rank=4, seq_len=200, dtype=hi.DT_F32, seed=21,
                          calib_std=0.3)


def _key(score, j):
    """64-bit selection key of (float32 score, chunk j): a larger key ranks
    higher in (score desc, index asc)."""
    u = int(np.float32(score).view(np.uint32))
    u = (~u & 0xFFFFFFFF) if u & 0x80000000 else (u | 0x80000000)
    return (u << 32) | (0xFFFFFFFF - j)


def _key_score(key):
    u = (key >> 32) & 0xFFFFFFFF
    u = (u & 0x7FFFFFFF) if u & 0x80000000 else (~u & 0xFFFFFFFF)
    return float(np.uint32(u).view(np.float32))


class FakeKernels:
    """The four context-parallel calls in numpy, for one rank's shard."""

    def __init__(self, p, lo, hi_):
        self.p, self.lo, self.hi = p, lo, hi_

    def _pos(self, seq_lens, b, append):
        return int(seq_lens[b]) - (0 if append else 1)

    def candidates(self, cfg, q, k_new, v_new, A, B, shard, chunk_base, keys, own, ws, ws_bytes,
                   stream):
        from oracle import oracle
        from problem import ocfg
        p = self.p
        K = p.top_k - 1
        for b in range(p.batch):
            t = self._pos(shard.seq_lens, b, k_new is not None)
            oc = t // CHUNK
            rb = np.full(p.n_q_heads, b, np.int32)
            rh = np.arange(p.n_q_heads, dtype=np.int32)
            rp = np.full(p.n_q_heads, t, np.int64)
            s = oracle.scores_rows(ocfg(p), q.numpy()[b], rb, rh, rp, p.A, p.B, p.landmarks,
                                   p.max_chunks, p.max_chunks)
            for h in range(p.n_q_heads):
                ks = sorted((_key(s[h, j], j) for j in range(self.lo, min(self.hi, oc))),
                            reverse=True)[:K]
                ks += [0] * (K - len(ks))
                keys[b, h] = torch_int64(ks)
                own[b, h] = float(np.float32(s[h, oc])) if self.lo <= oc < self.hi else -np.inf

    def select(self, cfg, world, all_keys, all_own, seq_lens, append, idx, w, stream):
        p = self.p
        K = p.top_k - 1
        for b in range(p.batch):
            oc = self._pos(seq_lens, b, append) // CHUNK
            for h in range(p.n_q_heads):
                ks = sorted((int(x) & 0xFFFFFFFFFFFFFFFF for x in all_keys[:, b, h].reshape(-1)
                             if int(x) != 0), reverse=True)[:K]
                js = [oc] + [0xFFFFFFFF - (x & 0xFFFFFFFF) for x in ks]
                ss = np.array([float(all_own[:, b, h].max())] + [_key_score(x) for x in ks])
                e = np.exp(ss - ss.max())
                e /= e.sum()
                idx[b, h] = -1
                w[b, h] = 0.0
                idx[b, h, :len(js)] = torch_int32(js)
                w[b, h, :len(js)] = torch_f32(e)

    def attend(self, cfg, q, k_new, v_new, shard, chunk_base, idx, w, partial, stream):
        from problem import to_f64
        p = self.p
        g_of = p.n_q_heads // p.n_kv_heads
        Kf, Vf = to_f64(p.K, p.dtype), to_f64(p.V, p.dtype)
        for b in range(p.batch):
            t = self._pos(shard.seq_lens, b, k_new is not None)
            for h in range(p.n_q_heads):
                g = h // g_of
                qv = to_f64(q.numpy()[b, h], p.dtype)
                acc = np.zeros(p.head_dim)
                for slot in range(p.top_k):
                    j = int(idx[b, h, slot])
                    if j < 0 or not (self.lo <= j < self.hi):
                        continue
                    k0, k1 = j * CHUNK, min((j + 1) * CHUNK, t + 1)
                    s = Kf[b, k0:k1, g] @ qv / np.sqrt(p.head_dim)
                    pr = np.exp(s - s.max())
                    acc += float(w[b, h, slot]) * (pr / pr.sum()) @ Vf[b, k0:k1, g]
                partial[b, h] = torch_f32(acc)

    def finish(self, cfg, total, out, seq_lens, append, stream):
        out.copy_(total)
        if append:
            seq_lens += 1


def torch_int64(v):
    import torch
    return torch.tensor(np.array(v, dtype=np.uint64).view(np.int64))


def torch_int32(v):
    import torch
    return torch.tensor(np.array(v, dtype=np.int32))


def torch_f32(v):
    import torch
    return torch.tensor(np.array(v, dtype=np.float32))


def _worker(rank, world, port, res):
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for x in (root, os.path.join(root, "tests")):
        sys.path.insert(0, x)
    from chunk_sparse_long_b200 import cp, hils
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p = _problem()
        lo, hi_ = (0, SPLIT) if rank == 0 else (SPLIT, p.max_chunks)
        cfg = hils.HilsConfig(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, CHUNK, p.top_k,
                              p.calib_rank, p.dtype)
        seq_lens = torch.full((p.batch,), p.seq_len, dtype=torch.int32)
        shard = hils.Cache(None, 0, None, hi_ - lo, None, seq_lens)
        q = torch.from_numpy(np.ascontiguousarray(p.q[:, p.seq_len - 1]))   # [B][Hq][d]
        out = torch.zeros((p.batch, p.n_q_heads, p.head_dim), dtype=torch.float32)
        dec = cp.Decoder(cfg, shard, lo, kernels=FakeKernels(p, lo, hi_), device="cpu")
        idx, w = dec.step(q, None, None, None, None, out)
        res.put((rank, idx.numpy().copy(), w.numpy().copy(), out.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_unsharded_decode_row():
    import torch.multiprocessing as mp
    from oracle import oracle
    from problem import ocfg
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = _problem()
    t = p.seq_len - 1
    rb, rh = np.meshgrid(np.arange(p.batch), np.arange(p.n_q_heads), indexing="ij")
    rb, rh = rb.reshape(-1).astype(np.int32), rh.reshape(-1).astype(np.int32)
    rp = np.full(rb.shape, t, np.int64)
    orc = oracle.hils_rows(ocfg(p), p.q[rb, t, rh], rb, rh, rp, p.A, p.B, p.pages, p.block_table,
                           p.landmarks)
    assert (orc["gap"] > 1e-6).all()           # no near ties: the selection is unique
    for rank, idx, w, out in res:
        np.testing.assert_array_equal(idx.reshape(-1, p.top_k), orc["idx"])
        np.testing.assert_allclose(w.reshape(-1, p.top_k), orc["w"], rtol=0, atol=1e-6)
        np.testing.assert_allclose(out.reshape(-1, p.head_dim), orc["out"], rtol=0, atol=1e-5)
    # both ranks hold some of the selected chunks, so the all-reduce mattered
    sel = orc["idx"][:, 1:]
    assert (sel[sel >= 0] < SPLIT).any() and (sel[sel >= 0] >= SPLIT).any()
