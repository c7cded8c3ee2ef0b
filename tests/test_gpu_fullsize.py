"""Parity at the benchmark sizes, in the launch configuration bench.py times.

The full workloads are generated on the device (hils_inputs.device_workload).
The CUDA path runs on all rows. Rows are then checked against the oracle, one
by one.  Selection and fusion weights: every row at 8K (131,072 rows), and at
128K every row of the last 1024 positions plus one row in 64 of the rest
(98,304 rows).  Outputs as well: 64 prefill rows at 128K and at 512K, 256 at
8K, every head of two 512K decode steps, every head of four of the 32
sequences for two B=32 decode steps, and every head of one 4M decode step.
The check applies the same rule as the small tests: selection exact wherever the oracle's score gap exceeds
1e-5, weights within 1e-5, and outputs within 2e-2 (bf16).

The oracle is given a compact page pool. It holds only the chunks that a
checked row can read: its own chunk, and the chunks the oracle or the GPU
selects. That pool is taken from the device after the run, so it also holds
the decode steps' appended tokens. At 4M the planted needle chunks must be
retrieved by every head at step 0.
"""
import numpy as np
import pytest

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _libs():
    import torch
    import hils_inputs as hi
    from chunk_sparse_long_b200 import hils
    from oracle import oracle
    import gpu_util as gu
    hils.load()
    return torch, hi, hils, oracle, gu


def _host(t, dtype, hi):
    import torch
    if dtype == hi.DT_BF16:
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def _cfgs(hils, oracle, w):
    cfg = hils.HilsConfig(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size, w.top_k,
                          w.calib_rank, w.dtype)
    oc = oracle.cfg(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size, w.top_k,
                    w.calib_rank, w.dtype)
    return cfg, oc


def _check_rows(torch, hi, oracle, gu, wl, oc, rows_q, rb, rh, rpos, gpu_idx, gpu_w, gpu_out):
    """Oracle on explicit rows over a compact page pool, compared with the GPU's
    selection, weights and outputs for the same rows."""
    w = wl["workload"]
    A, B = wl["A"].cpu().numpy(), wl["B"].cpu().numpy()
    lm = _host(wl["landmarks"], w.dtype, hi)
    bt = wl["block_table"].cpu().numpy()
    # selection only first: which chunks can the checked rows read?
    sel = oracle.hils_rows(oc, rows_q, rb, rh, rpos, A, B, None, bt, lm)
    need = set()
    for n in range(len(rb)):
        need.add((int(rb[n]), int(rpos[n]) // w.chunk_size))
        for j in list(sel["idx"][n]) + list(gpu_idx[n]):
            if j >= 0:
                need.add((int(rb[n]), int(j)))
    need = sorted(need)
    phys = torch.tensor([int(bt[b, j]) for b, j in need], dtype=torch.long,
                        device=wl["pages"].device)
    pages_c = _host(wl["pages"][phys], w.dtype, hi)
    bt_c = np.zeros_like(bt)
    for n, (b, j) in enumerate(need):
        bt_c[b, j] = n
    orc = oracle.hils_rows(oc, rows_q, rb, rh, rpos, A, B, pages_c, bt_c, lm)

    def rerun(ids, forced):
        return oracle.hils_rows(oc, rows_q[ids], rb[ids], rh[ids], rpos[ids], A, B, pages_c, bt_c,
                                lm, forced_idx=forced)

    return gu.compare(gpu_idx, gpu_w, gpu_out, orc, rerun, w.dtype), orc


def _prefill_sampled(name, n_random, seed):
    torch, hi, hils, oracle, gu = _libs()
    w = hi.WORKLOADS[name]
    wl = hi.device_workload(w)
    cfg, oc = _cfgs(hils, oracle, w)
    L, Hq, k, d = w.seq_len, w.n_q_heads, w.top_k, w.head_dim
    cache = hils.Cache(wl["pages"], wl["num_pages"], wl["block_table"], wl["max_chunks"],
                       wl["landmarks"])
    out = torch.empty_like(wl["q"])
    idx = torch.empty((w.batch, L, Hq, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((w.batch, L, Hq, k), dtype=torch.float32, device="cuda")
    nbytes = hils.workspace_size(cfg, hils.OP_PREFILL, L, wl["max_chunks"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    hils.prefill(cfg, wl["q"], L, 0, wl["A"], wl["B"], cache, out, idx, wts, ws, nbytes)
    hils.device_status()
    # chunk and tile edges, the last rows, and random rows
    rng = np.random.default_rng(seed)
    edges = [e for e in [0, 1, 63, 64, 65, 127, 128, 1983, 1984, 2047, 2048, 8191, 8192]
             if e < L] + [L - 65, L - 64, L - 1]
    pos = np.array(edges + list(rng.integers(0, L, n_random)), dtype=np.int64)
    heads = rng.integers(0, Hq, len(pos)).astype(np.int32)
    bb = rng.integers(0, w.batch, len(pos)).astype(np.int32)
    sel = torch.from_numpy(np.stack([bb, pos, heads], 1)).to("cuda")
    rows_q = _host(wl["q"][sel[:, 0], sel[:, 1], sel[:, 2]], w.dtype, hi)
    g_idx = idx[sel[:, 0], sel[:, 1], sel[:, 2]].cpu().numpy()
    g_w = wts[sel[:, 0], sel[:, 1], sel[:, 2]].cpu().numpy()
    g_out = out[sel[:, 0], sel[:, 1], sel[:, 2]].float().cpu().numpy()
    rep, _ = _check_rows(torch, hi, oracle, gu, wl, oc, rows_q, bb, heads, pos, g_idx, g_w, g_out)
    print(name, rep)


def _prefill_selection_rows(name, pick):
    """Selection and fusion weights of many rows (selection-only oracle: a few
    flops per landmark, so every row at 8K and a dense share at 128K fit in
    one test).  ``pick(L, Hq)`` gives the (position, head) rows to check."""
    torch, hi, hils, oracle, gu = _libs()
    w = hi.WORKLOADS[name]
    wl = hi.device_workload(w)
    cfg, oc = _cfgs(hils, oracle, w)
    L, Hq, k = w.seq_len, w.n_q_heads, w.top_k
    cache = hils.Cache(wl["pages"], wl["num_pages"], wl["block_table"], wl["max_chunks"],
                       wl["landmarks"])
    out = torch.empty_like(wl["q"])
    idx = torch.empty((w.batch, L, Hq, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((w.batch, L, Hq, k), dtype=torch.float32, device="cuda")
    nbytes = hils.workspace_size(cfg, hils.OP_PREFILL, L, wl["max_chunks"])
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    hils.prefill(cfg, wl["q"], L, 0, wl["A"], wl["B"], cache, out, idx, wts, ws, nbytes)
    hils.device_status()
    del ws, out
    pos, heads = pick(L, Hq)
    bb = np.zeros(len(pos), dtype=np.int32)
    sel = torch.from_numpy(np.stack([bb, pos, heads], 1)).to("cuda")
    rows_q = _host(wl["q"][sel[:, 0], sel[:, 1], sel[:, 2]], w.dtype, hi)
    g_idx = idx[sel[:, 0], sel[:, 1], sel[:, 2]].cpu().numpy()
    g_w = wts[sel[:, 0], sel[:, 1], sel[:, 2]].cpu().numpy()
    A, B = wl["A"].cpu().numpy(), wl["B"].cpu().numpy()
    lm = _host(wl["landmarks"], w.dtype, hi)
    bt = wl["block_table"].cpu().numpy()
    orc = oracle.hils_rows(oc, rows_q, bb, heads, pos, A, B, None, bt, lm)

    def rerun(ids, forced):
        return oracle.hils_rows(oc, rows_q[ids], bb[ids], heads[ids], pos[ids], A, B, None, bt, lm,
                                forced_idx=forced)

    rep = gu.compare(g_idx, g_w, None, orc, rerun, w.dtype)
    print(name, len(pos), "rows", rep)
    return len(pos)


def test_prefill_8k_selection_of_every_row_matches_oracle():
    def every_row(L, Hq):
        p, h = np.meshgrid(np.arange(L), np.arange(Hq), indexing="ij")
        return p.reshape(-1).astype(np.int64), h.reshape(-1).astype(np.int32)
    assert _prefill_selection_rows("prefill_8k", every_row) == 8192 * 16


def test_prefill_128k_gqa_selection_of_dense_rows_matches_oracle():
    """Every row of the last 1024 positions (the 8 tiles with the most landmark
    blocks, 16 each) and one row in 64 over the whole sequence."""
    def dense(L, Hq):
        p1, h1 = np.meshgrid(np.arange(L - 1024, L), np.arange(Hq), indexing="ij")
        r = np.arange(0, L * Hq, 64)
        pos = np.concatenate([p1.reshape(-1), r // Hq]).astype(np.int64)
        heads = np.concatenate([h1.reshape(-1), r % Hq]).astype(np.int32)
        return pos, heads
    assert _prefill_selection_rows("prefill_128k_gqa", dense) == 1024 * 32 + 131072 * 32 // 64


def test_prefill_128k_gqa_sampled_rows_match_oracle():
    _prefill_sampled("prefill_128k_gqa", 48, 2024)


def test_prefill_8k_sampled_rows_match_oracle():
    _prefill_sampled("prefill_8k", 240, 2025)


def test_prefill_512k_gqa_in_one_call_sampled_rows_match_oracle():
    """A 512K-token prefill at the 128K GQA shape in one call: its workspace
    (selection, pair records, q~ images; no per-pair partial outputs) fits on
    one GPU next to the inputs."""
    _prefill_sampled("prefill_512k_gqa", 48, 2026)


def _decode_steps(torch, hils, wl, cfg, n_steps):
    """n_steps eager decode steps in the bench's launch configuration; returns
    per step (idx, w, out) on the host."""
    w = wl["workload"]
    cache = hils.Cache(wl["pages"], wl["num_pages"], wl["block_table"], wl["max_chunks"],
                       wl["landmarks"], wl["seq_lens"])
    dt = wl["q_dec"].dtype
    nbytes = hils.workspace_size(cfg, hils.OP_DECODE, 1, wl["max_chunks"])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    res = []
    for s in range(n_steps):
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=dt, device="cuda")
        idx = torch.empty((w.batch, w.n_q_heads, w.top_k), dtype=torch.int32, device="cuda")
        wts = torch.empty((w.batch, w.n_q_heads, w.top_k), dtype=torch.float32, device="cuda")
        hils.decode(cfg, wl["q_dec"][s], wl["k_new"][s], wl["v_new"][s], wl["A"], wl["B"], cache,
                    out, idx, wts, ws, nbytes)
        res.append((idx.cpu().numpy(), wts.cpu().numpy(), out.float().cpu().numpy()))
    hils.device_status()
    return res


def _decode_rows(hi, wl, steps, res, seqs=None):
    """Rows (sequence b in seqs, every head) of the given steps."""
    w = wl["workload"]
    Hq = w.n_q_heads
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    rb, rh, rpos, rq, gi, gw, go = [], [], [], [], [], [], []
    for s in steps:
        for b in seqs:
            for h in range(Hq):
                rb.append(b)
                rh.append(h)
                rpos.append(w.seq_len + s)
            rq.append(_host(wl["q_dec"][s][b], w.dtype, hi))
            gi.append(res[s][0][b])
            gw.append(res[s][1][b])
            go.append(res[s][2][b])
    return (np.concatenate(rq), np.array(rb, np.int32), np.array(rh, np.int32),
            np.array(rpos, np.int64), np.concatenate(gi), np.concatenate(gw), np.concatenate(go))


def test_decode_512k_steps_match_oracle():
    torch, hi, hils, oracle, gu = _libs()
    w = hi.WORKLOADS["decode_512k"]
    wl = hi.device_workload(w)
    cfg, oc = _cfgs(hils, oracle, w)
    res = _decode_steps(torch, hils, wl, cfg, 2)
    assert int(wl["seq_lens"][0]) == w.seq_len + 2
    rq, rb, rh, rpos, gi, gw, go = _decode_rows(hi, wl, [0, 1], res)
    rep, _ = _check_rows(torch, hi, oracle, gu, wl, oc, rq, rb, rh, rpos, gi, gw, go)
    print("decode_512k", rep)


def test_decode_128k_b32_sampled_sequences_match_oracle():
    torch, hi, hils, oracle, gu = _libs()
    w = hi.WORKLOADS["decode_128k_b32"]
    wl = hi.device_workload(w)
    cfg, oc = _cfgs(hils, oracle, w)
    res = _decode_steps(torch, hils, wl, cfg, 2)
    assert (wl["seq_lens"].cpu().numpy() == w.seq_len + 2).all()
    rq, rb, rh, rpos, gi, gw, go = _decode_rows(hi, wl, [0, 1], res, seqs=[0, 7, 19, 31])
    rep, _ = _check_rows(torch, hi, oracle, gu, wl, oc, rq, rb, rh, rpos, gi, gw, go)
    print("decode_128k_b32", rep)


def test_decode_4m_step0_matches_oracle_and_finds_needles():
    torch, hi, hils, oracle, gu = _libs()
    w = hi.WORKLOADS["decode_4m"]
    wl = hi.device_workload(w)
    cfg, oc = _cfgs(hils, oracle, w)
    res = _decode_steps(torch, hils, wl, cfg, 1)
    rq, rb, rh, rpos, gi, gw, go = _decode_rows(hi, wl, [0], res)
    rep, orc = _check_rows(torch, hi, oracle, gu, wl, oc, rq, rb, rh, rpos, gi, gw, go)
    needles = set(int(c) for c in wl["needle_chunks"])
    recall = [len(needles & set(int(j) for j in gi[r])) for r in range(len(rb))]
    print("decode_4m", rep, "needles found per head:", recall)
    assert min(recall) == len(needles), recall
