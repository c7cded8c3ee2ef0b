"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test ties the oracle to something other than its own code: a
hand-derived worked example, special cases that reduce to a library routine
(torch's scaled_dot_product_attention in float64), brute-force sorting, and
closed forms of the calibration.  Method citations are to the pages of
"Hierarchical Sparse Attention Done Right" (HiLS): the ai-feeds.com digest,
section 方法, and the chatpaper abstract.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import hils_inputs as hi
from oracle import oracle
from problem import Problem, paged_from_logical, random_problem, run_oracle, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa(q, k, v, mask=None, causal=False):
    """torch SDPA in float64 on [H][L][d] arrays (library routine)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal)
    return o[0].numpy()


# ---------------------------------------------------------------- generator
def test_splitmix64_reference_outputs():
    ref = json.load(open(os.path.join(GOLDEN, "splitmix64_reference.json")))
    got = [int(hi.sm64(np.array([0], dtype=np.uint64))[0]),
           int(hi.sm64(np.array([hi.GOLDEN], dtype=np.uint64))[0])]
    assert [hex(x) for x in got] == ref["outputs_hex"]


def test_normal_stream_moments_and_determinism():
    x = hi.normal_f64(7, hi.TID_Q, 0, 200_000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    y = hi.normal_f64(7, hi.TID_Q, 1000, 10)
    np.testing.assert_array_equal(x[1000:1010], y)          # counter-based: any element alone
    z = hi.normal_f64(7, hi.TID_LM, 0, 10)
    assert not np.allclose(x[:10], z)                        # streams differ per tensor


def test_bf16_rounding_is_rne_like_torch():
    v = hi.normal(3, hi.TID_Q, 0, 100_000, 3.0, hi.DT_F32)
    ours = hi.normal(3, hi.TID_Q, 0, 100_000, 3.0, hi.DT_BF16)
    theirs = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, theirs)


# ----------------------------------------------------------- worked example
def test_worked_example_closed_forms():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_d1.json")))
    c = g["config"]
    S, L = c["chunk_size"], c["seq_len"]
    K = np.array(g["K"], np.float32).reshape(1, L, 1, 1)
    V = np.array(g["V"], np.float32).reshape(1, L, 1, 1)
    mc = (L + S - 1) // S
    pages, bt = paged_from_logical(K, V, S, mc, perm=np.array([2, 0, 1], np.int32))
    lm = np.array(g["landmarks"], np.float32).reshape(1, mc, 1, 1)
    rows = g["expected"]
    q_rows = np.array([g["q_by_head"][r["head"]] for r in rows], np.float32).reshape(-1, 1)
    oc = oracle.cfg(c["batch"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"], S, c["top_k"],
                    c["calib_rank"], 0)
    res = oracle.hils_rows(oc, q_rows, [0] * len(rows), [r["head"] for r in rows],
                           [r["pos"] for r in rows], np.array(g["A"], np.float32),
                           np.array(g["B"], np.float32), pages, bt, lm)
    ev = lambda s: eval(s, {"__builtins__": {}}, {"e": math.e})
    for n, r in enumerate(rows):
        assert res["idx"][n].tolist() == r["idx"], r
        np.testing.assert_allclose(res["w"][n], [ev(x) for x in r["w"]], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(res["out"][n, 0], ev(r["out"]), rtol=1e-13, atol=1e-15)


# ------------------------------------------- reductions to dense attention
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2)])
def test_chunk1_landmark_equals_key_is_dense_causal_attention(hq, hkv):
    """S=1, landmark_j = k_j, B=0 (so q~=q) and k >= L: the selected chunks are
    all causal keys, each chunk output is its v, and the fusion softmax is the
    dense softmax over q.k/sqrt(d)."""
    L, d = 40, 16
    p = random_problem(n_q_heads=hq, n_kv_heads=hkv, head_dim=d, chunk_size=1, top_k=L,
                       calib_rank=3, seq_len=L, seed=11, calib_std=0.5)
    p.B[:] = 0.0
    p.landmarks = p.K.copy()                      # [B][T][Hkv][d] == [B][chunks][Hkv][d]
    res = run_oracle(p)
    out = res["out"].reshape(L, hq, d).transpose(1, 0, 2)
    rep = hq // hkv
    q = to_f64(p.q[0], 0).transpose(1, 0, 2)
    k = np.repeat(to_f64(p.K[0], 0).transpose(1, 0, 2), rep, axis=0)
    v = np.repeat(to_f64(p.V[0], 0).transpose(1, 0, 2), rep, axis=0)
    np.testing.assert_allclose(out, sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(res["w"].sum(1), 1.0, rtol=1e-13)


def test_single_chunk_is_plain_causal_attention_with_raw_q():
    """L <= S: only the own chunk exists, so landmarks and calibration have no
    effect and the output is causal attention of the raw query."""
    L, d = 24, 8
    p = random_problem(head_dim=d, chunk_size=32, top_k=4, calib_rank=4, seq_len=L, seed=5,
                       calib_std=0.7)
    res = run_oracle(p)
    out = res["out"].reshape(L, 2, d).transpose(1, 0, 2)
    q, k, v = (to_f64(x[0], 0).transpose(1, 0, 2) for x in (p.q, p.K, p.V))
    np.testing.assert_allclose(out, sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-12)


def test_top1_is_block_diagonal_causal_attention():
    """k=1: every query attends only to its own chunk, causally."""
    L, d, S = 48, 8, 8
    p = random_problem(head_dim=d, chunk_size=S, top_k=1, seq_len=L, seed=6, calib_std=0.5)
    res = run_oracle(p)
    out = res["out"].reshape(L, 2, d).transpose(1, 0, 2)
    i = np.arange(L)
    mask = (i[:, None] // S == i[None, :] // S) & (i[None, :] <= i[:, None])
    q, k, v = (to_f64(x[0], 0).transpose(1, 0, 2) for x in (p.q, p.K, p.V))
    np.testing.assert_allclose(out, sdpa(q, k, v, mask=mask), rtol=1e-11, atol=1e-12)
    assert (res["idx"][:, 0] == np.repeat(i // S, 2)).all()


def test_constant_landmarks_pick_lowest_chunks_and_average():
    """All landmarks of a head equal: every score ties, so the tie rule picks
    chunks 0..k-2 besides the own chunk, the weights are uniform, and the
    output is the mean of the per-chunk attention outputs."""
    L, d, S, k = 64, 8, 8, 3
    p = random_problem(head_dim=d, chunk_size=S, top_k=k, seq_len=L, seed=8)
    p.landmarks[:] = p.landmarks[:, :1]          # chunk 0's landmark everywhere
    res = run_oracle(p)
    q, kk, v = (to_f64(x[0], 0) for x in (p.q, p.K, p.V))     # [L][H][d]
    for pos in range(L):
        own = pos // S
        want_idx = [own] + list(range(min(k - 1, own))) + [-1] * (k - 1 - min(k - 1, own))
        for h in range(2):
            r = pos * 2 + h
            assert res["idx"][r].tolist() == want_idx
            n = 1 + min(k - 1, own)
            np.testing.assert_allclose(res["w"][r][:n], 1.0 / n, rtol=1e-13)
            outs = []
            for j in want_idx[:n]:
                t0, t1 = j * S, min(j * S + S, pos + 1)
                outs.append(sdpa(q[pos:pos + 1, h][None], kk[t0:t1, h][None], v[t0:t1, h][None])[0, 0])
            np.testing.assert_allclose(res["out"][r], np.mean(outs, axis=0), rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------- selection
def test_selection_matches_bruteforce_sort_with_ties():
    rng = np.random.default_rng(0)
    S, k = 4, 5
    for trial in range(300):
        n_cols = int(rng.integers(1, 20))
        pos = int(rng.integers(0, n_cols * S))
        s = rng.integers(-3, 4, size=n_cols).astype(np.float64) * 0.5   # many exact ties
        s[pos // S + 1:] = -np.inf
        idx, w, gap = oracle.topk_rows(s[None], [pos], S, k)
        own = pos // S
        cands = sorted(range(own), key=lambda j: (-s[j], j))[: k - 1]
        want = [own] + cands + [-1] * (k - 1 - len(cands))
        assert idx[0].tolist() == want, (s, pos)
        sel = s[[own] + cands]
        e = np.exp(sel - sel.max())
        np.testing.assert_allclose(w[0][: len(sel)], e / e.sum(), rtol=1e-14)
        assert (w[0][len(sel):] == 0).all()
        left = [s[j] for j in range(own) if j not in cands]
        if cands and left:
            assert gap[0] == s[cands[-1]] - max(left)
        else:
            assert gap[0] == np.inf


# ------------------------------------------------------------ calibration
def test_calibration_rank1_closed_forms():
    """A = u (d x 1), B = v^T (1 x d): q~ = q + (q.u) v.  For q orthogonal to u
    the query is unchanged; for q = u/|u|^2 it moves by exactly v."""
    d = 6
    u = np.array([1, 2, 0, -1, 0, 0.5], np.float32)
    v = np.array([0.25, -1, 3, 0, 0.5, 2], np.float32)
    A, B = u[:, None], v[None, :]
    q_orth = np.array([2, -1, 5, 0, 7, 0], np.float64)          # u.q_orth == 0
    np.testing.assert_allclose(oracle.calibrate(q_orth, A, B), q_orth, rtol=0, atol=1e-15)
    q_u = u.astype(np.float64) / float(u.astype(np.float64) @ u)
    np.testing.assert_allclose(oracle.calibrate(q_u, A, B), q_u + v, rtol=1e-14, atol=1e-15)
    # the transposed product (q.v) u would differ: guard against a swapped operand
    assert not np.allclose(q_u + (q_u @ v) * u, q_u + v)


def test_calibration_rank2_closed_form():
    """A = [u1 u2] (d x 2), B = [v1; v2] (2 x d): q~ = q + (q.u1) v1 + (q.u2) v2.
    With u1, u2 orthogonal, q = u2/|u2|^2 has q.u1 = 0 and q.u2 = 1, so q~ = q + v2."""
    d = 5
    u1 = np.array([1, 1, 0, 0, 0], np.float32)
    u2 = np.array([1, -1, 2, 0, 0], np.float32)
    v1 = np.array([3, 0, 0, 1, 0], np.float32)
    v2 = np.array([0, 0.5, 0, 0, -2], np.float32)
    A = np.stack([u1, u2], axis=1)            # [d][2]
    B = np.stack([v1, v2], axis=0)            # [2][d]
    q = u2.astype(np.float64) / float(u2.astype(np.float64) @ u2)
    np.testing.assert_allclose(oracle.calibrate(q, A, B), q + v2, rtol=1e-14, atol=1e-15)
    q1 = u1.astype(np.float64) / 2.0          # q.u1 = 1, q.u2 = 0
    np.testing.assert_allclose(oracle.calibrate(q1, A, B), q1 + v1, rtol=1e-14, atol=1e-15)


def test_calibrated_query_drives_selection_but_not_attention():
    """q = e0 prefers chunk 0's landmark; the calibration q~ = q + (q.e0)(e1 - e0)
    turns it into e1, which prefers chunk 1.  Retrieval must follow q~."""
    d, S, L = 2, 2, 6
    K = np.zeros((1, L, 1, d), np.float32)
    V = np.arange(L * d, dtype=np.float32).reshape(1, L, 1, d)
    pages, bt = paged_from_logical(K, V, S, 3)
    lm = np.array([[[[1, 0]], [[0, 1]], [[0, 0]]]], np.float32)
    A = np.array([[1.0], [0.0]], np.float32)
    B = np.array([[-1.0, 1.0]], np.float32)
    oc = oracle.cfg(1, 1, 1, d, S, 2, 1, 0)
    q = np.array([[1.0, 0.0]], np.float32)
    res = oracle.hils_rows(oc, q, [0], [0], [5], A, B, pages, bt, lm)
    assert res["idx"][0].tolist() == [2, 1]
    res0 = oracle.hils_rows(oc, q, [0], [0], [5], A, 0 * B, pages, bt, lm)
    assert res0["idx"][0].tolist() == [2, 0]
    # keys are zero, so each chunk output is the plain mean of its values
    w = res["w"][0]
    np.testing.assert_allclose(res["out"][0], w[0] * V[0, 4:6, 0].mean(0) + w[1] * V[0, 2:4, 0].mean(0),
                               rtol=1e-14)


# ------------------------------------------------------------- invariants
def test_invariants_weights_convexity_and_page_permutation():
    p = random_problem(n_q_heads=4, n_kv_heads=2, head_dim=16, chunk_size=8, top_k=4, seq_len=96,
                       seed=21, spare_pages=5)
    res = run_oracle(p)
    np.testing.assert_allclose(res["w"].sum(1), 1.0, rtol=1e-13)
    assert (res["w"] >= 0).all()
    # each output coordinate is a convex combination of the selected V rows
    _, rb, rh, rp = p.rows()
    V = to_f64(p.V, 0)
    for r in range(0, len(rb), 7):
        g = rh[r] // 2
        toks = [t for j in res["idx"][r] if j >= 0 for t in range(j * 8, min(j * 8 + 8, rp[r] + 1))]
        vv = V[rb[r], toks, g]
        assert (res["out"][r] <= vv.max(0) + 1e-12).all() and (res["out"][r] >= vv.min(0) - 1e-12).all()
    # physical page order does not matter
    q = random_problem(n_q_heads=4, n_kv_heads=2, head_dim=16, chunk_size=8, top_k=4, seq_len=96,
                       seed=21, spare_pages=5, permute_pages=False)
    res2 = run_oracle(q)
    np.testing.assert_array_equal(res["idx"], res2["idx"])
    np.testing.assert_array_equal(res["out"], res2["out"])


def test_forced_selection_reproduces_own_choice_and_bf16_storage():
    p = random_problem(head_dim=16, chunk_size=8, top_k=3, seq_len=80, seed=4, dtype=hi.DT_BF16)
    res = run_oracle(p)
    res2 = run_oracle(p, forced_idx=res["idx"])
    np.testing.assert_array_equal(res["out"], res2["out"])
    np.testing.assert_array_equal(res["w"], res2["w"])
    # decode row == prefill row: a query at position t over a cache of t+1 tokens
    t = 57
    qr, rb, rh, rp = p.rows()
    sel = (rp == t)
    one = oracle.hils_rows(oracle.cfg(1, 2, 2, 16, 8, 3, 4, 1), qr[sel], rb[sel], rh[sel], rp[sel],
                           p.A, p.B, p.pages, p.block_table, p.landmarks)
    np.testing.assert_array_equal(one["out"], res["out"][sel])


def test_scores_rows_agree_with_selected_scores():
    p = random_problem(head_dim=16, chunk_size=8, top_k=3, seq_len=80, seed=9)
    qr, rb, rh, rp = p.rows()
    from problem import ocfg
    s = oracle.scores_rows(ocfg(p), qr, rb, rh, rp, p.A, p.B, p.landmarks, p.max_chunks, p.max_chunks)
    res = run_oracle(p)
    for r in range(len(rb)):
        own = rp[r] // 8
        assert np.isinf(s[r, own + 1:]).all() and np.isfinite(s[r, :own + 1]).all()
        for a, j in enumerate(res["idx"][r]):
            if j >= 0:
                assert s[r, j] == res["sel_scores"][r, a]
    idx, w, _ = oracle.topk_rows(s, rp, 8, 3)
    np.testing.assert_array_equal(idx, res["idx"])
