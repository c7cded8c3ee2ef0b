"""HiLS attention backward with the selection held fixed: CPU oracle.
TEST INFRASTRUCTURE ONLY.

Only the tests (and nothing in the product path) use this module.  It is the
plain float64 definition of the gradients of the forward that the C oracle in
hils_oracle.c computes, with the chunk selection taken as given: the pages
describe training end to end under the language-modelling loss, with the
retrieval scores inside the forward pass so that gradients reach them (the
ai-feeds.com digest, sections "关键模块" item 1, the scores are fully
differentiable, and "输出与训练"; the chatpaper abstract, chunk selection
learned end to end).  Which chunks are selected is a discrete choice and has
no gradient; the fusion weights, the per-chunk attention and the calibration
do.

Forward, for query row (b, i, h) at position t = q_pos0 + i, KV head
g = h // (Hq / Hkv), chunk size S, selection idx[b, i, h] (-1 pads):
    q~ = q + (q A) B
    s_j = q~ . lm[b, j, g] / sqrt(d)               for each selected chunk j
    w = softmax over the selected s_j
    P_j = softmax over keys u of chunk j with u <= t of q . K[b, u, g] / sqrt(d)
    O_j = sum_u P_j[u] V[b, u, g]
    out = sum_j w_j O_j
Backward of the scalar sum(dout * out), in the same notation:
    dw_j  = dout . O_j
    ds_j  = w_j (dw_j - sum_l w_l dw_l)            (softmax derivative)
    dq~   = sum_j ds_j lm_j / sqrt(d),    dlm_j += ds_j q~ / sqrt(d)
    per chunk, with G = w_j dout:
      dV[u] += P_j[u] G,   dP[u] = G . V[u],   dS[u] = P_j[u] (dP[u] - G . O_j)
      dq += sum_u dS[u] K[u] / sqrt(d),   dK[u] += dS[u] q / sqrt(d)
    calibration (q~ = q + q A B):
      dq += dq~ + (dq~ B^T) A^T,   dA += q^T (dq~ B^T),   dB += (q A)^T dq~

Arrays are logical (not paged): q [B][L][Hq][d], K and V [B][T][Hkv][d],
lm [B][C][Hkv][d], A [d][r], B [r][d], idx [B][L][Hq][k], dout like q.
Every computation is float64.  The functions are split by step so that the
mutation tests can replace one step with a plausible mistake and check that
the pins catch it.
"""
from __future__ import annotations

import numpy as np


def from_storage(a, dtype: int) -> np.ndarray:
    """Storage form (float32 values, or bf16 bit patterns as uint16) -> float64."""
    a = np.asarray(a)
    if dtype == 0:
        return a.astype(np.float64)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def calibrate(q, A, B):
    """q~ = q + (q A) B for a float64 vector q."""
    return q + (q @ A) @ B


def fusion_weights(s):
    """Softmax of the selected chunks' scores (outer softmax)."""
    e = np.exp(s - s.max())
    return e / e.sum()


def chunk_attention(q, Kc, Vc, scale):
    """One chunk's attention of query q over the visible keys Kc, Vc."""
    z = Kc @ q * scale
    p = np.exp(z - z.max())
    p /= p.sum()
    return p, p @ Vc


def fusion_backward(w, dw):
    """Gradient of the selected scores from the fusion weights' gradients."""
    return w * (dw - np.dot(w, dw))


def chunk_attention_backward(q, Kc, Vc, p, O, G, scale):
    """Gradients of one chunk's attention given G = dL/dO_j.
    Returns (dq, dKc, dVc)."""
    dVc = np.outer(p, G)
    dP = Vc @ G
    dS = p * (dP - np.dot(G, O))
    return dS @ Kc * scale, np.outer(dS, q) * scale, dVc


def calib_backward(q, A, B, dqt):
    """Gradients through q~ = q + (q A) B given dq~.  Returns (dq, dA, dB)."""
    u = B @ dqt                      # dq~ B^T, length r
    return dqt + A @ u, np.outer(q, u), np.outer(q @ A, dqt)


def _rows(q, idx):
    Bn, L, Hq, _ = q.shape
    for b in range(Bn):
        for i in range(L):
            for h in range(Hq):
                yield b, i, h, [int(j) for j in idx[b, i, h] if j >= 0]


def _visible(j, S, t):
    """Key positions of chunk j visible to a query at position t."""
    return j * S, min((j + 1) * S, t + 1)


def forward(q, q_pos0, A, B, K, V, lm, idx, chunk_size):
    """The forward with the selection given.  Returns dict(out, w) with w
    [B][L][Hq][k] (0 in padded slots)."""
    Bn, L, Hq, d = q.shape
    Hkv = K.shape[2]
    grp = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    out = np.zeros_like(q)
    wts = np.zeros(idx.shape, dtype=np.float64)
    for b, i, h, js in _rows(q, idx):
        g, t = h // grp, q_pos0 + i
        qv = q[b, i, h]
        qt = calibrate(qv, A, B)
        s = np.array([qt @ lm[b, j, g] * scale for j in js])
        w = fusion_weights(s)
        for n, j in enumerate(js):
            u0, u1 = _visible(j, chunk_size, t)
            _, O = chunk_attention(qv, K[b, u0:u1, g], V[b, u0:u1, g], scale)
            out[b, i, h] += w[n] * O
        wts[b, i, h, :len(js)] = w
    return {"out": out, "w": wts}


def backward(q, q_pos0, A, B, K, V, lm, idx, dout, chunk_size):
    """Gradients of sum(dout * out) with the selection held fixed.
    Returns dict(dq, dK, dV, dlm, dA, dB, ds) in float64; ds [B][L][Hq][k] is
    the gradient of the selected scores (0 in padded slots)."""
    Bn, L, Hq, d = q.shape
    Hkv = K.shape[2]
    grp = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    dq = np.zeros_like(q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dlm = np.zeros_like(lm)
    dA = np.zeros_like(A)
    dB = np.zeros_like(B)
    ds_all = np.zeros(idx.shape, dtype=np.float64)
    for b, i, h, js in _rows(q, idx):
        g, t = h // grp, q_pos0 + i
        qv, go = q[b, i, h], dout[b, i, h]
        qt = calibrate(qv, A, B)
        s = np.array([qt @ lm[b, j, g] * scale for j in js])
        w = fusion_weights(s)
        dw = np.zeros(len(js))
        for n, j in enumerate(js):
            u0, u1 = _visible(j, chunk_size, t)
            Kc, Vc = K[b, u0:u1, g], V[b, u0:u1, g]
            p, O = chunk_attention(qv, Kc, Vc, scale)
            dw[n] = go @ O
            dqa, dKc, dVc = chunk_attention_backward(qv, Kc, Vc, p, O, w[n] * go, scale)
            dq[b, i, h] += dqa
            dK[b, u0:u1, g] += dKc
            dV[b, u0:u1, g] += dVc
        ds = fusion_backward(w, dw)
        ds_all[b, i, h, :len(js)] = ds
        dqt = np.zeros(d)
        for n, j in enumerate(js):
            dqt += ds[n] * lm[b, j, g] * scale
            dlm[b, j, g] += ds[n] * qt * scale
        dqc, dAr, dBr = calib_backward(qv, A, B, dqt)
        dq[b, i, h] += dqc
        dA += dAr
        dB += dBr
    return {"dq": dq, "dK": dK, "dV": dV, "dlm": dlm, "dA": dA, "dB": dB, "ds": ds_all}


def logical_kv(pages, block_table, seq_len, dtype):
    """Logical K, V [B][T][Hkv][d] (float64) of a paged cache
    pages [P][2][Hkv][S][d] under block_table [B][C]."""
    pg = from_storage(pages, dtype)
    S = pg.shape[3]
    bt = np.asarray(block_table)
    Bn = bt.shape[0]
    T = seq_len
    K = np.zeros((Bn, T, pg.shape[2], pg.shape[4]))
    V = np.zeros_like(K)
    for b in range(Bn):
        for u in range(T):
            page = bt[b, u // S]
            K[b, u] = pg[page, 0, :, u % S]
            V[b, u] = pg[page, 1, :, u % S]
    return K, V
