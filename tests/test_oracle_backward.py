"""Pins of the backward oracle (oracle/backward.py), on the CPU.

- Its forward, given the selection, equals the C oracle's forward (the pinned
  definition of the method) on the same stored inputs.
- Every gradient equals a central finite difference of that forward: the
  selection is held fixed, so sum(dout * out) is a smooth function of q, K,
  V, the landmarks, A and B.
- One chunk that holds the whole sequence and k = 1 is ordinary causal
  attention: the gradients of q, K and V equal torch autograd through
  torch's scaled_dot_product_attention in float64, and the score path gives
  nothing (w = 1 is constant).
- The outer softmax is shift-invariant, so every row's score gradients sum
  to zero.
- A plausible mistake planted in any one step of the oracle makes the
  finite-difference pin fail."""
import numpy as np
import pytest

from oracle import backward as ob
from oracle import oracle
from problem import ocfg, random_problem
import hils_inputs as hi


def _tiny(seed=5, k=3, q_pos0=0, seq_len=24, dtype=hi.DT_F32, chunk=4, Hq=2, Hkv=1, d=4, r=2):
    p = random_problem(batch=1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, chunk_size=chunk,
                       top_k=k, calib_rank=r, seq_len=seq_len, q_pos0=q_pos0, dtype=dtype,
                       seed=seed, calib_std=0.5)
    q = ob.from_storage(p.q, dtype)
    K, V = ob.from_storage(p.K, dtype), ob.from_storage(p.V, dtype)
    lm = ob.from_storage(p.landmarks, dtype)
    A, B = p.A.astype(np.float64), p.B.astype(np.float64)
    # the selection: the C oracle's, row by row
    Bn, L, H, _ = q.shape
    rb, ri, rh = np.meshgrid(np.arange(Bn), np.arange(L), np.arange(H), indexing="ij")
    rb, ri, rh = rb.reshape(-1), ri.reshape(-1), rh.reshape(-1)
    orc = oracle.hils_rows(ocfg(p), p.q[rb, ri, rh], rb.astype(np.int32), rh.astype(np.int32),
                           (q_pos0 + ri).astype(np.int64), p.A, p.B, p.pages, p.block_table,
                           p.landmarks)
    idx = orc["idx"].reshape(Bn, L, H, k)
    dout = np.random.default_rng(seed + 100).standard_normal(q.shape)
    return dict(p=p, q=q, K=K, V=V, lm=lm, A=A, B=B, idx=idx, dout=dout, orc=orc, q_pos0=q_pos0,
                chunk=chunk)


def _loss(t, **over):
    a = dict(q=t["q"], K=t["K"], V=t["V"], lm=t["lm"], A=t["A"], B=t["B"])
    a.update(over)
    out = ob.forward(a["q"], t["q_pos0"], a["A"], a["B"], a["K"], a["V"], a["lm"], t["idx"],
                     t["chunk"])["out"]
    return float(np.sum(t["dout"] * out))


def _fd_errors(t, h=1e-5):
    """Max |finite difference - oracle gradient| per input, and the scale."""
    g = ob.backward(t["q"], t["q_pos0"], t["A"], t["B"], t["K"], t["V"], t["lm"], t["idx"],
                    t["dout"], t["chunk"])
    errs = {}
    for name, gname in (("q", "dq"), ("K", "dK"), ("V", "dV"), ("lm", "dlm"), ("A", "dA"),
                        ("B", "dB")):
        x = t[name].copy()
        fd = np.zeros_like(x)
        for e in np.ndindex(x.shape):
            x0 = x[e]
            x[e] = x0 + h
            lp = _loss(t, **{name: x})
            x[e] = x0 - h
            lm_ = _loss(t, **{name: x})
            x[e] = x0
            fd[e] = (lp - lm_) / (2 * h)
        errs[name] = float(np.max(np.abs(fd - g[gname]))), float(np.max(np.abs(fd)))
    return errs


def test_forward_with_given_selection_matches_c_oracle():
    t = _tiny(seed=7, k=3, q_pos0=5, seq_len=40, d=8, Hq=4, Hkv=2, r=3)
    f = ob.forward(t["q"], t["q_pos0"], t["A"], t["B"], t["K"], t["V"], t["lm"], t["idx"],
                   t["chunk"])
    n = f["out"].shape
    np.testing.assert_allclose(f["out"].reshape(-1, n[-1]), t["orc"]["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["w"].reshape(t["orc"]["w"].shape), t["orc"]["w"], rtol=0,
                               atol=1e-12)


@pytest.mark.parametrize("case", [dict(seed=5, k=3), dict(seed=6, k=4, q_pos0=6, seq_len=30),
                                  dict(seed=8, k=2, Hq=4, Hkv=2, dtype=hi.DT_BF16)])
def test_gradients_match_finite_differences(case):
    t = _tiny(**case)
    for name, (err, scale) in _fd_errors(t).items():
        assert scale > 1e-3, (name, scale)            # the gradient is not trivially zero
        assert err <= 1e-7 + 1e-6 * scale, (name, err, scale)


def test_one_chunk_is_causal_attention_under_torch_autograd():
    import torch
    t = _tiny(seed=9, k=1, seq_len=16, chunk=16, Hq=4, Hkv=2, d=8, r=3)
    g = ob.backward(t["q"], 0, t["A"], t["B"], t["K"], t["V"], t["lm"], t["idx"], t["dout"], 16)
    q = torch.tensor(t["q"], requires_grad=True)          # [B][L][Hq][d]
    K = torch.tensor(t["K"], requires_grad=True)          # [B][T][Hkv][d]
    V = torch.tensor(t["V"], requires_grad=True)
    grp = q.shape[2] // K.shape[2]
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), K.repeat_interleave(grp, 2).transpose(1, 2),
        V.repeat_interleave(grp, 2).transpose(1, 2), is_causal=True).transpose(1, 2)
    (out * torch.tensor(t["dout"])).sum().backward()
    np.testing.assert_allclose(g["dq"], q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dK"], K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dV"], V.grad.numpy(), rtol=0, atol=1e-12)
    for name in ("dlm", "dA", "dB", "ds"):
        assert np.abs(g[name]).max() < 1e-12, name


def test_score_gradients_of_each_row_sum_to_zero():
    t = _tiny(seed=10, k=4, seq_len=32, Hq=4, Hkv=2, d=8)
    g = ob.backward(t["q"], 0, t["A"], t["B"], t["K"], t["V"], t["lm"], t["idx"], t["dout"],
                    t["chunk"])
    assert np.abs(g["ds"].sum(axis=-1)).max() < 1e-12
    assert np.abs(g["ds"]).max() > 1e-3


# ---- planted mistakes: each must turn the finite-difference pin red ---------
def _wrong_fusion(w, dw):
    return w * dw                                             # drops the softmax's mean term


def _wrong_attention_missing_mean(q, Kc, Vc, p, O, G, scale):
    dVc = np.outer(p, G)
    dS = p * (Vc @ G)                                         # drops - G.O
    return dS @ Kc * scale, np.outer(dS, q) * scale, dVc


def _wrong_attention_dk_scale(q, Kc, Vc, p, O, G, scale):
    dVc = np.outer(p, G)
    dS = p * (Vc @ G - np.dot(G, O))
    return dS @ Kc * scale, np.outer(dS, q), dVc              # dK without 1/sqrt(d)


def _wrong_calib_identity(q, A, B, dqt):
    u = B @ dqt
    return A @ u, np.outer(q, u), np.outer(q @ A, dqt)        # drops dq~ itself


def _wrong_calib_da(q, A, B, dqt):
    u = B @ dqt
    return dqt + A @ u, np.outer(q + (q @ A) @ B, u), np.outer(q @ A, dqt)   # q~ for q in dA


def _wrong_calib_db(q, A, B, dqt):
    u = B @ dqt
    return dqt + A @ u, np.outer(q, u), np.outer(q[:A.shape[1]], dqt)   # dB without A


@pytest.mark.parametrize("fn,patch", [
    ("fusion_backward", _wrong_fusion),
    ("chunk_attention_backward", _wrong_attention_missing_mean),
    ("chunk_attention_backward", _wrong_attention_dk_scale),
    ("calib_backward", _wrong_calib_identity),
    ("calib_backward", _wrong_calib_da),
    ("calib_backward", _wrong_calib_db),
])
def test_planted_mistake_is_caught(monkeypatch, fn, patch):
    monkeypatch.setattr(ob, fn, patch)
    t = _tiny(seed=5, k=3)
    errs = _fd_errors(t)
    assert any(err > 1e-7 + 1e-6 * scale for err, scale in errs.values()), errs


def test_two_single_token_chunks_closed_form():
    """Chunks of one token, d = 1, no calibration, two positions, k = 2.
    Row 0 sees only its own chunk: out_0 = v_0, so dv_0 gets dout_0 and
    nothing else moves (a softmax over one key has no gradient).  Row 1
    fuses chunk 1 (its own) and chunk 0 with w = softmax(q_1 [lm_1, lm_0]):
    out_1 = w_1 v_1 + w_0 v_0.  By hand:
        dv_1 = w_1 dout_1,  dv_0 = dout_0 + w_0 dout_1,  dK = 0,
        ds_1 = -ds_0 = w_0 w_1 dout_1 (v_1 - v_0),
        dq_1 = ds_1 (lm_1 - lm_0),  dlm_1 = ds_1 q_1,  dlm_0 = -ds_1 q_1."""
    q = np.array([0.3, 0.5]).reshape(1, 2, 1, 1)
    K = np.array([0.7, -0.2]).reshape(1, 2, 1, 1)
    V = np.array([1.5, -0.5]).reshape(1, 2, 1, 1)
    lm = np.array([1.0, -1.0]).reshape(1, 2, 1, 1)
    A, B = np.zeros((1, 0)), np.zeros((0, 1))
    idx = np.array([[0, -1], [1, 0]]).reshape(1, 2, 1, 2)
    dout = np.array([0.25, 2.0]).reshape(1, 2, 1, 1)
    g = ob.backward(q, 0, A, B, K, V, lm, idx, dout, 1)
    e1, e0 = np.exp(0.5 * -1.0), np.exp(0.5 * 1.0)
    w1, w0 = e1 / (e1 + e0), e0 / (e1 + e0)
    ds1 = w0 * w1 * 2.0 * (-0.5 - 1.5)
    np.testing.assert_allclose(g["dV"].reshape(2), [0.25 + w0 * 2.0, w1 * 2.0], rtol=1e-14)
    np.testing.assert_allclose(g["dK"].reshape(2), [0.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(g["dq"].reshape(2), [0.0, ds1 * (-1.0 - 1.0)], atol=1e-15)
    np.testing.assert_allclose(g["dlm"].reshape(2), [-ds1 * 0.5, ds1 * 0.5], atol=1e-15)
    np.testing.assert_allclose(g["ds"].reshape(2, 2), [[0.0, 0.0], [ds1, -ds1]], atol=1e-15)
