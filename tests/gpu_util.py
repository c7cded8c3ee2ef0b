"""Helpers for the GPU parity tests: move a host Problem to the device, run the
library through the C ABI, and compare with the oracle under the selection rule.

Selection rule: chunk indices must be bit-exact wherever the oracle's score gap
at the selection boundary exceeds 1e-5.  Where it does not, or where two
selected chunks' scores are within 1e-5 of each other (so their order is not
fixed), the GPU's choice must be valid -- every chunk it picked scores at
least the oracle's last selected score minus 1e-5, in non-increasing order up
to 1e-5 -- and its output is then checked against the oracle run with the
GPU's selection forced.
"""
from __future__ import annotations

import numpy as np
import torch

import hils_inputs as hi
from chunk_sparse_long_b200 import hils
from oracle import oracle

GAP = 1e-5
TOL_OUT = {hi.DT_F32: 1e-3, hi.DT_BF16: 2e-2}
TOL_W = 1e-5


def dev(a: np.ndarray, dtype: int = None) -> torch.Tensor:
    """Storage-form numpy array (float32, or uint16 bf16 bits, or ints) -> CUDA tensor."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def host_storage(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def cfg_of(p) -> hils.HilsConfig:
    return hils.HilsConfig(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.chunk_size, p.top_k,
                           p.calib_rank, p.dtype)


class DevProblem:
    """Device copies of a tests.problem.Problem."""

    def __init__(self, p):
        self.p = p
        self.q = dev(p.q)
        self.A = dev(p.A)
        self.B = dev(p.B)
        self.pages = dev(p.pages)
        self.bt = dev(p.block_table)
        self.lm = dev(p.landmarks)
        self.seq_lens = torch.full((p.batch,), p.seq_len, dtype=torch.int32, device="cuda")
        self.cache = hils.Cache(self.pages, p.pages.shape[0], self.bt, p.max_chunks, self.lm,
                                self.seq_lens)
        self.cfg = cfg_of(p)


def run_prefill(dp: DevProblem, ws_pad: int = 0):
    p = dp.p
    rows = p.batch * p.q_len * p.n_q_heads
    out = torch.empty((p.batch, p.q_len, p.n_q_heads, p.head_dim), device="cuda",
                      dtype=torch.float32 if p.dtype == hi.DT_F32 else torch.bfloat16)
    idx = torch.empty((rows, p.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((rows, p.top_k), dtype=torch.float32, device="cuda")
    nbytes = hils.workspace_size(dp.cfg, hils.OP_PREFILL, p.q_len, p.max_chunks)
    ws = torch.empty(nbytes + ws_pad, dtype=torch.uint8, device="cuda")
    ws.fill_(0xAB)                         # the workspace needs no initialisation
    hils.prefill(dp.cfg, dp.q, p.q_len, p.q_pos0, dp.A, dp.B, dp.cache, out, idx, w, ws, ws.numel())
    hils.device_status()
    return out, idx, w


def compare(gpu_idx, gpu_w, gpu_out, orc, rerun_forced, dtype, gap=GAP, tol_out=None,
            tol_w=TOL_W):
    """Check GPU selection/weights/outputs against an oracle result for the same rows.

    rerun_forced(row_ids, forced_idx) -> oracle result dict for those rows with the
    selection forced.  Returns a small report dict."""
    tol_out = TOL_OUT[dtype] if tol_out is None else tol_out
    gi = np.asarray(gpu_idx)
    oi = orc["idx"]
    ref_out = orc["out"].copy() if orc["out"] is not None else None
    ref_w = orc["w"].copy()
    mism = np.nonzero(np.any(gi != oi, axis=1))[0]
    if len(mism):
        f = rerun_forced(mism, gi[mism])
        for n, r in enumerate(mism):
            sel_o = oi[r][oi[r] >= 0]
            sel_g = gi[r][gi[r] >= 0]
            assert len(sel_o) == len(sel_g) and sel_o[0] == sel_g[0], (r, oi[r], gi[r])
            if set(sel_o.tolist()) != set(sel_g.tolist()):
                assert orc["gap"][r] <= gap, f"row {r}: selection differs with gap {orc['gap'][r]}"
            fs = f["sel_scores"][n][1:len(sel_g)]
            last = orc["sel_scores"][r][len(sel_o) - 1] if len(sel_o) > 1 else np.inf
            assert (fs >= last - gap).all(), (r, fs, last)
            assert (np.diff(fs) <= gap).all(), (r, fs)
            ref_w[r] = f["w"][n]
            if ref_out is not None:
                ref_out[r] = f["out"][n]
    np.testing.assert_allclose(np.asarray(gpu_w), ref_w, rtol=0, atol=tol_w)
    err = None
    if ref_out is not None:
        err = float(np.max(np.abs(np.asarray(gpu_out) - ref_out))) if ref_out.size else 0.0
        assert err <= tol_out, f"max abs error {err} > {tol_out}"
    return {"mismatched_rows": int(len(mism)), "max_abs_err": err}
