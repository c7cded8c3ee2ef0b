"""Small synthetic HiLS problems for the tests (host side, numpy).

Builds the paged chunk-granular cache from logical K/V arrays and draws
seeded inputs from ``hils_inputs``.  Data movement only: no attention
arithmetic lives here.
"""
from __future__ import annotations

import dataclasses

import numpy as np

import hils_inputs as hi


@dataclasses.dataclass
class Problem:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk_size: int
    top_k: int
    calib_rank: int
    dtype: int
    seq_len: int            # tokens in the cache
    q: np.ndarray           # [B][Lq][Hq][d] storage form
    q_pos0: int
    A: np.ndarray           # [d][r] float32
    B: np.ndarray           # [r][d] float32
    K: np.ndarray           # [B][T][Hkv][d] storage form (logical order)
    V: np.ndarray
    landmarks: np.ndarray   # [B][max_chunks][Hkv][d] storage form
    pages: np.ndarray       # [n_pages][2][Hkv][S][d]
    block_table: np.ndarray # [B][max_chunks] int32

    @property
    def q_len(self):
        return self.q.shape[1]

    @property
    def max_chunks(self):
        return self.block_table.shape[1]

    def rows(self):
        """All query rows as (q_rows, row_b, row_h, row_pos), in [B][Lq][Hq] order."""
        Bn, Lq, H, d = self.q.shape
        b, i, h = np.meshgrid(np.arange(Bn), np.arange(Lq), np.arange(H), indexing="ij")
        return (self.q.reshape(-1, d), b.reshape(-1).astype(np.int32),
                h.reshape(-1).astype(np.int32), (i.reshape(-1) + self.q_pos0).astype(np.int64))


def paged_from_logical(K, V, S, max_chunks, perm=None, spare_pages=0):
    """Lay logical K/V [B][T][Hkv][d] out as pages [P][2][Hkv][S][d] and a block
    table [B][max_chunks]; ``perm`` maps logical page order to physical ids."""
    Bn, T, Hkv, d = K.shape
    n_pages = Bn * max_chunks + spare_pages
    if perm is None:
        perm = np.arange(n_pages, dtype=np.int32)
    pages = np.zeros((n_pages, 2, Hkv, S, d), dtype=K.dtype)
    bt = np.zeros((Bn, max_chunks), dtype=np.int32)
    for b in range(Bn):
        for j in range(max_chunks):
            p = int(perm[b * max_chunks + j])
            bt[b, j] = p
            t0, t1 = j * S, min((j + 1) * S, T)
            if t1 > t0:
                pages[p, 0, :, : t1 - t0, :] = K[b, t0:t1].transpose(1, 0, 2)
                pages[p, 1, :, : t1 - t0, :] = V[b, t0:t1].transpose(1, 0, 2)
    return pages, bt


def random_problem(batch=1, n_q_heads=2, n_kv_heads=2, head_dim=16, chunk_size=8, top_k=3,
                   calib_rank=4, seq_len=64, q_len=None, q_pos0=0, dtype=hi.DT_F32, seed=0,
                   calib_std=0.02, permute_pages=True, spare_pages=0):
    """Seeded N(0,1) problem.  The cache holds ``seq_len`` tokens; queries are
    the ``q_len`` positions starting at ``q_pos0`` (default: all of them)."""
    if q_len is None:
        q_len = seq_len - q_pos0
    S, d = chunk_size, head_dim
    max_chunks = (seq_len + S - 1) // S
    n = lambda tid, shape, std=1.0: hi.normal(seed, tid, 0, int(np.prod(shape)), std,
                                              dtype).reshape(shape)
    q = n(hi.TID_Q, (batch, q_len, n_q_heads, d))
    kv = n(hi.TID_PAGES, (2, batch, seq_len, n_kv_heads, d))
    lm = n(hi.TID_LM, (batch, max_chunks, n_kv_heads, d))
    A = hi.normal(seed, hi.TID_A, 0, d * calib_rank, calib_std, hi.DT_F32).reshape(d, calib_rank)
    Bm = hi.normal(seed, hi.TID_B, 0, calib_rank * d, calib_std, hi.DT_F32).reshape(calib_rank, d)
    perm = hi.page_permutation(seed, batch * max_chunks + spare_pages) if permute_pages else None
    pages, bt = paged_from_logical(kv[0], kv[1], S, max_chunks, perm, spare_pages)
    return Problem(batch, n_q_heads, n_kv_heads, d, S, top_k, calib_rank, dtype, seq_len, q, q_pos0,
                   A, Bm, kv[0], kv[1], lm, pages, bt)


def to_f64(a, dtype):
    """Storage form (float32 array or bf16 bits) to float64."""
    if dtype == hi.DT_F32:
        return np.asarray(a, dtype=np.float64)
    return hi.bf16_bits_to_f32(a).astype(np.float64)


def ocfg(p: Problem, **over):
    from oracle import oracle
    f = dict(batch=p.batch, n_q_heads=p.n_q_heads, n_kv_heads=p.n_kv_heads, head_dim=p.head_dim,
             chunk_size=p.chunk_size, top_k=p.top_k, calib_rank=p.calib_rank, dtype=p.dtype)
    f.update(over)
    return oracle.cfg(**f)


def run_oracle(p: Problem, forced_idx=None, **over):
    from oracle import oracle
    qr, rb, rh, rp = p.rows()
    return oracle.hils_rows(ocfg(p, **over), qr, rb, rh, rp, p.A, p.B, p.pages, p.block_table,
                            p.landmarks, forced_idx)
