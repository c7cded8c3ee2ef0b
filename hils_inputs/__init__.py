"""Seeded synthetic inputs for the HiLS attention forward.

This module is shared by the oracle side and the CUDA side of the tests and
the bench.  It holds only random-number generation and the shapes of the
workloads: none of the method's arithmetic lives here.

Generator (counter-based, so any element can be regenerated on its own):

* ``sm64(x)`` is one output of the splitmix64 generator (Steele, Lea and
  Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):
  add the golden-ratio increment 0x9E3779B97F4A7C15, then two
  xor-shift-multiply rounds and a final xor-shift.
* a tensor's stream key is ``sm64(sm64(seed) ^ tensor_id)``;
* element ``i`` of the tensor draws two 64-bit words
  ``a = sm64(key + 2*i*G)`` and ``b = sm64(key + (2*i+1)*G)`` (``G`` is the
  increment), takes ``u1 = ((a >> 11) + 1) * 2**-53`` in (0, 1] and
  ``u2 = (b >> 11) * 2**-53`` in [0, 1), and forms one standard normal by the
  Box-Muller transform ``sqrt(-2 ln u1) * cos(2 pi u2)`` in float64;
* the value is multiplied by ``std`` in float64 and rounded to float32 by
  round-to-nearest-even; a bf16 input is that float32 rounded once more to
  bf16 by round-to-nearest-even.

The same definition is implemented for the device in ``gen_device.cu``
(built into ``libhils_gen.so``) so that multi-gigabyte caches can be filled
on the GPU; a test checks the two bit for bit.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

# tensor ids: one independent stream per input tensor
TID_Q = 1          # prefill queries [B][L][Hq][d]
TID_LM = 2         # landmarks [B][max_chunks][Hkv][d]
TID_PAGES = 3      # paged K/V storage, by physical element index
TID_A = 4          # calibration A [d][r]
TID_B = 5          # calibration B [r][d]
TID_QDEC = 6       # decode queries [steps][B][Hq][d]
TID_KNEW = 7       # decode appended keys [steps][B][Hkv][d]
TID_VNEW = 8       # decode appended values [steps][B][Hkv][d]
TID_PERM = 9       # page permutation keys
TID_NEEDLE = 10    # needle chunk positions
TID_DOUT = 11      # output gradients of the prefill backward [B][L][Hq][d]

DT_F32 = 0
DT_BF16 = 1


def _u64(x):
    return np.asarray(x, dtype=np.uint64)


def sm64(z: np.ndarray) -> np.ndarray:
    """splitmix64 output for state ``z`` (uint64 array, wraps mod 2**64)."""
    with np.errstate(over="ignore"):
        z = _u64(z) + np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tid: int) -> int:
    k0 = int(sm64(_u64([seed]))[0])
    return int(sm64(_u64([k0 ^ tid]))[0])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even), returned as uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return (r & np.uint64(0xFFFF)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f64(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    """Standard normals (float64) of elements ``start .. start+count-1`` of a stream."""
    key = stream_key(seed, tid)
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        ca = np.uint64(key) + (np.uint64(2) * i) * np.uint64(GOLDEN)
        cb = np.uint64(key) + (np.uint64(2) * i + np.uint64(1)) * np.uint64(GOLDEN)
    a = sm64(ca)
    b = sm64(cb)
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (b >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def normal(seed: int, tid: int, start: int, count: int, std: float = 1.0,
           dtype: int = DT_BF16) -> np.ndarray:
    """Elements of a stream in storage form: float32 array, or uint16 bf16 bits."""
    v = (normal_f64(seed, tid, start, count) * float(std)).astype(np.float32)
    if dtype == DT_F32:
        return v
    return f32_to_bf16_bits(v)


def uniform_u64(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    key = stream_key(seed, tid)
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return sm64(np.uint64(key) + i * np.uint64(GOLDEN))


# ----------------------------------------------------------------------------
# device generator (same definition), used to fill large tensors on the GPU
# ----------------------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
GEN_LIB = os.path.join(_HERE, "libhils_gen.so")
_gen = None


def build_gen(force: bool = False) -> str:
    import subprocess
    src = os.path.join(_HERE, "gen_device.cu")
    if force or not os.path.exists(GEN_LIB) or os.path.getmtime(GEN_LIB) < os.path.getmtime(src):
        cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
               "-o", GEN_LIB, src]
        subprocess.check_call(cmd)
    return GEN_LIB


def _genlib():
    global _gen
    if _gen is None:
        if not os.path.exists(GEN_LIB):
            build_gen()
        _gen = ctypes.CDLL(GEN_LIB)
        _gen.hils_gen_normal.restype = ctypes.c_int
        _gen.hils_gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                         ctypes.c_uint64, ctypes.c_double, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_void_p]
    return _gen


def normal_device(out, seed: int, tid: int, start: int = 0, std: float = 1.0,
                  stream: Optional[int] = None) -> None:
    """Fill a contiguous CUDA tensor (float32 or bfloat16) with stream elements
    ``start .. start+numel-1``; bit-identical to :func:`normal`."""
    import torch
    assert out.is_cuda and out.is_contiguous()
    dt = {torch.float32: DT_F32, torch.bfloat16: DT_BF16}[out.dtype]
    if stream is None:
        stream = torch.cuda.current_stream(out.device).cuda_stream
    rc = _genlib().hils_gen_normal(seed, tid, start, out.numel(), float(std), dt,
                                   out.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"hils_gen_normal failed with CUDA error {rc}")


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and recipe of one synthetic workload."""
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk_size: int
    top_k: int
    calib_rank: int
    dtype: int           # DT_F32 or DT_BF16
    seq_len: int         # prefill length L, or decode context before step 0
    seed: int
    mode: str            # "prefill" or "decode"
    decode_steps: int = 0
    needles: int = 0     # planted needle chunks (see module functions)

    @property
    def n_chunks(self) -> int:
        return (self.seq_len + self.decode_steps + self.chunk_size - 1) // self.chunk_size


# The five workloads: tiny fp32 correctness; 345M-style prefill; GQA 128K
# prefill; 512K decode (B=1 and B=32 at 128K); 4M-token extrapolation decode.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 2, 64, 64, 4, 8, DT_F32, 1024, 0, "prefill"),
    "prefill_8k": Workload("prefill_8k", 1, 16, 16, 64, 64, 16, 16, DT_BF16, 8192, 2, "prefill"),
    "prefill_128k_gqa": Workload("prefill_128k_gqa", 1, 32, 8, 128, 64, 32, 32, DT_BF16,
                                 131072, 3, "prefill", needles=1),
    # the 128K GQA shape at 16K tokens: a profiling-size case (a few GB on the device)
    "prefill_16k_gqa": Workload("prefill_16k_gqa", 1, 32, 8, 128, 64, 32, 32, DT_BF16, 16384, 3,
                                "prefill"),
    # the 128K GQA shape at 512K tokens: a long prefill in one call (about 26 GB
    # of workspace, 43 GB on the device in all)
    "prefill_512k_gqa": Workload("prefill_512k_gqa", 1, 32, 8, 128, 64, 32, 32, DT_BF16,
                                 524288, 6, "prefill"),
    "decode_512k": Workload("decode_512k", 1, 16, 16, 64, 64, 16, 16, DT_BF16, 524288, 4,
                            "decode", decode_steps=256),
    "decode_128k_b32": Workload("decode_128k_b32", 32, 16, 16, 64, 64, 16, 16, DT_BF16, 131072,
                                4, "decode", decode_steps=256),
    "decode_4m": Workload("decode_4m", 1, 16, 16, 64, 64, 16, 16, DT_BF16, 4194304, 5,
                          "decode", decode_steps=256, needles=8),
}


def page_permutation(seed: int, n_pages: int) -> np.ndarray:
    """A seeded permutation of physical page ids (the block table's order)."""
    keys = uniform_u64(seed, TID_PERM, 0, n_pages)
    return np.argsort(keys, kind="stable").astype(np.int32)


def needle_chunks(seed: int, count: int, n_chunks: int) -> np.ndarray:
    """Seeded, distinct chunk indices in [0, n_chunks) for planted needles."""
    out = []
    j = 0
    while len(out) < count:
        u = int(uniform_u64(seed, TID_NEEDLE, j, 1)[0])
        c = int(u % n_chunks)
        if c not in out:
            out.append(c)
        j += 1
    return np.array(sorted(out), dtype=np.int64)


# ----------------------------------------------------------------------------
# full-size workloads on the device
# ----------------------------------------------------------------------------
SPARE_PAGES = 4


def device_workload(w: Workload, device="cuda", seed_offset: int = 0) -> dict:
    """Allocate and fill every input tensor of workload ``w`` on ``device``.

    Recipe (all N(0,1) unless stated; A and B are N(0, 0.02) float32):
      pages       [P][2][Hkv][S][d], P = B*max_chunks + 4 spare pages, drawn by
                  physical element index from stream TID_PAGES;
      block_table sequence b's chunk j -> page perm[b*max_chunks + j], perm a
                  seeded permutation of the page ids (TID_PERM);
      landmarks   [B][max_chunks][Hkv][d] (TID_LM);
      prefill:    q [B][L][Hq][d] (TID_Q);
      decode:     q_dec [steps][B][Hq][d] (TID_QDEC), k_new and v_new
                  [steps][B][Hkv][d] (TID_KNEW, TID_VNEW), seq_lens = context.
    Needles: a prefill workload with ``needles`` plants, per KV head g, one
    chunk (seeded) whose landmark is sqrt(d) m_g/|m_g|, m_g the mean of the
    raw queries of g's query heads over all positions; a decode workload plants
    ``needles`` chunks (seeded depths, shared by the heads) whose landmark for
    KV head g is 4 q0/|q0|, q0 the raw step-0 query of g's first query head,
    so its score is about +4 standard deviations above the N(0,1) background.
    """
    import torch
    seed = w.seed + seed_offset
    B, Hq, Hkv, d, S = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk_size
    dt = torch.bfloat16 if w.dtype == DT_BF16 else torch.float32
    max_chunks = w.n_chunks
    n_pages = B * max_chunks + SPARE_PAGES
    out = {"workload": w, "max_chunks": max_chunks, "num_pages": n_pages}
    pages = torch.empty((n_pages, 2, Hkv, S, d), dtype=dt, device=device)
    normal_device(pages, seed, TID_PAGES)
    perm = page_permutation(seed, n_pages)
    out["pages"] = pages
    out["block_table"] = torch.from_numpy(
        np.ascontiguousarray(perm[: B * max_chunks].reshape(B, max_chunks))).to(device)
    lm = torch.empty((B, max_chunks, Hkv, d), dtype=dt, device=device)
    normal_device(lm, seed, TID_LM)
    out["A"] = torch.from_numpy(normal(seed, TID_A, 0, d * w.calib_rank, 0.02, DT_F32)
                                .reshape(d, w.calib_rank)).to(device)
    out["B"] = torch.from_numpy(normal(seed, TID_B, 0, w.calib_rank * d, 0.02, DT_F32)
                                .reshape(w.calib_rank, d)).to(device)
    group = Hq // Hkv
    if w.mode == "prefill":
        q = torch.empty((B, w.seq_len, Hq, d), dtype=dt, device=device)
        normal_device(q, seed, TID_Q)
        out["q"] = q
        if w.needles:
            n_vis = (w.seq_len + S - 1) // S
            chunks = needle_chunks(seed, Hkv * w.needles, n_vis)
            m = q.view(B, w.seq_len, Hkv, group, d).sum(dim=(1, 3), dtype=torch.float64)
            for b in range(B):
                for g in range(Hkv):
                    for n in range(w.needles):
                        c = int(chunks[g * w.needles + n])
                        v = math.sqrt(d) * m[b, g] / torch.linalg.vector_norm(m[b, g])
                        lm[b, c, g] = v.float().to(dt)
            out["needle_chunks"] = chunks.reshape(Hkv, w.needles)
    else:
        steps = w.decode_steps
        qd = torch.empty((steps, B, Hq, d), dtype=dt, device=device)
        normal_device(qd, seed, TID_QDEC)
        kn = torch.empty((steps, B, Hkv, d), dtype=dt, device=device)
        vn = torch.empty((steps, B, Hkv, d), dtype=dt, device=device)
        normal_device(kn, seed, TID_KNEW)
        normal_device(vn, seed, TID_VNEW)
        out.update(q_dec=qd, k_new=kn, v_new=vn)
        out["seq_lens"] = torch.full((B,), w.seq_len, dtype=torch.int32, device=device)
        if w.needles:
            chunks = needle_chunks(seed, w.needles, w.seq_len // S)
            q0 = qd[0].double()                                    # [B][Hq][d]
            for b in range(B):
                for g in range(Hkv):
                    v = 4.0 * q0[b, g * group] / torch.linalg.vector_norm(q0[b, g * group])
                    for c in chunks:
                        lm[b, int(c), g] = v.float().to(dt)
            out["needle_chunks"] = chunks
    out["landmarks"] = lm
    return out
