"""Python binding of libhils.so (the HiLS C ABI declared in include/hils.h).

Argument marshalling only: every step of the forward runs in the CUDA
library.  Tensors are torch CUDA tensors (torch is used for device memory and
streams); each function passes their device pointers and sizes to the
C entry point of the same name and raises ``HilsError`` on a non-zero status.
If the library has not been built this module fails loudly at load time --
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhils.so")

HILS_F32, HILS_BF16 = 0, 1
OP_SCORE, OP_TOPK, OP_PREFILL, OP_DECODE, OP_PREFILL_BACKWARD = 0, 1, 2, 3, 4
STATUS = {0: "HILS_OK", 1: "HILS_ERR_INVALID_ARG", 2: "HILS_ERR_UNSUPPORTED",
          3: "HILS_ERR_WORKSPACE", 4: "HILS_ERR_CUDA", 5: "HILS_ERR_TIMEOUT",
          6: "HILS_ERR_DEVICE_CHECK"}

EXPORTED = ("hils_workspace_size", "hils_score", "hils_topk", "hils_prefill", "hils_decode",
            "hils_device_status", "hils_last_error", "hils_version", "hils_profile_enable",
            "hils_profile_collect", "hils_profile_read", "hils_profile_reset",
            "hils_decode_noalloc", "hils_decode_noalloc_capacity", "hils_set_wait_limit_ns",
            "hils_decode_cp_candidates", "hils_decode_cp_select", "hils_decode_cp_attend",
            "hils_decode_cp_finish", "hils_prefill_backward")


class HilsError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("chunk_size", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("calib_rank", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class KVCache(ctypes.Structure):
    _fields_ = [("pages", ctypes.c_void_p), ("num_pages", ctypes.c_int64),
                ("block_table", ctypes.c_void_p), ("max_chunks", ctypes.c_int32),
                ("landmarks", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libhils.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m chunk_sparse_long_b200.build`"
                           " (there is no fallback implementation)")
    L = ctypes.CDLL(path)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    cfgp, cachep = ctypes.POINTER(Config), ctypes.POINTER(KVCache)
    L.hils_workspace_size.restype = ctypes.c_size_t
    L.hils_workspace_size.argtypes = [cfgp, ctypes.c_int, I64, I32]
    L.hils_score.restype = ctypes.c_int
    L.hils_score.argtypes = [cfgp, P, I64, I64, P, P, cachep, P, I32, P]
    L.hils_topk.restype = ctypes.c_int
    L.hils_topk.argtypes = [cfgp, P, I64, I64, I32, P, P, P]
    L.hils_prefill.restype = ctypes.c_int
    L.hils_prefill.argtypes = [cfgp, P, I64, I64, P, P, cachep, P, P, P, P, ctypes.c_size_t, P]
    L.hils_prefill_backward.restype = ctypes.c_int
    L.hils_prefill_backward.argtypes = [cfgp, P, I64, I64, P, P, cachep, P, P, P, P, P, P, P, P,
                                        P, P, ctypes.c_size_t, P]
    L.hils_decode.restype = ctypes.c_int
    L.hils_decode.argtypes = [cfgp, P, P, P, P, P, cachep, P, P, P, P, ctypes.c_size_t, P]
    L.hils_device_status.restype = ctypes.c_int
    L.hils_device_status.argtypes = [P]
    L.hils_last_error.restype = ctypes.c_char_p
    L.hils_last_error.argtypes = []
    L.hils_version.restype = ctypes.c_char_p
    L.hils_version.argtypes = []
    L.hils_profile_enable.restype = ctypes.c_int
    L.hils_profile_enable.argtypes = [ctypes.c_int]
    L.hils_profile_collect.restype = ctypes.c_int
    L.hils_profile_collect.argtypes = []
    L.hils_profile_read.restype = ctypes.c_int
    L.hils_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                                    ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_longlong)]
    L.hils_profile_reset.restype = ctypes.c_int
    L.hils_profile_reset.argtypes = []
    L.hils_decode_noalloc.restype = ctypes.c_int
    L.hils_decode_noalloc.argtypes = [cfgp, P, P, P, P, P, cachep, P, P, P, P]
    L.hils_decode_noalloc_capacity.restype = ctypes.c_size_t
    L.hils_decode_noalloc_capacity.argtypes = []
    L.hils_set_wait_limit_ns.restype = ctypes.c_int
    L.hils_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.hils_decode_cp_candidates.restype = ctypes.c_int
    L.hils_decode_cp_candidates.argtypes = [cfgp, P, P, P, P, P, cachep, I64, P, P, P,
                                            ctypes.c_size_t, P]
    L.hils_decode_cp_select.restype = ctypes.c_int
    L.hils_decode_cp_select.argtypes = [cfgp, I32, P, P, P, I32, P, P, P]
    L.hils_decode_cp_attend.restype = ctypes.c_int
    L.hils_decode_cp_attend.argtypes = [cfgp, P, P, P, cachep, I64, P, P, P, P]
    L.hils_decode_cp_finish.restype = ctypes.c_int
    L.hils_decode_cp_finish.argtypes = [cfgp, P, P, P, I32, P]
    _lib = L
    return L


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        raise HilsError(rc, where, load().hils_last_error().decode())


@dataclasses.dataclass
class HilsConfig:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk_size: int
    top_k: int
    calib_rank: int
    dtype: int

    def c(self) -> Config:
        return Config(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim,
                      self.chunk_size, self.top_k, self.calib_rank, self.dtype)


@dataclasses.dataclass
class Cache:
    """The paged cache: torch CUDA tensors (or raw device pointers)."""
    pages: object               # [num_pages][2][Hkv][S][d]
    num_pages: int
    block_table: object         # int32 [B][max_chunks]
    max_chunks: int
    landmarks: object           # [B][max_chunks][Hkv][d]
    seq_lens: object = None     # int32 [B]

    def c(self) -> KVCache:
        return KVCache(_ptr(self.pages), self.num_pages, _ptr(self.block_table), self.max_chunks,
                       _ptr(self.landmarks), _ptr(self.seq_lens))


def version() -> str:
    return load().hils_version().decode()


def workspace_size(cfg: HilsConfig, op: int, q_len: int, max_chunks: int) -> int:
    return int(load().hils_workspace_size(ctypes.byref(cfg.c()), op, q_len, max_chunks))


def score(cfg, q, q_len, q_pos0, A, B, cache: Cache, scores, n_cols, stream=None):
    _check(load().hils_score(ctypes.byref(cfg.c()), _ptr(q), q_len, q_pos0, _ptr(A), _ptr(B),
                             ctypes.byref(cache.c()), _ptr(scores), n_cols, _stream(stream)),
           "hils_score")


def topk(cfg, scores, q_len, q_pos0, n_cols, idx, w, stream=None):
    _check(load().hils_topk(ctypes.byref(cfg.c()), _ptr(scores), q_len, q_pos0, n_cols, _ptr(idx),
                            _ptr(w), _stream(stream)), "hils_topk")


def prefill(cfg, q, q_len, q_pos0, A, B, cache: Cache, out, idx_out, w_out, ws, ws_bytes,
            stream=None):
    _check(load().hils_prefill(ctypes.byref(cfg.c()), _ptr(q), q_len, q_pos0, _ptr(A), _ptr(B),
                               ctypes.byref(cache.c()), _ptr(out), _ptr(idx_out), _ptr(w_out),
                               _ptr(ws), ws_bytes, _stream(stream)), "hils_prefill")


def prefill_backward(cfg, q, q_len, q_pos0, A, B, cache: Cache, idx, w, out, dout, dq, dpages,
                     dlm, dA, dB, ws, ws_bytes, stream=None):
    """Gradients of sum(dout * out) of hils_prefill (its output `out`, its
    selection idx and w held fixed); dq, dpages, dlm, dA and dB are float32
    and added into."""
    _check(load().hils_prefill_backward(ctypes.byref(cfg.c()), _ptr(q), q_len, q_pos0, _ptr(A),
                                        _ptr(B), ctypes.byref(cache.c()), _ptr(idx), _ptr(w),
                                        _ptr(out), _ptr(dout), _ptr(dq), _ptr(dpages), _ptr(dlm),
                                        _ptr(dA), _ptr(dB), _ptr(ws), ws_bytes, _stream(stream)),
           "hils_prefill_backward")


def decode(cfg, q, k_new, v_new, A, B, cache: Cache, out, idx_out, w_out, ws, ws_bytes,
           stream=None):
    _check(load().hils_decode(ctypes.byref(cfg.c()), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(A),
                              _ptr(B), ctypes.byref(cache.c()), _ptr(out), _ptr(idx_out),
                              _ptr(w_out), _ptr(ws), ws_bytes, _stream(stream)), "hils_decode")


def decode_noalloc(cfg, q, k_new, v_new, A, B, cache: Cache, out, idx_out, w_out, stream=None):
    """hils_decode for callers that cannot allocate: scratch is the library's
    built-in array (see include/hils.h); calls on one device must not overlap."""
    _check(load().hils_decode_noalloc(ctypes.byref(cfg.c()), _ptr(q), _ptr(k_new), _ptr(v_new),
                                      _ptr(A), _ptr(B), ctypes.byref(cache.c()), _ptr(out),
                                      _ptr(idx_out), _ptr(w_out), _stream(stream)),
           "hils_decode_noalloc")


def decode_cp_candidates(cfg, q, k_new, v_new, A, B, shard: Cache, chunk_base, keys, own_score,
                         ws, ws_bytes, stream=None):
    """Context-parallel decode, step 1 (include/hils.h): this shard's best k-1
    selection keys (int64 tensor holding the 64-bit keys) and own-chunk score;
    ws is the shard's zeroed decode workspace."""
    _check(load().hils_decode_cp_candidates(ctypes.byref(cfg.c()), _ptr(q), _ptr(k_new),
                                            _ptr(v_new), _ptr(A), _ptr(B),
                                            ctypes.byref(shard.c()), chunk_base, _ptr(keys),
                                            _ptr(own_score), _ptr(ws), ws_bytes, _stream(stream)),
           "hils_decode_cp_candidates")


def decode_cp_select(cfg, world, keys, own_scores, seq_lens, append, idx, w, stream=None):
    """Context-parallel decode, step 3: the selection from the gathered lists."""
    _check(load().hils_decode_cp_select(ctypes.byref(cfg.c()), world, _ptr(keys), _ptr(own_scores),
                                        _ptr(seq_lens), int(bool(append)), _ptr(idx), _ptr(w),
                                        _stream(stream)), "hils_decode_cp_select")


def decode_cp_attend(cfg, q, k_new, v_new, shard: Cache, chunk_base, idx, w, partial,
                     stream=None):
    """Context-parallel decode, step 4: this shard's weighted outputs (float32)."""
    _check(load().hils_decode_cp_attend(ctypes.byref(cfg.c()), _ptr(q), _ptr(k_new), _ptr(v_new),
                                        ctypes.byref(shard.c()), chunk_base, _ptr(idx), _ptr(w),
                                        _ptr(partial), _stream(stream)), "hils_decode_cp_attend")


def decode_cp_finish(cfg, total, out, seq_lens, append, stream=None):
    """Context-parallel decode, step 6: the output from the summed partials."""
    _check(load().hils_decode_cp_finish(ctypes.byref(cfg.c()), _ptr(total), _ptr(out),
                                        _ptr(seq_lens), int(bool(append)), _stream(stream)),
           "hils_decode_cp_finish")


def decode_noalloc_capacity() -> int:
    return int(load().hils_decode_noalloc_capacity())


def set_wait_limit_ns(ns: int) -> None:
    """Testing hook: kernels give up on a pipeline wait after ``ns`` nanoseconds
    (0 restores the default) and report HILS_ERR_TIMEOUT."""
    _check(load().hils_set_wait_limit_ns(int(ns)), "hils_set_wait_limit_ns")


def device_status(stream=None):
    _check(load().hils_device_status(_stream(stream)), "hils_device_status")


def profile_enable(on: bool = True):
    _check(load().hils_profile_enable(1 if on else 0), "hils_profile_enable")


def profile_reset():
    _check(load().hils_profile_reset(), "hils_profile_reset")


def profile_read() -> dict:
    """{phase: (total_ms, launches)} of the kernels timed since the last reset."""
    L = load()
    _check(L.hils_profile_collect(), "hils_profile_collect")
    out = {}
    i = 0
    name = ctypes.c_char_p()
    ms = ctypes.c_double()
    n = ctypes.c_longlong()
    while L.hils_profile_read(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(n)) == 0:
        out[name.value.decode()] = (ms.value, n.value)
        i += 1
    return out
