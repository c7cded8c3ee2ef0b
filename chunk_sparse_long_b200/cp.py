"""Context-parallel decode step: one sequence's chunks spread over the ranks of
a torch.distributed group, one GPU per rank (the C entry points are the
hils_decode_cp_* calls of include/hils.h).

Rank r holds the chunks chunk_base .. chunk_base + shard.max_chunks - 1 of
every sequence in a cache of its own; shard.seq_lens holds the global token
counts on every rank.  A step crosses GPUs twice: an all-gather of each
rank's best k-1 selection keys and own-chunk score (k 64-bit keys and one
float per head), and an all-reduce (sum) of each rank's weighted outputs (d
floats per head).  Everything else runs in the library's kernels; this module
only owns the small exchange buffers and the shard's workspace and calls the
collectives, on the current stream.
"""
from __future__ import annotations

from . import hils


class LibraryKernels:
    """The library's context-parallel calls (the default kernel layer)."""

    candidates = staticmethod(hils.decode_cp_candidates)
    select = staticmethod(hils.decode_cp_select)
    attend = staticmethod(hils.decode_cp_attend)
    finish = staticmethod(hils.decode_cp_finish)


def _world(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group)
    return 1


def _gather(t, out, group):
    """All-gather of t over the group into out [world][...], in rank order."""
    import torch.distributed as dist
    if out.shape[0] == 1:
        out[0].copy_(t)
        return out
    dist.all_gather_into_tensor(out.view(-1, *t.shape[1:]), t.contiguous(), group=group)
    return out


class Decoder:
    """One rank's side of the context-parallel decode of a batch.

    cfg       hils.HilsConfig of the whole problem
    shard     hils.Cache of this rank's chunks (max_chunks = chunks held)
    chunk_base  global index of the shard's first chunk
    The workspace and the exchange buffers are allocated once, here, so that
    steps can be repeated (or captured) without allocation."""

    def __init__(self, cfg, shard, chunk_base: int, *, group=None, kernels=None, device=None):
        import torch
        self.cfg, self.shard, self.chunk_base, self.group = cfg, shard, int(chunk_base), group
        self.kern = kernels or LibraryKernels
        self.world = _world(group)
        Bn, Hq, d, k = cfg.batch, cfg.n_q_heads, cfg.head_dim, cfg.top_k
        K = max(k - 1, 1)
        dev = torch.device(device) if device is not None else (
            torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu"))
        self.keys = torch.zeros((Bn, Hq, K), dtype=torch.int64, device=dev)   # 64-bit keys
        self.own = torch.empty((Bn, Hq), dtype=torch.float32, device=dev)
        self.all_keys = torch.zeros((self.world, Bn, Hq, K), dtype=torch.int64, device=dev)
        self.all_own = torch.empty((self.world, Bn, Hq), dtype=torch.float32, device=dev)
        self.idx = torch.empty((Bn, Hq, k), dtype=torch.int32, device=dev)
        self.w = torch.empty((Bn, Hq, k), dtype=torch.float32, device=dev)
        self.partial = torch.empty((Bn, Hq, d), dtype=torch.float32, device=dev)
        if self.kern is LibraryKernels:
            self.ws_bytes = hils.workspace_size(cfg, hils.OP_DECODE, 1, shard.max_chunks)
        else:
            self.ws_bytes = 256
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)   # zeroed once

    def step(self, q, k_new, v_new, A, B, out):
        """One decode step of every sequence, on the current stream (the one
        the collectives use).  q [B][Hq][d] and, when appending, k_new and
        v_new [B][Hkv][d] are the same on every rank; out [B][Hq][d] receives
        the step's output on every rank.  Returns (idx, w), the global
        selection [B][Hq][k] (chunk indices and fusion weights), buffers that
        the next step overwrites."""
        import torch.distributed as dist
        kern, cfg = self.kern, self.cfg
        stream = None
        append = k_new is not None
        kern.candidates(cfg, q, k_new, v_new, A, B, self.shard, self.chunk_base, self.keys,
                        self.own, self.ws, self.ws_bytes, stream)
        _gather(self.keys, self.all_keys, self.group)
        _gather(self.own, self.all_own, self.group)
        kern.select(cfg, self.world, self.all_keys, self.all_own, self.shard.seq_lens, append,
                    self.idx, self.w, stream)
        kern.attend(cfg, q, k_new, v_new, self.shard, self.chunk_base, self.idx, self.w,
                    self.partial, stream)
        if self.world > 1:
            dist.all_reduce(self.partial, group=self.group)
        kern.finish(cfg, self.partial, out, self.shard.seq_lens, append, stream)
        return self.idx, self.w
