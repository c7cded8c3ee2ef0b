"""The C-ABI library loads, exports every function include/hils.h declares, and
rejects bad arguments on the host before launching anything (no GPU needed:
every call here returns during validation)."""
import ctypes
import os
import re

import pytest

from chunk_sparse_long_b200 import build as build_mod
from chunk_sparse_long_b200 import hils

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hils.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return hils.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("hils_score", "hils_topk", "hils_prefill", "hils_decode", "hils_workspace_size",
              "hils_last_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in hils.h but not exported"
    assert set(hils.EXPORTED) >= set(declared_functions())


def test_exports_are_c_symbols():
    out = os.popen(f"nm -D --defined-only {hils.LIB_PATH}").read()
    for n in declared_functions():
        assert re.search(rf"\bT {n}$", out, re.M), f"{n} is not an unmangled text symbol"


def cfg(**over):
    f = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=64, chunk_size=64, top_k=4,
             calib_rank=8, dtype=hils.HILS_BF16)
    f.update(over)
    return hils.HilsConfig(**f)


FAKE = 1 << 20        # an aligned non-null pointer value; never dereferenced here


def cache(**over):
    f = dict(pages=FAKE, num_pages=8, block_table=FAKE, max_chunks=8, landmarks=FAKE, seq_lens=FAKE)
    f.update(over)
    return hils.Cache(**f)


def status_of(fn, *a):
    with pytest.raises(hils.HilsError) as e:
        fn(*a)
    return e.value.status, str(e.value)


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=96), 2), (dict(chunk_size=32), 2), (dict(top_k=0), 1), (dict(top_k=33), 1),
    (dict(n_q_heads=3), 1), (dict(calib_rank=65), 1), (dict(dtype=7), 1), (dict(n_kv_heads=0), 1),
])
def test_bad_config_is_rejected(lib, over, status):
    st, msg = status_of(hils.prefill, cfg(**over), FAKE, 64, 0, FAKE, FAKE, cache(), FAKE, None,
                        None, FAKE, 1 << 30, 0)
    assert st == status, msg


def test_prefill_argument_checks(lib):
    c = cfg()
    ws = hils.workspace_size(c, hils.OP_PREFILL, 128, 8)
    assert ws > 0
    assert status_of(hils.prefill, c, None, 128, 0, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)[0] == 1
    assert status_of(hils.prefill, c, FAKE + 4, 128, 0, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)[0] == 1
    assert status_of(hils.prefill, c, FAKE, 128, 0, None, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)[0] == 1
    # the last query's chunk must be inside the block table
    assert status_of(hils.prefill, c, FAKE, 8 * 64 + 1, 0, FAKE, FAKE, cache(), FAKE, None, None, FAKE, 1 << 40, 0)[0] == 1
    st, msg = status_of(hils.prefill, c, FAKE, 128, 0, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws - 1, 0)
    assert st == 3 and "workspace" in msg
    assert status_of(hils.prefill, c, FAKE, 128, 0, FAKE, FAKE, cache(), FAKE, None, None, FAKE + 16, ws, 0)[0] == 1
    assert status_of(hils.prefill, c, FAKE, 128, 0, FAKE, FAKE, cache(pages=None), FAKE, None, None, FAKE, ws, 0)[0] == 1
    assert status_of(hils.prefill, c, FAKE, 128, 0, FAKE, FAKE, cache(num_pages=0), FAKE, None, None, FAKE, ws, 0)[0] == 1


def test_decode_argument_checks(lib):
    c = cfg()
    ws = hils.workspace_size(c, hils.OP_DECODE, 1, 8)
    assert ws > 0
    assert status_of(hils.decode, c, FAKE, FAKE, None, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)[0] == 1
    assert status_of(hils.decode, c, FAKE, None, None, FAKE, FAKE, cache(seq_lens=None), FAKE, None, None, FAKE, ws, 0)[0] == 1
    assert status_of(hils.decode, c, FAKE, None, None, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws - 1, 0)[0] == 3
    assert status_of(hils.decode, cfg(n_q_heads=128, n_kv_heads=2), FAKE, None, None, FAKE, FAKE, cache(), FAKE, None, None, FAKE, 1 << 30, 0)[0] == 2
    # the calibration matrices are read in 16-byte units
    st, msg = status_of(hils.decode, c, FAKE, None, None, FAKE + 4, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)
    assert st == 1 and "aligned" in msg
    # and so are the appended token's k and v
    st, msg = status_of(hils.decode, c, FAKE, FAKE + 4, FAKE, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)
    assert st == 1 and "aligned" in msg
    st, msg = status_of(hils.decode, c, FAKE, FAKE, FAKE + 8, FAKE, FAKE, cache(), FAKE, None, None, FAKE, ws, 0)
    assert st == 1 and "aligned" in msg


def test_score_and_topk_argument_checks(lib):
    c = cfg()
    assert status_of(hils.score, c, FAKE, 64, 0, FAKE, FAKE, cache(), None, 8, 0)[0] == 1
    assert status_of(hils.score, c, FAKE, 64, 0, FAKE, FAKE, cache(), FAKE, 9, 0)[0] == 1
    assert status_of(hils.score, c, FAKE, 65, 0, FAKE, FAKE, cache(), FAKE, 1, 0)[0] == 1
    assert status_of(hils.topk, c, FAKE, 64, 64, 1, FAKE, FAKE, 0)[0] == 1
    assert status_of(hils.topk, c, None, 64, 0, 1, FAKE, FAKE, 0)[0] == 1


def test_workspace_size_rejects_bad_op(lib):
    assert hils.workspace_size(cfg(), 9, 10, 10) == 0
    assert b"unknown op" in lib.hils_last_error()


def test_prefill_backward_argument_checks(lib):
    c = cfg(head_dim=128)
    ws = hils.workspace_size(c, hils.OP_PREFILL_BACKWARD, 128, 8)
    assert ws > 0

    def call(**over):
        a = dict(q=FAKE, q_len=128, q_pos0=0, A=FAKE, B=FAKE, cache=cache(), idx=FAKE, w=FAKE,
                 out=FAKE, dout=FAKE, dq=FAKE, dpages=FAKE, dlm=FAKE, dA=FAKE, dB=FAKE, ws=FAKE,
                 ws_bytes=ws)
        a.update(over)
        return status_of(hils.prefill_backward, c if "c" not in over else over.pop("c"),
                         *[a[k] for k in ("q", "q_len", "q_pos0", "A", "B", "cache", "idx", "w",
                                          "out", "dout", "dq", "dpages", "dlm", "dA", "dB", "ws",
                                          "ws_bytes")], 0)

    assert call(idx=None)[0] == 1
    assert call(w=None)[0] == 1
    st, msg = call(out=None)
    assert st == 1 and "out" in msg
    assert call(out=FAKE + 8)[0] == 1
    assert call(dout=FAKE + 2)[0] == 1
    st, msg = call(dq=FAKE + 4)
    assert st == 1 and "dq" in msg
    assert call(dpages=None)[0] == 1
    assert call(dlm=None)[0] == 1
    st, msg = call(dA=None)
    assert st == 1 and "calib_rank" in msg
    st, msg = call(ws_bytes=ws - 1)
    assert st == 3 and "workspace" in msg
    assert call(ws=FAKE + 16)[0] == 1
    # the last query's chunk must be inside the block table
    assert call(q_len=8 * 64 + 1, ws_bytes=1 << 40)[0] == 1


def test_backward_workspace_depends_on_the_path(lib):
    # bf16 at head_dim 128 keeps per-row and per-chunk sums; the CUDA-core
    # path keeps one float per (row, slot) pair instead
    tc = hils.workspace_size(cfg(head_dim=128), hils.OP_PREFILL_BACKWARD, 4096, 64)
    simt = hils.workspace_size(cfg(head_dim=128, dtype=hils.HILS_F32), hils.OP_PREFILL_BACKWARD,
                               4096, 64)
    assert tc > 0 and simt > 0 and tc != simt
    # both grow with the query block
    assert hils.workspace_size(cfg(head_dim=128), hils.OP_PREFILL_BACKWARD, 8192, 64) > tc


def test_context_parallel_argument_checks(lib):
    c = cfg()
    ws = hils.workspace_size(c, hils.OP_DECODE, 1, 8)
    cand = hils.decode_cp_candidates
    assert status_of(cand, c, FAKE, None, None, FAKE, FAKE, cache(seq_lens=None), 0, FAKE, FAKE,
                     FAKE, ws, 0)[0] == 1
    assert status_of(cand, c, FAKE, None, None, FAKE, FAKE, cache(), -1, FAKE, FAKE, FAKE, ws,
                     0)[0] == 1
    assert status_of(cand, c, FAKE, None, None, FAKE, FAKE, cache(), 0, None, FAKE, FAKE, ws,
                     0)[0] == 1
    assert status_of(cand, c, FAKE, FAKE, None, FAKE, FAKE, cache(), 0, FAKE, FAKE, FAKE, ws,
                     0)[0] == 1
    st, msg = status_of(cand, c, FAKE, None, None, FAKE, FAKE, cache(), 0, FAKE, FAKE, FAKE,
                        ws - 1, 0)
    assert st == 3 and "workspace" in msg
    assert status_of(hils.decode_cp_select, c, 0, FAKE, FAKE, FAKE, True, FAKE, FAKE, 0)[0] == 1
    assert status_of(hils.decode_cp_select, c, 2, FAKE, FAKE, None, True, FAKE, FAKE, 0)[0] == 1
    assert status_of(hils.decode_cp_attend, c, FAKE, None, None, cache(), 0, FAKE, FAKE, None,
                     0)[0] == 1
    assert status_of(hils.decode_cp_attend, c, FAKE, None, None, cache(), -3, FAKE, FAKE, FAKE,
                     0)[0] == 1
    assert status_of(hils.decode_cp_finish, c, FAKE, FAKE, None, True, 0)[0] == 1
    assert status_of(hils.decode_cp_finish, c, None, FAKE, FAKE, False, 0)[0] == 1
