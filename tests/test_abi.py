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
