"""The C-ABI library loads, exports every symbol its header declares, and rejects bad
arguments on the host (no GPU needed: none of these calls reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from compressed_sparse_attention_score_b200 import build
    build.build()
    import compressed_sparse_attention_score_b200 as pkg
    return pkg.raw()


def test_header_declares_the_boundary():
    names = declared()
    for n in ["csa2_pack_kv", "csa2_pack_swa", "csa2_index_score", "csa2_topk", "csa2_sparse_attn",
              "csa2_swa_attn", "csa2_merge", "csa2_workspace_size", "csa2_check", "csa2_last_error_string",
              "csa2_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    import compressed_sparse_attention_score_b200 as pkg
    for n in declared():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (csa2_\w+)", out))
    assert set(declared()) <= exported
    # the binding wraps every declared entry point under the same name
    assert set(declared()) <= set(pkg.EXPORTED)


def test_version(lib):
    assert lib.csa2_version() >= 100


def test_workspace_size(lib):
    ws = lib.csa2_workspace_size
    assert ws(2, 32, 1, 65536, 512, 0) == 0                           # Reuse needs none
    full = ws(0, 8, 1, 1 << 20, 512, 16384)
    assert full >= 8 * (1 << 20) * 4 + 8 * 512 * 4
    assert ws(1, 8, 1, 1 << 20, 512, 16384) == 8 * 512 * 4               # Reindex of a 16384 pool: selection only
    assert ws(1, 8, 1, 1 << 20, 512, 16385) >= 8 * 16385 * 4 + 8 * 512 * 4   # larger pools: scores too
    assert ws(0, 1024, 1, 1 << 17, 512, 0) == 1024 * 512 * 4             # prefill chunk: selection only


def test_host_side_argument_checks(lib):
    from compressed_sparse_attention_score_b200 import csa2_cache
    c = csa2_cache()
    # NULL cache / inputs are rejected before any launch
    assert lib.csa2_pack_kv(None, None, 0, None, 1, 1, None, None, None, None) == 1
    assert lib.csa2_topk(None, None, 1, 10, 5, None, None, 0, None, None, None) == 1
    assert lib.csa2_merge(None, None, None, None, 1, 512, None, None, None) == 1
    assert b"NULL" in lib.csa2_last_error_string()
    # a cache with planes but no layout
    buf = ctypes.create_string_buffer(1024)
    addr = (ctypes.addressof(buf) + 15) & ~15
    c.kv_codes = c.kv_scales = c.ix_codes = c.ix_scales = c.num_entries = addr
    c.batch, c.ratio, c.num_slots = 1, 1, 1
    assert lib.csa2_index_score(addr, addr, 1, 1, addr, None, 0, 16, ctypes.byref(c), addr, None, None) == 1
    c.seq_stride = 4
    assert lib.csa2_index_score(addr, addr, 2, 1, addr, None, 0, 16, ctypes.byref(c), addr, None, None) == 2
    c.ratio = 0
    assert lib.csa2_pack_kv(addr, addr, 0, None, 1, 1, addr, ctypes.byref(c), None, None) == 1
    # bad window / mode / workspace
    assert lib.csa2_swa_attn(addr, 1, 1, addr, addr, addr, 64, 128, 1.0, addr, addr, None, None) == 1
    c.ratio = 1
    assert lib.csa2_sparse_attn(7, addr, 1, 1, addr, 1.0, None, None, 512, 0, None, None, None, 16,
                                ctypes.byref(c), None, None, 0, 0, None, addr, addr, None, 0, None, None) == 1
    assert lib.csa2_sparse_attn(2, addr, 1, 1, addr, 1.0, None, None, 1024, 0, None, addr, None, 16,
                                ctypes.byref(c), None, None, 0, 0, None, addr, addr, None, 0, None, None) == 3
    assert lib.csa2_sparse_attn(0, addr, 1, 1, addr, 1.0, addr, addr, 512, 0, None, None, None, 16,
                                ctypes.byref(c), None, None, 0, 0, None, addr, addr, None, 0, None, None) == 1
    assert b"workspace" in lib.csa2_last_error_string()
    # this step's window token needs the window branch and one query per sequence
    assert lib.csa2_sparse_attn(2, addr, 1, 2, addr, 1.0, None, None, 512, 0, None, addr, None, 16,
                                ctypes.byref(c), addr, addr, 128, 128, addr, addr, addr, None, 0, None, None) == 1
    assert b"swa_new" in lib.csa2_last_error_string()


def test_zero_work_calls_are_no_ops(lib):
    # nothing to do: CSA2_OK without reading any pointer (all NULL here) and without a launch
    assert lib.csa2_pack_kv(None, None, 0, None, 0, 5, None, None, None, None) == 0
    assert lib.csa2_pack_swa(None, 0, 3, 0, None, None, None, 128, None, None) == 0
    assert lib.csa2_index_score(None, None, 0, 1, None, None, 0, 16, None, None, None, None) == 0
    assert lib.csa2_topk(None, None, 0, 10, 5, None, None, 0, None, None, None) == 0
    assert lib.csa2_sparse_attn(2, None, 0, 1, None, 1.0, None, None, 512, 0, None, None, None, 16,
                                None, None, None, 0, 0, None, None, None, None, 0, None, None) == 0
    assert lib.csa2_swa_attn(None, 0, 1, None, None, None, 128, 128, 1.0, None, None, None, None) == 0
    assert lib.csa2_merge(None, None, None, None, 0, 512, None, None, None) == 0
    # negative sizes are still errors
    assert lib.csa2_topk(None, None, -1, 10, 5, None, None, 0, None, None, None) == 1
    assert lib.csa2_merge(None, None, None, None, -1, 512, None, None, None) == 1
