"""csa2_sparse_attn_noalloc: the entry point for callers that cannot allocate device memory.

Such callers (an engine whose memory pool owns the whole device, a serving loop
that forbids cudaMalloc/cudaFree on its hot path) get scratch from a fixed array
inside the library instead of a workspace.  This file is collected last on
purpose; it runs both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from workloads import configs as W

from tests.helpers import ATOL_MAX, ATOL_MEAN, K, gpu_cache, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(lib, mode, q, q_pos, cache, tau, max_entries, k, q_ix, w, pool_k, pool_io, idx_out, o, lse, err):
    """Call the C entry point directly (plain pointers through the C ABI)."""
    d = cache.desc()
    B, Q = q.shape[0], q.shape[1]
    return lib.csa2_sparse_attn_noalloc(
        mode, q.data_ptr(), B, Q, q_pos.data_ptr(), ctypes.c_float(tau), q_ix.data_ptr(), w.data_ptr(), k, pool_k,
        None if pool_io is None else pool_io.data_ptr(), None, idx_out.data_ptr(), max_entries, ctypes.byref(d),
        None, None, 0, 0, o.data_ptr(), lse.data_ptr(), err.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _device_free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def _close(a, b):
    d = np.abs(to_np(a) - to_np(b))
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    k = K()
    lib = k.raw()
    spec = W.scaled(W.tiny_full(), [4096, 3001], B=2)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    _, q_ix2, w2, _ = W.query_tensors(spec, 1, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    # reference: the existing entry point with a caller workspace -- a Full layer with a pool, then a
    # Reindex layer on that pool
    idx_ref = torch.empty((2, 1, 512), dtype=torch.int32, device=DEV)
    pool_ref = torch.empty((2, 1, 1024), dtype=torch.int32, device=DEV)
    o_ref, lse_ref = k.csa2_sparse_attn("full", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w,
                                        pool_k=1024, pool_io=pool_ref, idx_out=idx_ref, err=err)
    ridx_ref = torch.empty((2, 1, 512), dtype=torch.int32, device=DEV)
    ro_ref, rlse_ref = k.csa2_sparse_attn("reindex", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix2, w=w2,
                                          pool_k=1024, pool_io=pool_ref, idx_out=ridx_ref, err=err)
    assert k.csa2_check(err) == 0
    assert 0 < k.csa2_workspace_size("full", 2, 1, spec.max_entries, 512, 1024) <= lib.csa2_noalloc_scratch_bytes()
    for it in range(2):
        o = torch.full((2, 1, 64, 512), float("nan"), dtype=torch.float32, device=DEV)
        lse = torch.full((2, 1, 64), float("nan"), dtype=torch.float32, device=DEV)
        idx = torch.full((2, 1, 512), -7, dtype=torch.int32, device=DEV)
        pool = torch.full((2, 1, 1024), -7, dtype=torch.int32, device=DEV)
        ro, rlse = torch.full_like(o, float("nan")), torch.full_like(lse, float("nan"))
        ridx = torch.full_like(idx, -7)
        free0 = _device_free_bytes()
        st = _call_noalloc(lib, 0, q, q_pos, cache, spec.tau, spec.max_entries, 512, q_ix, w, 1024, pool, idx, o,
                           lse, err)
        assert st == 0, lib.csa2_last_error_string()
        st = _call_noalloc(lib, 1, q, q_pos, cache, spec.tau, spec.max_entries, 512, q_ix2, w2, 1024, pool, ridx, ro,
                           rlse, err)
        assert st == 0, lib.csa2_last_error_string()
        if it > 0:   # the first call on the device loads the library's module, with the scratch in it
            assert _device_free_bytes() == free0      # later calls take no device memory
        assert k.csa2_check(err) == 0
        np.testing.assert_array_equal(to_np(idx), to_np(idx_ref))
        np.testing.assert_array_equal(to_np(pool), to_np(pool_ref))
        np.testing.assert_array_equal(to_np(ridx), to_np(ridx_ref))
        _close(o, o_ref)
        _close(lse, lse_ref)
        _close(ro, ro_ref)
        _close(rlse, rlse_ref)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    k = K()
    lib = k.raw()
    cap = lib.csa2_noalloc_scratch_bytes()
    spec = W.scaled(W.tiny_full(), [4096], B=1)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    o = torch.empty((1, 1, 64, 512), dtype=torch.float32, device=DEV)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((1, 1, 512), dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    too_many = cap // 4 + 1                       # more fp32 scores than the scratch holds
    assert k.csa2_workspace_size("full", 1, 1, too_many, 512, 0) > cap
    st = _call_noalloc(lib, 0, q, q_pos, cache, spec.tau, too_many, 512, q_ix, w, 0, None, idx, o, lse, err)
    assert st == 3  # CSA2_ERR_UNSUPPORTED
    assert b"static scratch" in lib.csa2_last_error_string()


def test_noalloc_reports_a_short_max_entries():
    """A query that sees more entries than max_entries (a caller that lowered it to fit the
    scratch) gets CSA2_ERR_SHAPE on the device, not a silently truncated scan."""
    k = K()
    lib = k.raw()
    spec = W.scaled(W.tiny_full(), [4096], B=1)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    o = torch.empty((1, 1, 64, 512), dtype=torch.float32, device=DEV)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((1, 1, 512), dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = _call_noalloc(lib, 0, q, q_pos, cache, spec.tau, 1500, 512, q_ix, w, 0, None, idx, o, lse, err)
    assert st == 0
    assert k.csa2_check(err) == 2  # CSA2_ERR_SHAPE: 2048 entries visible, 1500 scored
