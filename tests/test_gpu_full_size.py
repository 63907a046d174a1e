"""GPU parity at the full workload sizes, on sampled sequences / query rows the oracle computes one by one.

hier1m runs exactly the step bench.py times (same calls, same launch configuration, replayed from
CUDA graphs as the bench does after one eager step).
"""
import numpy as np
import pytest
import torch

from oracle import csa2 as OC
from workloads import configs as W

from tests.helpers import (K, check_attention, check_topk, fill_main, gpu_attend_given, gpu_cache, oracle_seq,
                           oracle_swa, to_np)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def _err():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _rings(spec, layer, R=128):
    k = K()
    x, pos = W.swa_tokens(spec, layer, DEV)
    codes = torch.zeros((spec.B, R, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((spec.B, R), dtype=torch.float32, device=DEV)
    k.csa2_pack_swa(x, pos, codes, scale, err=_err())
    return codes, scale, x, pos


def test_hier1m_bench_step_sampled():
    import bench
    spec = W.hier1m()
    wl = bench.Hier1M(spec, torch.device(DEV))
    wl.step()
    torch.cuda.synchronize()
    assert K().csa2_check(wl.err) == 0
    eager = [t.clone() for t in (wl.o, wl.lse, wl.idx, wl.pool)]
    wl.capture()
    for t in (wl.o, wl.lse):
        t.fill_(float("nan"))
    for t in (wl.idx, wl.pool):
        t.fill_(-7)
    wl.step(graphs=True)
    torch.cuda.synchronize()
    assert K().csa2_check(wl.err) == 0
    for a, e in zip((wl.o, wl.lse, wl.idx, wl.pool), eager):   # the graphs replay the same kernels
        assert torch.equal(a, e)
    b = 3
    c = oracle_seq(spec, b, main_rows=[], gen_device=DEV)
    pos = spec.tokens[b] - 1
    ring = []
    for layer in range(5):
        x, p = W.swa_tokens(spec, layer, DEV)
        ring.append(oracle_swa(to_np(x[b]), to_np(p[b]), 128))
    q = to_np(wl.q[:, b, 0])
    q_ix = to_np(wl.q_ix[:, b, 0])
    w = to_np(wl.w[:, b, 0])
    # Full layer: pool and top-512 over all 2^20 keys
    ref_idx, ref_pool, scores = OC.full_select(c, 0, pos, q_ix[0], w[0], spec.k, spec.pool_k)
    check_topk(to_np(wl.pool[b, 0]), scores, ref_pool, spec.pool_k, "hier1m pool")
    one = wl.cache.seq_view(b)
    qb = lambda layer: wl.q[layer][b:b + 1].contiguous()    # noqa: E731
    swa = lambda layer: (wl.swa_codes[layer][b:b + 1].contiguous(), wl.swa_scale[layer][b:b + 1].contiguous())  # noqa
    q_pos = wl.q_pos[b:b + 1].contiguous()
    go, gl = wl.o[0, b, 0], wl.lse[0, b, 0]
    if not check_topk(to_np(wl.idx[0, b, 0]), scores, ref_idx, spec.k, "hier1m full idx"):
        go, gl = gpu_attend_given(qb(0), q_pos, one, spec.tau, wl.N, ref_idx[None, None], swa=swa(0), fused=True)
        go, gl = go[0, 0], gl[0, 0]
    fill_main(c, spec, b, ref_idx, gen_device=DEV)
    ref = OC.decode_layer("reuse", c, 0, pos, q[0], spec.tau, ring[0], idx=ref_idx)
    check_attention(to_np(go), to_np(gl), ref["o"], ref["lse"], "hier1m full")
    compared = 1
    # the planted cluster dominates the selection
    cl = set(W.cluster_positions(spec, b).tolist())
    assert sum(int(i) in cl for i in ref_idx) > 0.9 * spec.k
    # Reindex layers, always on the oracle's pool: the bench step's own outputs where the GPU pool is
    # the oracle's, else the same Reindex call run again on the oracle's pool
    pool_same = np.array_equal(to_np(wl.pool[b, 0]), ref_pool)
    ref_pool_t = torch.from_numpy(ref_pool[None, None]).to(torch.int32).to(DEV)
    k = K()
    for layer in range(1, 5):
        ri, pscores = OC.reindex_select(c, 0, pos, q_ix[layer], w[layer], spec.k, ref_pool)
        if pool_same:
            gi, go, gl = to_np(wl.idx[layer, b, 0]), wl.o[layer, b, 0], wl.lse[layer, b, 0]
        else:
            err = torch.zeros(1, dtype=torch.int32, device=DEV)
            gi_t = torch.empty((1, 1, spec.k), dtype=torch.int32, device=DEV)
            go, gl = k.csa2_sparse_attn("reindex", qb(layer), q_pos, one, spec.tau, wl.N, k=spec.k,
                                        q_ix=wl.q_ix[layer][b:b + 1].contiguous(),
                                        w=wl.w[layer][b:b + 1].contiguous(), pool_k=spec.pool_k,
                                        pool_io=ref_pool_t, idx_out=gi_t, err=err, swa_codes=swa(layer)[0],
                                        swa_scale=swa(layer)[1])
            assert k.csa2_check(err) == 0
            gi, go, gl = to_np(gi_t[0, 0]), go[0, 0], gl[0, 0]
        gpos = np.array([np.searchsorted(ref_pool, v) if v >= 0 else -1 for v in gi])
        rpos = np.array([np.searchsorted(ref_pool, v) if v >= 0 else -1 for v in ri])
        if not check_topk(gpos, pscores, rpos, spec.k, f"hier1m reindex {layer}"):
            go, gl = gpu_attend_given(qb(layer), q_pos, one, spec.tau, wl.N, ri[None, None], swa=swa(layer),
                                      fused=True)
            go, gl = go[0, 0], gl[0, 0]
        fill_main(c, spec, b, ri, gen_device=DEV)
        ref = OC.decode_layer("reuse", c, 0, pos, q[layer], spec.tau, ring[layer], idx=ri)
        check_attention(to_np(go), to_np(gl), ref["o"], ref["lse"], f"hier1m reindex {layer}")
        compared += 1
    assert compared == 5


def test_reuse64k_full_size_sampled():
    k = K()
    spec = W.reuse64k()
    cache = gpu_cache(spec)
    q, _, _, q_pos = W.query_tensors(spec, 0, DEV)
    idx = W.reuse_indices(spec, DEV)
    codes, scale, x, pos = _rings(spec, 0)
    err = _err()
    o1, l1 = k.csa2_sparse_attn("reuse", q, q_pos, cache, spec.tau, spec.max_entries, idx_in=idx, err=err)
    o2, l2 = k.csa2_swa_attn(q, q_pos, codes, scale, spec.tau, err=err)
    o, lse = k.csa2_merge(o1, l1, o2, l2)
    assert k.csa2_check(err) == 0
    for b in (0, 17, 31):
        ri = to_np(idx[b, 0])
        c = oracle_seq(spec, b, main_rows=ri, gen_device=DEV)
        ring = oracle_swa(to_np(x[b]), to_np(pos[b]), 128)
        ref = OC.decode_layer("reuse", c, 0, int(q_pos[b, 0]), to_np(q[b, 0]), spec.tau, ring, idx=ri)
        check_attention(to_np(o[b, 0]), to_np(lse[b, 0]), ref["o"], ref["lse"], f"reuse64k b={b}")


def test_prefill8k_full_size_sampled():
    k = K()
    spec = W.prefill8k()
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    x, pos = W.swa_tokens(spec, 0, DEV)
    R = spec.q_len + 128
    codes = torch.zeros((1, R, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((1, R), dtype=torch.float32, device=DEV)
    err = _err()
    k.csa2_pack_swa(x, pos, codes, scale, err=err)
    idx_out = torch.empty((1, spec.q_len, spec.k), dtype=torch.int32, device=DEV)
    o1, l1 = k.csa2_sparse_attn("full", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w,
                                idx_out=idx_out, err=err)
    o2, l2 = k.csa2_swa_attn(q, q_pos, codes, scale, spec.tau, err=err)
    o, lse = k.csa2_merge(o1, l1, o2, l2)
    assert k.csa2_check(err) == 0
    c = oracle_seq(spec, 0, main_rows=[], gen_device=DEV)
    ring = oracle_swa(to_np(x[0]), to_np(pos[0]), R)
    rows = (0, 1, 4095, 8190, 8191)
    compared = 0
    for qi in rows:
        p = int(q_pos[0, qi])
        ref_idx, _, scores = OC.full_select(c, 0, p, to_np(q_ix[0, qi]), to_np(w[0, qi]), spec.k)
        go, gl = o[0, qi], lse[0, qi]
        if not check_topk(to_np(idx_out[0, qi]), scores, ref_idx, spec.k, f"prefill8k q={qi}"):
            go, gl = gpu_attend_given(q[:, qi:qi + 1].contiguous(), q_pos[:, qi:qi + 1].contiguous(), cache,
                                      spec.tau, spec.max_entries, ref_idx[None, None], swa=(codes, scale))
            go, gl = go[0, 0], gl[0, 0]
        fill_main(c, spec, 0, ref_idx, gen_device=DEV)
        ref = OC.decode_layer("reuse", c, 0, p, to_np(q[0, qi]), spec.tau, ring, idx=ref_idx)
        check_attention(to_np(go), to_np(gl), ref["o"], ref["lse"], f"prefill8k q={qi}")
        compared += 1
    assert compared == len(rows)


def test_mixed64_full_size_sampled():
    k = K()
    spec = W.mixed64()
    table, pages = W.page_layout(spec, DEV)
    base = k.GlobalKVCache(spec.B, 1, num_slots=pages * 256, page_table=table, page_size=256)
    err = _err()
    for b in range(spec.B):
        kv, ix = W.token_latents(spec, b, DEV)
        v = base.seq_view(b)
        v.ratio = spec.seq_ratio(b)
        k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), torch.zeros(1, dtype=torch.int32, device=DEV),
                       v, err=err)
        base.num_entries[b] = spec.entries(b)
        del kv, ix
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    idx_all = W.reuse_indices(spec, DEV)
    for mode, ratio, samples in (("full", 2, (0, 40)), ("reuse", 1, (1, 63))):
        ids = [b for b in range(spec.B) if spec.seq_mode(b) == mode]
        sel = torch.tensor(ids, device=DEV)
        view = k.GlobalKVCache(len(ids), ratio, num_slots=base.num_slots, page_table=table[sel].contiguous(),
                               page_size=256, planes=base.planes, num_entries=base.num_entries[sel].contiguous())
        maxe = max(spec.entries(b) for b in ids)
        idx_out = torch.empty((len(ids), 1, 512), dtype=torch.int32, device=DEV)
        o, lse = k.csa2_sparse_attn(mode, q[sel].contiguous(), q_pos[sel].contiguous(), view, spec.tau, maxe,
                                    q_ix=q_ix[sel].contiguous(), w=w[sel].contiguous(),
                                    idx_in=idx_all[sel].contiguous() if mode == "reuse" else None,
                                    idx_out=idx_out if mode == "full" else None, err=err)
        assert k.csa2_check(err) == 0
        compared = 0
        for b in samples:
            j = ids.index(b)
            p = int(q_pos[b, 0])
            c = oracle_seq(spec, b, main_rows=[], gen_device=DEV)
            go, gl = o[j, 0], lse[j, 0]
            if mode == "full":
                ref_idx, _, scores = OC.full_select(c, 0, p, to_np(q_ix[b, 0]), to_np(w[b, 0]), 512)
                if not check_topk(to_np(idx_out[j, 0]), scores, ref_idx, 512, f"mixed64 full b={b}"):
                    one = k.GlobalKVCache(1, ratio, num_slots=base.num_slots, page_table=table[b:b + 1].contiguous(),
                                          page_size=256, planes=base.planes,
                                          num_entries=base.num_entries[b:b + 1].contiguous())
                    go, gl = gpu_attend_given(q[b:b + 1].contiguous(), q_pos[b:b + 1].contiguous(), one, spec.tau,
                                              maxe, ref_idx[None, None])
                    go, gl = go[0, 0], gl[0, 0]
            else:
                ref_idx = to_np(idx_all[b, 0])
            fill_main(c, spec, b, ref_idx, gen_device=DEV)
            oo, ol = OC.sparse_attention(c, 0, to_np(q[b, 0]), ref_idx, spec.tau)
            check_attention(to_np(go), to_np(gl), oo, ol, f"mixed64 {mode} b={b}")
            compared += 1
        assert compared == len(samples)
