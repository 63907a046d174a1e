"""GPU parity of the multi-layer decode driver (csa2_decode_step) against the oracle's 40-layer stack.

One token per sequence goes through the pages' schedule (two window-only layers, four Full
layers over their own caches, four Reindex layers searching the decoder's pool, thirty Reuse
layers).  Every layer's output, every selection, the pool, the appended cache entries and the
packed window tokens are compared; where a selection legitimately differs at a near-tie the
GPU is re-run on the oracle's entries, so every layer is always compared.
"""
import numpy as np
import pytest
import torch

from oracle import csa2 as OC
from workloads import configs as W

from tests.helpers import (K, check_attention, check_topk, gpu_attend_given, oracle_seq, oracle_swa, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _model(T=4000, B=2, pool_k=1024):
    import bench
    spec = W.scaled(W.model40(), T, B=B, pool_k=pool_k)
    return spec, bench.Model40(spec, torch.device(DEV))


def test_decode_step_runs_the_pages_40_layers():
    k = K()
    spec, m = _model()
    m.step()
    torch.cuda.synchronize()
    assert k.csa2_check(m.err) == 0
    # the same step replayed from a CUDA graph gives the same bits
    eager = [t.clone() for t in (m.o, m.lse, m.idx, m.pool)]
    m.capture()
    for t in (m.o, m.lse):
        t.fill_(float("nan"))
    m.step(graphs=True)
    torch.cuda.synchronize()
    assert k.csa2_check(m.err) == 0
    for a, e in zip((m.o, m.lse, m.idx, m.pool), eager):
        assert torch.equal(a, e)
    full_layers = sorted(OC.FULL_LAYERS)
    assert m.ratios == [OC.FULL_LAYERS[f] for f in full_layers]
    pos = m.pos_
    compared = 0
    for b in range(spec.B):
        caches, oc_by_cache = {}, []
        for c, layer in enumerate(full_layers):
            r = m.ratios[c]
            oc = oracle_seq(m.cache_specs[c], b, gen_device=DEV)
            caches[layer] = oc
            oc_by_cache.append(oc)
            # this step appended the entry its token completed, bit for bit, and raised num_entries
            j = spec.tokens[b] // r - 1
            slot = b * m.caches[c].seq_stride + j
            assert int(m.caches[c].num_entries[b]) == j + 1 == int(oc.num_entries[0])
            for plane, ref in ((m.caches[c].kv_codes, oc.kv_codes), (m.caches[c].kv_scales, oc.kv_scales),
                               (m.caches[c].ix_codes, oc.ix_codes), (m.caches[c].ix_scales, oc.ix_scales)):
                np.testing.assert_array_equal(to_np(plane[slot]), ref[0, j])
        layers = []
        for layer in range(OC.NUM_LAYERS):
            x, p = W.swa_tokens(spec, layer, DEV)
            ring = oracle_swa(to_np(x[b]), to_np(p[b]), m.R)
            np.testing.assert_array_equal(to_np(m.swa_codes[layer, b]), ring[0])     # this token packed too
            np.testing.assert_array_equal(to_np(m.swa_scale[layer, b]), ring[1])
            layers.append({"q": to_np(m.q[layer, b]), "q_ix": to_np(m.q_ix[layer, b]), "w": to_np(m.w[layer, b]),
                           "swa": ring})
        ref = OC.decode_model(caches, 0, pos, layers, spec.tau, k=spec.k, pool_k=spec.pool_k)
        q_pos = m.pos[b:b + 1, None].contiguous()
        qrow = lambda layer: m.q[layer, b:b + 1, None].contiguous()   # noqa: E731
        swa = lambda layer: (m.swa_codes[layer, b:b + 1].contiguous(), m.swa_scale[layer, b:b + 1].contiguous())  # noqa
        direct = {}   # selecting layer -> the step's own outputs are comparable
        pool_same = True
        for layer in range(OC.NUM_LAYERS):
            mode, r = OC.layer_mode(layer), ref[layer]
            if mode == "swa":
                check_attention(to_np(m.o[layer, b]), to_np(m.lse[layer, b]), r["o"], r["lse"], f"swa {layer}")
                compared += 1
                continue
            if mode == "full":
                c = full_layers.index(layer)
                _, _, scores = OC.full_select(caches[layer], 0, pos, layers[layer]["q_ix"], layers[layer]["w"],
                                              spec.k)
                direct[layer] = check_topk(to_np(m.idx[layer, b]), scores, r["idx"], spec.k, f"full {layer}")
                if r["pool"] is not None:
                    check_topk(to_np(m.pool[c, b]), scores, r["pool"], spec.pool_k, f"pool {layer}")
                    pool_same = np.array_equal(to_np(m.pool[c, b]), r["pool"])
            elif mode == "reindex":
                pool = ref[OC.pool_layer()]["pool"]
                _, pscores = OC.reindex_select(caches[OC.pool_layer()], 0, pos, layers[layer]["q_ix"],
                                               layers[layer]["w"], spec.k, pool)
                if pool_same:
                    gi = to_np(m.idx[layer, b])
                else:     # the same Reindex call on the oracle's pool
                    err = torch.zeros(1, dtype=torch.int32, device=DEV)
                    gi_t = torch.empty((1, 1, spec.k), dtype=torch.int32, device=DEV)
                    k.csa2_sparse_attn("reindex", qrow(layer), q_pos, m.caches[3].seq_view(b), spec.tau,
                                       m.max_entries[3], k=spec.k, q_ix=m.q_ix[layer, b:b + 1, None].contiguous(),
                                       w=m.w[layer, b:b + 1, None].contiguous(), pool_k=spec.pool_k,
                                       pool_io=torch.from_numpy(pool[None, None]).to(torch.int32).to(DEV),
                                       idx_out=gi_t, err=err)
                    assert k.csa2_check(err) == 0
                    gi = to_np(gi_t[0, 0])
                gpos = np.array([np.searchsorted(pool, v) if v >= 0 else -1 for v in gi])
                rpos = np.array([np.searchsorted(pool, v) if v >= 0 else -1 for v in r["idx"]])
                direct[layer] = check_topk(gpos, pscores, rpos, spec.k, f"reindex {layer}") and pool_same
            h = r["head"]
            c = m.plan[h][2]
            if direct[h]:
                go, gl = m.o[layer, b], m.lse[layer, b]
            else:         # the layer on the oracle's entries
                go, gl = gpu_attend_given(qrow(layer), q_pos, m.caches[c].seq_view(b), spec.tau, m.max_entries[c],
                                          ref[h]["idx"][None, None], swa=swa(layer), fused=True)
                go, gl = go[0, 0], gl[0, 0]
            check_attention(to_np(go), to_np(gl), r["o"], r["lse"], f"{mode} {layer} b={b}")
            compared += 1
    assert compared == spec.B * OC.NUM_LAYERS


def test_reindex_recall_matches_the_oracle():
    """Recall of each Reindex layer's pool-restricted top-k against an exact top-k over the whole
    decoder cache: the GPU's figure against the oracle's on the same inputs."""
    spec, m = _model(T=6000, B=2, pool_k=1024)
    m.step()
    torch.cuda.synchronize()
    rec = m.reindex_recall()
    assert sorted(rec) == sorted(OC.REINDEX_LAYERS)
    dec = sorted(OC.FULL_LAYERS)[-1]
    c = len(m.ratios) - 1
    pos = m.pos_
    want = {layer: 0.0 for layer in rec}
    for b in range(spec.B):
        oc = oracle_seq(m.cache_specs[c], b, main_rows=[], gen_device=DEV)
        _, pool, _ = OC.full_select(oc, 0, pos, to_np(m.q_ix[dec, b]), to_np(m.w[dec, b]), spec.k, spec.pool_k)
        for layer in rec:
            q_ix, w = to_np(m.q_ix[layer, b]), to_np(m.w[layer, b])
            got, _ = OC.reindex_select(oc, 0, pos, q_ix, w, spec.k, pool)
            exact, _, _ = OC.full_select(oc, 0, pos, q_ix, w, spec.k)
            want[layer] += len(set(got.tolist()) & set(exact.tolist()) - {-1}) / spec.k / spec.B
    for layer in rec:
        assert abs(rec[layer] - want[layer]) <= 2.0 / spec.k, (layer, rec[layer], want[layer])
        assert 0.0 < want[layer] <= 1.0
