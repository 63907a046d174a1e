"""Shared pieces of the GPU parity tests: build caches on both sides, compare results.

The GPU side packs with the library; the oracle side packs the same seeded
latents (copied to the host as fp32) with its own codec.  Nothing flows from
the GPU path into the oracle.
"""
import math

import numpy as np
import torch

from oracle import csa2 as OC
from oracle import formats as OF
from workloads import configs as W

ATOL_MAX, ATOL_MEAN = 2e-3, 2e-4     # attention outputs: max-abs / mean-abs vs the oracle
TOPK_GAP = 1e-4                      # relative gap above which top-k sets must match exactly


def K():
    import compressed_sparse_attention_score_b200 as k
    return k


# ------------------------------------------------------------------ caches
def gpu_cache(spec, device="cuda", seqs=None, ratio=None):
    """Pack the spec's sequences into a device cache through csa2_pack_kv."""
    k = K()
    ratio = spec.ratio if ratio is None else ratio
    if spec.paged:
        table, pages = W.page_layout(spec, device)
        cache = k.GlobalKVCache(spec.B, ratio, num_slots=pages * spec.page_size, page_table=table,
                                page_size=spec.page_size)
    else:
        cache = k.GlobalKVCache(spec.B, ratio, seq_stride=max(spec.max_entries, 1))
    err = torch.zeros(1, dtype=torch.int32, device=device)
    for b in (range(spec.B) if seqs is None else seqs):
        kv, ix = W.token_latents(spec, b, device)
        view = cache.seq_view(b)
        view.ratio = spec.seq_ratio(b)
        k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(),
                       torch.zeros(1, dtype=torch.int32, device=device), view, err=err)
        cache.num_entries[b] = spec.entries(b)
        del kv, ix
    assert k.csa2_check(err) == 0
    return cache


def oracle_seq(spec, b, main_rows=None, gen_device="cpu"):
    """Oracle cache (batch 1) of sequence b: every indexer key, main entries for main_rows (None = all)."""
    kv, ix = W.token_latents(spec, b, gen_device)
    kv = kv.float().cpu().numpy()
    ix = ix.float().cpu().numpy()
    r = spec.seq_ratio(b)
    n = spec.entries(b)
    c = OC.Cache(1, max(n, 1), r)
    c.num_entries[0] = n
    eix = OC.compress(ix[: n * r], r) if r > 1 else ix[:n]
    c.ix_codes[0, :n], c.ix_scales[0, :n] = OF.pack_indexer(eix)
    rows = np.arange(n) if main_rows is None else np.unique(np.asarray(main_rows, np.int64))
    rows = rows[(rows >= 0) & (rows < n)]
    if len(rows):
        tok = (rows[:, None] * r + np.arange(r)[None, :]).reshape(-1)
        ekv = OC.compress(kv[tok], r)
        c.kv_codes[0, rows], c.kv_scales[0, rows] = OF.pack_main(ekv)
    return c


def fill_main(c, spec, b, rows, gen_device="cpu"):
    """Pack more main entries into an oracle cache made by oracle_seq."""
    kv, _ = W.token_latents(spec, b, gen_device)
    kv = kv.float().cpu().numpy()
    r = spec.seq_ratio(b)
    rows = np.unique(np.asarray(rows, np.int64))
    rows = rows[(rows >= 0) & (rows < c.num_entries[0])]
    if len(rows):
        tok = (rows[:, None] * r + np.arange(r)[None, :]).reshape(-1)
        c.kv_codes[0, rows], c.kv_scales[0, rows] = OF.pack_main(OC.compress(kv[tok], r))


def oracle_swa(x, pos, R):
    """Oracle SWA ring of one sequence from hidden states x [T][512] at positions pos [T]."""
    codes = np.zeros((R, 512), np.uint8)
    scale = np.zeros(R, np.float32)
    c, s = OF.pack_swa(np.asarray(x, np.float32))
    for t in range(len(pos)):
        if pos[t] >= 0:
            codes[pos[t] % R], scale[pos[t] % R] = c[t], s[t]
    return codes, scale


# ------------------------------------------------------------------ comparisons
def check_attention(o, lse, oo, ol, what=""):
    o = np.asarray(o, np.float64)
    oo = np.asarray(oo, np.float64)
    lse = np.asarray(lse, np.float64)
    ol = np.asarray(ol, np.float64)
    assert o.shape == oo.shape, (o.shape, oo.shape)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(ol), err_msg=f"{what}: empty rows differ")
    d = np.abs(o - oo)
    assert d.max() <= ATOL_MAX, f"{what}: o max-abs {d.max():.3g}"
    assert d.mean() <= ATOL_MEAN, f"{what}: o mean-abs {d.mean():.3g}"
    fin = np.isfinite(ol)
    if fin.any():
        dl = np.abs(lse[fin] - ol[fin])
        assert dl.max() <= ATOL_MAX, f"{what}: lse max-abs {dl.max():.3g}"
        assert dl.mean() <= ATOL_MEAN, f"{what}: lse mean-abs {dl.mean():.3g}"


def check_topk(gpu_idx, scores, oracle_idx, k, what=""):
    """Top-k parity: exact where the oracle's k/k+1 gap is clear, score multisets at near-ties.

    gpu_idx / oracle_idx are positions into `scores` (the oracle's float64 scores).
    Returns True when the sets are identical.
    """
    g = np.asarray(gpu_idx, np.int64)
    ref = np.asarray(oracle_idx, np.int64)
    s = np.asarray(scores, np.float64)
    gs = g[g >= 0]
    assert np.all(np.diff(gs) > 0), f"{what}: gpu indices not strictly ascending"
    assert np.all(g[len(gs):] == -1), f"{what}: pads not at the end"
    assert len(gs) == int((ref >= 0).sum()), f"{what}: count {len(gs)} vs {(ref >= 0).sum()}"
    if len(gs):
        assert gs.max() < len(s) and np.all(np.isfinite(s[gs])), f"{what}: selected an invalid position"
    if np.array_equal(g, ref):
        return True
    order = np.lexsort((np.arange(len(s)), -s))
    valid = np.isfinite(s)
    sk = s[order[k - 1]]
    sk1 = s[order[k]] if k < len(s) and valid[order[k]] else -math.inf
    gap = (sk - sk1) / max(abs(sk), 1e-30)
    assert gap <= TOPK_GAP, f"{what}: sets differ although the k/k+1 gap is {gap:.3g}"
    a = np.sort(s[gs])
    b = np.sort(s[ref[ref >= 0]])
    np.testing.assert_allclose(a, b, rtol=TOPK_GAP, atol=0, err_msg=f"{what}: near-tie score multisets")
    return False


def gpu_attend_given(q, q_pos, cache, tau, max_entries, idx, swa=None, fused=False):
    """GPU attention (Reuse mode) of the query rows q [B][Q][64][512] over the given entry lists
    idx [B][Q][k] (e.g. the oracle's selection where the GPU's differs at a near-tie).  With
    swa = (codes, scale) the sliding-window branch is merged: in the same call when fused, else
    by csa2_swa_attn + csa2_merge.  Returns (o, lse)."""
    k = K()
    err = torch.zeros(1, dtype=torch.int32, device=q.device)
    idx = torch.as_tensor(np.asarray(idx), dtype=torch.int32).to(q.device).contiguous()
    if swa is not None and fused:
        o, lse = k.csa2_sparse_attn("reuse", q, q_pos, cache, tau, max_entries, k=idx.shape[-1], idx_in=idx, err=err,
                                    swa_codes=swa[0], swa_scale=swa[1])
    else:
        o, lse = k.csa2_sparse_attn("reuse", q, q_pos, cache, tau, max_entries, k=idx.shape[-1], idx_in=idx, err=err)
        if swa is not None:
            o2, l2 = k.csa2_swa_attn(q, q_pos, swa[0], swa[1], tau, err=err)
            o, lse = k.csa2_merge(o, lse, o2, l2)
    assert k.csa2_check(err) == 0
    return o, lse


def to_np(t):
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float16) else t.detach().cpu().numpy()
