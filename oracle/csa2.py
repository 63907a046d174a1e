"""CSA2 decode/prefill steps restated plainly on the CPU (float64 unless noted).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module;
only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg use it.

Pages, by title:
  [XHH]   "DeepSeek-V4.1 模型结构（0）：一张图看懂 DeepSeek-V4.1-Flash"
  [DAIW]  "DeepSeek V4.1 Flash 深度解析"
  [PRISM] "从V4到V4.1 Flash：架构的激进进化"

The pages give the modes, sizes and byte counts but no formulas.  Readings:
  * compressor: entry j = sum over its r tokens of w_t * x_t in fp32, left to
    right, each product and sum rounded separately; w_t = fp32(1/r) by default.
  * indexer score: s_n = sum_h w_h * relu(q^_h . k^_n) with q^ the MXFP4
    quantisation of the indexer query (same codec as the keys), no 1/sqrt(d).
  * visibility: entry n exists for a query at position p iff
    n < min(num_entries, floor((p + 1) / r)).
  * top-k: order by (score desc, index asc), keep k, return ascending index,
    pad with -1.
  * attention: one dequantised 512-d entry serves as key and value; logits
    tau * q . v, natural-log lse; an empty key set gives o = 0, lse = -inf.
  * SWA: window = positions max(0, p - W + 1) .. p, same attention.
  * merge of the two branches: log-sum-exp combination (one softmax over the
    union of both key sets).
"""
import math

import numpy as np

from . import formats as F

NEG_INF = -math.inf

# --------------------------------------------------------------------------- schedule
# [XHH] Q&A "40 层具体如何排布": layers 0-1 pure SWA; Full 2, 8, 14, 20;
# Reindex 24, 28, 32, 36; the rest Reuse.  [PRISM] 编码器层 / 解码器层: encoder
# CSA2 layers compress about two tokens per entry, the decoder keeps ratio 1.
NUM_LAYERS = 40
SWA_ONLY_LAYERS = (0, 1)
FULL_LAYERS = {2: 2, 8: 2, 14: 2, 20: 1}          # layer -> compression ratio
REINDEX_LAYERS = (24, 28, 32, 36)


def layer_mode(layer):
    if layer in SWA_ONLY_LAYERS:
        return "swa"
    if layer in FULL_LAYERS:
        return "full"
    if layer in REINDEX_LAYERS:
        return "reindex"
    return "reuse"


def entries_per_token():
    """Only Full layers write global KV, one entry per `ratio` tokens."""
    return sum(1.0 / r for r in FULL_LAYERS.values())


def global_kv_bytes_per_token():
    return entries_per_token() * (F.MAIN_ENTRY_BYTES + F.IX_ENTRY_BYTES)


# --------------------------------------------------------------------------- compressor
def compress(lat, ratio, pool_w=None):
    """[T, d] token latents -> [floor(T / r), d] entry latents (fp32)."""
    lat = np.asarray(lat, dtype=np.float32)
    T = lat.shape[0]
    n = T // ratio
    if pool_w is None:
        w = np.full(T, np.float32(1.0) / np.float32(ratio), dtype=np.float32)
    else:
        w = np.asarray(pool_w, dtype=np.float32)
    out = np.empty((n,) + lat.shape[1:], dtype=np.float32)
    for j in range(n):
        t0 = j * ratio
        acc = (w[t0] * lat[t0]).astype(np.float32)
        for t in range(t0 + 1, t0 + ratio):
            acc = (acc + (w[t] * lat[t]).astype(np.float32)).astype(np.float32)
        out[j] = acc
    return out


# Reading for a learned ("gated") compressor: [PRISM] 编码器层 says only that the encoder pools
# about two tokens into an entry; the rule is a learned weighting the pages do not give.  Read
# as a gated sum: per channel, the r tokens of a group are weighted by the softmax (over those
# r tokens) of gate logits that the model computes and the caller supplies.  Every step is an
# fp32 operation in a fixed order, exp included, so that the quantised codes are one answer.
LOG2E_F32 = np.float32(1.4426950408889634)
EXP2_TAYLOR_F32 = [np.float32(math.log(2) ** i / math.factorial(i)) for i in range(8)]


def exp_fp32(x):
    """exp(x) from fp32 operations: t = x log2(e), n = rint(t), f = t - n, 2^f = e^(f ln 2) by its
    Taylor polynomial of degree 7 (Horner, each product and sum rounded), times 2^n (0 below
    2^-126, inf above 2^127)."""
    x = np.asarray(x, np.float32)
    t = (x * LOG2E_F32).astype(np.float32)
    n = np.rint(t).astype(np.float32)
    f = (t - n).astype(np.float32)
    p = np.full(x.shape, EXP2_TAYLOR_F32[7], np.float32)
    for c in EXP2_TAYLOR_F32[6::-1]:
        p = (p * f).astype(np.float32)
        p = (p + c).astype(np.float32)
    ni = n.astype(np.int64)
    scale = np.ldexp(np.ones(x.shape, np.float32), np.clip(ni, -126, 127)).astype(np.float32)
    out = (p * scale).astype(np.float32)
    out = np.where(ni < -126, np.float32(0), out)
    return np.where(ni > 127, np.float32(np.inf), out).astype(np.float32)


def compress_gated(lat, gate, ratio):
    """[T, d] latents and [T, d] gate logits -> [floor(T / r), d] entries: per channel the softmax
    of the group's logits (max subtracted, exp_fp32, sum left to right, fp32 division) weights the
    group's latents, summed left to right."""
    lat = np.asarray(lat, dtype=np.float32)
    gate = np.asarray(gate, dtype=np.float32)
    n = lat.shape[0] // ratio
    out = np.empty((n,) + lat.shape[1:], dtype=np.float32)
    for j in range(n):
        g = gate[j * ratio:(j + 1) * ratio]
        e = exp_fp32((g - g.max(axis=0)).astype(np.float32))
        den = e[0]
        for t in range(1, ratio):
            den = (den + e[t]).astype(np.float32)
        acc = None
        for t in range(ratio):
            term = ((e[t] / den).astype(np.float32) * lat[j * ratio + t]).astype(np.float32)
            acc = term if acc is None else (acc + term).astype(np.float32)
        out[j] = acc
    return out


class Cache:
    """Logical per-sequence global KV planes (the oracle ignores physical paging)."""

    def __init__(self, B, capacity, ratio):
        self.ratio = ratio
        self.kv_codes = np.zeros((B, capacity, F.MAIN_CODE_BYTES), np.uint8)
        self.kv_scales = np.zeros((B, capacity, F.MAIN_SCALE_BYTES), np.uint8)
        self.ix_codes = np.zeros((B, capacity, F.IX_CODE_BYTES), np.uint8)
        self.ix_scales = np.zeros((B, capacity, F.IX_SCALE_BYTES), np.uint8)
        self.num_entries = np.zeros(B, np.int64)

    def pack(self, b, first_entry, lat_kv, lat_ix, pool_w=None):
        """Compress and quantise a run of tokens of sequence b into entries."""
        ekv = compress(lat_kv, self.ratio, pool_w)
        eix = compress(lat_ix, self.ratio, pool_w)
        n = ekv.shape[0]
        sl = slice(first_entry, first_entry + n)
        self.kv_codes[b, sl], self.kv_scales[b, sl] = F.pack_main(ekv)
        self.ix_codes[b, sl], self.ix_scales[b, sl] = F.pack_indexer(eix)
        return n

    def visible(self, b, pos):
        return int(min(self.num_entries[b], (pos + 1) // self.ratio))

    def main_values(self, b, idx):
        return F.unpack_main(self.kv_codes[b, idx], self.kv_scales[b, idx])

    def indexer_values(self, b, idx):
        return F.unpack_indexer(self.ix_codes[b, idx], self.ix_scales[b, idx])


# --------------------------------------------------------------------------- indexer
def quantised_query(q_ix):
    """MXFP4 quantisation of the indexer query heads: [H_I, 128] -> float64."""
    c, s = F.pack_indexer(np.asarray(q_ix, dtype=np.float32))
    return F.unpack_indexer(c, s)


def indexer_scores(q_ix, w, keys):
    """Lightning-indexer score of each key row.

    q_ix [H_I, 128] fp32, w [H_I], keys [n, 128] dequantised -> [n] float64.
    """
    qh = quantised_query(q_ix)
    dots = np.asarray(keys, dtype=np.float64) @ qh.T           # [n, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64)


# --------------------------------------------------------------------------- top-k
def topk(scores, k, n_valid=None):
    """Positions of the k best scores, ascending, -1 padded.

    Candidates are positions < n_valid whose score is not -inf; the order is
    score descending, then position ascending.
    """
    s = np.asarray(scores, dtype=np.float64)
    n = len(s) if n_valid is None else min(int(n_valid), len(s))
    pos = np.arange(n)
    pos = pos[s[:n] != NEG_INF]
    order = pos[np.lexsort((pos, -s[pos]))]
    sel = np.sort(order[:k])
    out = np.full(k, -1, np.int64)
    out[: len(sel)] = sel
    return out


# --------------------------------------------------------------------------- attention
def attend(q, keys, tau):
    """Softmax attention of heads q [H, D] over keys [m, D] used as values too."""
    q = np.asarray(q, dtype=np.float64)
    H, D = q.shape
    keys = np.asarray(keys, dtype=np.float64).reshape(-1, D)
    if keys.shape[0] == 0:
        return np.zeros((H, D)), np.full(H, NEG_INF)
    logits = tau * (q @ keys.T)
    mx = logits.max(axis=1)
    e = np.exp(logits - mx[:, None])
    ssum = e.sum(axis=1)
    return (e @ keys) / ssum[:, None], mx + np.log(ssum)


def merge(o1, l1, o2, l2):
    """Combine two attention partials over disjoint key sets."""
    o1, o2 = np.asarray(o1, np.float64), np.asarray(o2, np.float64)
    l1, l2 = np.asarray(l1, np.float64), np.asarray(l2, np.float64)
    m = np.maximum(l1, l2)
    empty = m == NEG_INF
    ms = np.where(empty, 0.0, m)
    a1 = np.where(l1 == NEG_INF, 0.0, np.exp(l1 - ms))
    a2 = np.where(l2 == NEG_INF, 0.0, np.exp(l2 - ms))
    den = np.where(empty, 1.0, a1 + a2)
    o = (a1[..., None] * o1 + a2[..., None] * o2) / den[..., None]
    lse = np.where(empty, NEG_INF, ms + np.log(den))
    return o, lse


# --------------------------------------------------------------------------- modes
def full_select(cache, b, pos, q_ix, w, k, pool_k=0):
    """Full mode: score every visible entry, keep top-k (and the top-pool_k pool)."""
    n = cache.visible(b, pos)
    scores = indexer_scores(q_ix, w, cache.indexer_values(b, np.arange(n)))
    idx = topk(scores, k)
    pool = topk(scores, pool_k) if pool_k > 0 else None
    return idx, pool, scores


def reindex_select(cache, b, pos, q_ix, w, k, pool):
    """Reindex mode: score only the pool's entries, keep their top-k."""
    pool = np.asarray(pool, dtype=np.int64)
    n = cache.visible(b, pos)
    scores = np.full(len(pool), NEG_INF)
    live = (pool >= 0) & (pool < n)
    if live.any():
        scores[live] = indexer_scores(q_ix, w, cache.indexer_values(b, pool[live]))
    sel = topk(scores, k)
    out = np.where(sel >= 0, pool[np.maximum(sel, 0)], -1)
    return out, scores


def sparse_attention(cache, b, q, idx, tau):
    """Attention of q [H, 512] over the listed entries (-1 entries skipped)."""
    idx = np.asarray(idx, dtype=np.int64)
    idx = idx[idx >= 0]
    return attend(q, cache.main_values(b, idx), tau)


def swa_attention(q, pos, swa_codes, swa_scale, window, tau):
    """Sliding-window branch for one query: ring slot of position t is t mod R."""
    R = swa_codes.shape[0]
    lo = max(0, pos - window + 1)
    slots = np.arange(lo, pos + 1) % R
    keys = F.unpack_swa(swa_codes[slots], swa_scale[slots])
    return attend(q, keys, tau)


def decode_layer(mode, cache, b, pos, q, tau, swa, window=128, q_ix=None, w=None,
                 k=512, pool_k=0, pool=None, idx=None):
    """One CSA2 layer for one query: global branch, SWA branch, merge.

    swa = (codes [R, 512], scale [R]) of this layer.  Returns a dict with o,
    lse, idx (the entries attended) and pool (Full with pool_k > 0).
    """
    out = {"pool": None}
    if mode == "full":
        idx, out["pool"], _ = full_select(cache, b, pos, q_ix, w, k, pool_k)
    elif mode == "reindex":
        idx, _ = reindex_select(cache, b, pos, q_ix, w, k, pool)
    elif mode != "reuse":
        raise ValueError(mode)
    o1, l1 = sparse_attention(cache, b, q, idx, tau)
    o2, l2 = swa_attention(q, pos, swa[0], swa[1], window, tau)
    out["o"], out["lse"] = merge(o1, l1, o2, l2)
    out["idx"] = np.asarray(idx)
    out["sparse"] = (o1, l1)
    out["swa"] = (o2, l2)
    return out


# --------------------------------------------------------------------------- the layer stack
# [XHH] Q&A "40 层具体如何排布" gives each layer's mode; 延伸解读 "CSA2 共享池": only the Full
# layers produce global KV and the layers after them reuse it (Reuse also reuses the indices of
# the nearest layer that selected them).  [PRISM] 解码器层: the decoder's first layer (the last
# Full layer) keeps the candidate pool that the Reindex layers search.
def pool_layer():
    return max(FULL_LAYERS)


def decode_model(caches, b, pos, layers, tau, k=512, pool_k=16384, window=128):
    """One decode token of sequence b at position pos through the NUM_LAYERS layers.

    caches: {Full layer -> Cache} (each Full layer's own global KV, written at its ratio);
    layers[l]: dict with q [H, 512], swa = (codes [R, 512], scale [R]) and, for Full and Reindex
    layers, q_ix [H_I, 128] and w [H_I].  Returns per layer the decode_layer dict plus "head"
    (the layer whose entries it attends, or None for the sliding-window-only layers).
    """
    out = []
    head, head_cache = None, None
    for l in range(NUM_LAYERS):
        mode, L = layer_mode(l), layers[l]
        if mode == "swa":
            o, lse = swa_attention(L["q"], pos, L["swa"][0], L["swa"][1], window, tau)
            out.append({"o": o, "lse": lse, "idx": None, "pool": None, "head": None})
            continue
        if mode == "full":
            head, head_cache = l, caches[l]
            r = decode_layer("full", head_cache, b, pos, L["q"], tau, L["swa"], window, q_ix=L["q_ix"], w=L["w"],
                             k=k, pool_k=pool_k if l == pool_layer() else 0)
        elif mode == "reindex":
            head, head_cache = l, caches[pool_layer()]
            r = decode_layer("reindex", head_cache, b, pos, L["q"], tau, L["swa"], window, q_ix=L["q_ix"],
                             w=L["w"], k=k, pool=out[pool_layer()]["pool"])
        else:
            r = decode_layer("reuse", head_cache, b, pos, L["q"], tau, L["swa"], window, idx=out[head]["idx"])
        r["head"] = head
        out.append(r)
    return out
