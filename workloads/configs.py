"""The five CSA2 workloads as seeded synthetic input recipes (shapes and draws only).

Every array is a function of (seed, name, sequence/layer index), so one
sequence's inputs can be regenerated alone on any device.  Nothing here
quantises, scores or attends: it only draws inputs.

  tiny_full   batch 1, 4096-token context at ratio 2 (2048 entries), Full mode
  reuse64k    batch 32, 65536 entries at ratio 1, 512 given indices, Reuse mode
  hier1m      batch 8, 2^20 entries at ratio 1, Full layer with a 16384 pool,
              then 4 Reindex layers; a planted 2% high-similarity key cluster
  prefill8k   8192 causal queries after a 262144-token prefix at ratio 2
  mixed64     64 ragged sequences (4096..2^20 tokens), even = Full at ratio 2,
              odd = Reuse at ratio 1, paged cache of 256-entry pages
"""
import math
from dataclasses import dataclass, field, replace

import torch

from . import choice, log_uniform_ints, normal, permutation, uniform

D, DI, H, HI = 512, 128, 64, 64
SWA_WINDOW = 128


@dataclass
class Spec:
    name: str
    B: int
    tokens: list            # context tokens per sequence (the query is the last one in decode)
    ratio: int
    mode: str               # "full", "reuse", "hier" (Full + Reindex layers), "prefill", "mixed"
    k: int = 512
    pool_k: int = 0
    n_reindex: int = 0
    tau: float = 1.0 / math.sqrt(D)
    q_std: float = 1.0
    cluster_frac: float = 0.0
    q_len: int = 1          # query tokens per sequence (prefill chunk length)
    paged: bool = False
    page_size: int = 256
    lat_dtype: torch.dtype = torch.float32
    seed: int = 0
    ratios: list = field(default_factory=list)   # per sequence (mixed)
    modes: list = field(default_factory=list)    # per sequence (mixed)

    def entries(self, b):
        return self.tokens[b] // self.seq_ratio(b)

    def seq_ratio(self, b):
        return self.ratios[b] if self.ratios else self.ratio

    def seq_mode(self, b):
        return self.modes[b] if self.modes else self.mode

    def query_pos(self, b):
        """Positions of this sequence's query tokens (the chunk ends at the last token)."""
        L = self.tokens[b]
        return list(range(L - self.q_len, L))

    @property
    def max_entries(self):
        return max(self.entries(b) for b in range(self.B))


def tiny_full(seed=0):
    return Spec("tiny_full", 1, [4096], 2, "full", seed=seed)


def reuse64k(seed=0):
    return Spec("reuse64k", 32, [65536] * 32, 1, "reuse", tau=1.0, q_std=1.0 / math.sqrt(D), seed=seed)


def hier1m(seed=0):
    return Spec("hier1m", 8, [1 << 20] * 8, 1, "hier", pool_k=16384, n_reindex=4, cluster_frac=0.02,
                lat_dtype=torch.bfloat16, seed=seed)


def prefill8k(seed=0):
    return Spec("prefill8k", 1, [262144 + 8192], 2, "prefill", q_len=8192, lat_dtype=torch.bfloat16, seed=seed)


def mixed64(seed=0):
    L = log_uniform_ints(64, 4096, 1 << 20, seed, "mixed", "lengths").tolist()
    ratios = [2 if b % 2 == 0 else 1 for b in range(64)]
    modes = ["full" if b % 2 == 0 else "reuse" for b in range(64)]
    return Spec("mixed64", 64, L, 1, "mixed", paged=True, ratios=ratios, modes=modes,
                lat_dtype=torch.bfloat16, seed=seed)


def model40(seed=0):
    """One decode token of 8 sequences at 2^20 tokens through the pages' 40-layer stack: four caches
    (three encoder caches at ratio 2, the decoder's at ratio 1, 16384-entry pool), each with the
    planted 2 % indexer cluster of hier1m."""
    return Spec("model40", 8, [1 << 20] * 8, 1, "model", pool_k=16384, cluster_frac=0.02,
                lat_dtype=torch.bfloat16, seed=seed)


CONFIGS = {"tiny_full": tiny_full, "reuse64k": reuse64k, "hier1m": hier1m, "prefill8k": prefill8k,
           "mixed64": mixed64, "model40": model40}


def cache_spec(spec, cache, ratio, shares_queries=False):
    """The latent recipe of one of a layer stack's caches (its own draws, its own ratio).  The cache
    that shares_queries keeps the stack's own draws, so its planted cluster is the one the
    indexer queries of query_tensors lean towards."""
    return replace(spec, name=spec.name if shares_queries else f"{spec.name}-cache{cache}", ratio=ratio)


def scaled(spec, tokens, B=None, **kw):
    """Same recipe at another size (parity cases the oracle finishes in seconds)."""
    B = spec.B if B is None else B
    toks = tokens if isinstance(tokens, list) else [tokens] * B
    extra = {}
    if spec.ratios:
        extra["ratios"] = spec.ratios[:B]
        extra["modes"] = spec.modes[:B]
    return replace(spec, B=B, tokens=toks, **extra, **kw)


# ---------------------------------------------------------------- draws
def cluster_center(spec, b, device="cpu"):
    return normal((DI,), spec.seed, spec.name, "cluster_u", b, device=device)


def cluster_positions(spec, b):
    n = spec.entries(b) * spec.seq_ratio(b)
    m = int(round(spec.cluster_frac * n))
    return choice(n, m, spec.seed, spec.name, "cluster_pos", b).to(torch.int64)


def token_latents(spec, b, device="cpu", start=0, stop=None):
    """Main-KV and indexer latents of tokens [start, stop) of sequence b (N(0,1))."""
    T = spec.tokens[b]
    kv = normal((T, D), spec.seed, spec.name, "lat_kv", b, device=device, dtype=spec.lat_dtype)
    ix = normal((T, DI), spec.seed, spec.name, "lat_ix", b, device=device, dtype=torch.float32)
    if spec.cluster_frac > 0:
        pos = cluster_positions(spec, b).to(device)
        u = cluster_center(spec, b, device)
        noise = normal((len(pos), DI), spec.seed, spec.name, "cluster_noise", b, device=device, std=0.5)
        ix[pos] = u + noise
    ix = ix.to(spec.lat_dtype)
    stop = T if stop is None else stop
    return kv[start:stop], ix[start:stop]


def query_tensors(spec, layer, device="cpu"):
    """q [B][Q][64][512], q_ix [B][Q][64][128], w [B][Q][64] (bf16) and q_pos [B][Q] for one layer."""
    B, Q = spec.B, spec.q_len
    q = normal((B, Q, H, D), spec.seed, spec.name, "q", layer, device=device, std=spec.q_std,
               dtype=torch.bfloat16)
    if spec.cluster_frac > 0:
        u = torch.stack([cluster_center(spec, b, device) for b in range(B)])
        q_ix = normal((B, Q, HI, DI), spec.seed, spec.name, "q_ix", layer, device=device)
        q_ix = (q_ix + u[:, None, None, :]).to(torch.bfloat16)
    else:
        q_ix = normal((B, Q, HI, DI), spec.seed, spec.name, "q_ix", layer, device=device, dtype=torch.bfloat16)
    w = uniform((B, Q, HI), spec.seed, spec.name, "w", layer, device=device, dtype=torch.bfloat16)
    q_pos = torch.tensor([spec.query_pos(b) for b in range(B)], dtype=torch.int32, device=device)
    return q, q_ix, w, q_pos


def reuse_indices(spec, device="cpu"):
    """[B][Q][k] entry indices, uniform without replacement over each sequence's entries."""
    rows = []
    for b in range(spec.B):
        n = spec.entries(b)
        per_q = [choice(n, min(spec.k, n), spec.seed, spec.name, "idx", b, qi) for qi in range(spec.q_len)]
        per_q = [torch.cat([r, torch.full((spec.k - len(r),), -1, dtype=torch.int32)]) for r in per_q]
        rows.append(torch.stack(per_q))
    return torch.stack(rows).to(device)


def swa_tokens(spec, layer, device="cpu"):
    """Hidden states of the tokens the SWA ring must hold: [B][W - 1 + Q][512] bf16 and their positions."""
    span = SWA_WINDOW - 1 + spec.q_len
    x = normal((spec.B, span, D), spec.seed, spec.name, "swa", layer, device=device, dtype=torch.bfloat16)
    pos = torch.tensor([[spec.tokens[b] - span + t for t in range(span)] for b in range(spec.B)],
                       dtype=torch.int32, device=device)
    return x, pos


def page_layout(spec, device="cpu"):
    """Paged cache: page_table [B][max_pages] (int32) into a shuffled global pool, and the pool size."""
    P = spec.page_size
    pages = [(spec.entries(b) + P - 1) // P for b in range(spec.B)]
    total = sum(pages)
    perm = permutation(total, spec.seed, spec.name, "pages")
    maxp = max(pages)
    table = torch.full((spec.B, maxp), -1, dtype=torch.int32)
    o = 0
    for b, n in enumerate(pages):
        table[b, :n] = perm[o:o + n]
        o += n
    return table.to(device), total
