#!/usr/bin/env python
"""CSA2 decode benchmark: query-tokens/s per CSA2 layer on the hierarchical 1M-context workload.

One step = one decode token for each of the 8 sequences through one Full layer
and four Reindex layers over a 2^20-entry FP4 global KV cache:
  pack the token's global KV entry (main + indexer) and its SWA entry per layer,
  Full layer: indexer scan of all 2^20 entries, top-16384 pool + top-512,
              sparse attention, SWA attention, log-sum-exp merge,
  each Reindex layer: indexer over the pool, top-512, sparse attention, SWA, merge.
value = 8 tokens x 5 layers / step time (device-resident inputs, CUDA events).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl csa2|reference]
Under torchrun each rank runs its own 8 sequences (weak scaling, no collective
on the data path); timing is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import re
import threading
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode query-tokens/s per CSA2 layer at 64K–1M ctx; indexer+gather HBM GB/s vs peak"
UNIT = "query-tokens/s/layer"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["csa2", "reference"], default="csa2")
    ap.add_argument("--workload", default="hier1m")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seqs", type=int, default=1)
    ap.add_argument("--batch", type=int, default=0, help="override the sequence count (profiling runs)")
    ap.add_argument("--eager", action="store_true", help="launch every kernel from Python instead of replaying "
                    "CUDA graphs of the step")
    return ap.parse_args()


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons, read through NVML every 0.5 ms on a helper thread while the
    timed region runs (reads only: no clock or other GPU setting is changed)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, dev):
        self.sm, self.reasons, self.max_mhz, self.thread = [], set(), None, None
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(dev).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(dev.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self.nvml, self.h = pynvml, h
        self.done = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nvml
        masks = [(name, getattr(nv, attr, 0)) for name, attr in self.REASONS]
        while True:
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons.update(name for name, m in masks if bits & m)
            except Exception:
                return
            if self.done.wait(0.0005):
                return

    def stop(self):
        if self.thread is None:
            return None
        self.done.set()
        self.thread.join(timeout=5)
        if not self.sm:
            return None
        sm = sorted(self.sm)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(sm), "source": "NVML, every 0.5 ms during the timed steps"}


# ---------------------------------------------------------------- the workload on the GPU
class Hier1M:
    """Device state of the hierarchical Full -> Reindex decode workload."""

    LAYERS = 5   # one Full layer, four Reindex layers

    def __init__(self, spec, dev):
        import compressed_sparse_attention_score_b200 as k
        from workloads import configs as W
        self.k, self.spec, self.dev = k, spec, dev
        B, N = spec.B, spec.entries(0)
        self.B, self.N = B, N
        self.cache = k.GlobalKVCache(B, spec.ratio, seq_stride=N)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        for b in range(B):
            kv, ix = W.token_latents(spec, b, dev)
            k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), zero, self.cache.seq_view(b), err=err)
            del kv, ix
        self.cache.num_entries.fill_(N)
        torch.cuda.synchronize()
        # per-step inputs (device-resident copies; the e2e run refills them from pinned host memory)
        L = self.LAYERS
        self.new_kv = torch.empty((B, 1, 512), dtype=torch.bfloat16, device=dev)
        self.new_ix = torch.empty((B, 1, 128), dtype=torch.bfloat16, device=dev)
        kv_last, ix_last = [], []
        for b in range(B):
            kv, ix = W.token_latents(spec, b, dev, start=N - 1, stop=N)
            kv_last.append(kv)
            ix_last.append(ix)
        self.new_kv.copy_(torch.stack(kv_last))
        self.new_ix.copy_(torch.stack(ix_last))
        self.first_entry = torch.full((B,), N - 1, dtype=torch.int32, device=dev)
        qs = [W.query_tensors(spec, layer, dev) for layer in range(L)]
        self.q = torch.stack([t[0] for t in qs])          # [L][B][1][64][512]
        self.q_ix = torch.stack([t[1] for t in qs])       # [L][B][1][64][128]
        self.w = torch.stack([t[2] for t in qs])          # [L][B][1][64]
        self.q_pos = qs[0][3]                             # [B][1]
        self.R = 128
        self.swa_codes = torch.zeros((L, B, self.R, 512), dtype=torch.uint8, device=dev)
        self.swa_scale = torch.zeros((L, B, self.R), dtype=torch.float32, device=dev)
        self.swa_new = torch.empty((L, B, 1, 512), dtype=torch.bfloat16, device=dev)
        for layer in range(L):
            x, pos = W.swa_tokens(spec, layer, dev)
            k.csa2_pack_swa(x, pos, self.swa_codes[layer], self.swa_scale[layer], err=err)
            self.swa_new[layer].copy_(x[:, -1:, :])
        self.swa_pos = self.q_pos.contiguous()
        # outputs and scratch
        self.o = torch.empty((L, B, 1, 64, 512), dtype=torch.float32, device=dev)
        self.lse = torch.empty((L, B, 1, 64), dtype=torch.float32, device=dev)
        self.scores = torch.empty((B, 1, N), dtype=torch.float32, device=dev)
        self.pool = torch.empty((B, 1, spec.pool_k), dtype=torch.int32, device=dev)
        self.idx = torch.empty((L, B, 1, spec.k), dtype=torch.int32, device=dev)   # per layer
        self.ws_reindex = torch.empty(k.csa2_workspace_size("reindex", B, 1, N, spec.k, spec.pool_k),
                                      dtype=torch.uint8, device=dev)
        self.err = err
        torch.cuda.synchronize()
        assert k.csa2_check(err) == 0

    # kernels launched per step, by call: pack_kv 1; per layer one attention launch that packs the layer's window
    # token and covers the sparse branch, the SWA branch and their log-sum-exp merge; the Full layer's indexer
    # scan 1 and top-k 1 (its top-512 and pool share one launch); per Reindex layer one launch that scores the
    # pool and selects
    def launches_per_step(self):
        return 1 + 3 + (self.LAYERS - 1) * 2

    # The step in three parts: [pack the new token's entry], [the Full layer's scan], [its top-k and
    # attention; the four Reindex layers].  The scan stays a separate part so that CUDA events can time it
    # even when the other two parts are replayed as CUDA graphs.  Every layer's window token is packed into
    # its SWA ring inside that layer's attention launch (swa_new).
    def part_pre(self):
        self.k.csa2_pack_kv(self.new_kv, self.new_ix, self.first_entry, self.cache, err=self.err)

    def part_scan(self):
        self.k.csa2_index_score(self.q_ix[0], self.w[0], self.q_pos, self.cache, self.N, scores=self.scores,
                                err=self.err)

    def part_post(self):
        k, s = self.k, self.spec
        k.csa2_topk(self.scores, s.k, idx=self.idx[0], k2=s.pool_k, idx2=self.pool)
        for layer in range(self.LAYERS):
            q, q_ix, w = self.q[layer], self.q_ix[layer], self.w[layer]
            swa = dict(swa_codes=self.swa_codes[layer], swa_scale=self.swa_scale[layer], swa_new=self.swa_new[layer])
            if layer == 0:
                k.csa2_sparse_attn("reuse", q, self.q_pos, self.cache, s.tau, self.N, k=s.k, idx_in=self.idx[0],
                                   o=self.o[layer], lse=self.lse[layer], err=self.err, **swa)
            else:
                k.csa2_sparse_attn("reindex", q, self.q_pos, self.cache, s.tau, self.N, k=s.k, q_ix=q_ix, w=w,
                                   pool_k=s.pool_k, pool_io=self.pool, idx_out=self.idx[layer], o=self.o[layer],
                                   lse=self.lse[layer], ws=self.ws_reindex, err=self.err, **swa)

    def capture(self):
        """Record part_pre and part_post as CUDA graphs (after at least one eager step)."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.graphs = (torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph())
        with torch.cuda.stream(side):
            with torch.cuda.graph(self.graphs[0], stream=side):
                self.part_pre()
            with torch.cuda.graph(self.graphs[1], stream=side):
                self.part_post()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()

    def step(self, scan_events=None, graphs=False):
        """One decode step: eagerly, or replaying the captured graphs around an eager scan."""
        self.graphs[0].replay() if graphs else self.part_pre()
        if scan_events:
            scan_events[0].record()
        self.part_scan()
        if scan_events:
            scan_events[1].record()
        self.graphs[1].replay() if graphs else self.part_post()

    def host_io(self):
        """Pinned host copies of one step's inputs and outputs (for the end-to-end run)."""
        ins = [self.new_kv, self.new_ix, self.q, self.q_ix, self.w, self.swa_new]
        outs = [self.o, self.lse]
        h_in = [t.cpu().pin_memory() for t in ins]
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
        return ins, h_in, outs, h_out

    # Double-buffered step inputs and outputs, for an end-to-end loop that copies step i + 1's inputs
    # in and step i - 1's outputs out while step i computes.
    IO_NAMES = ("new_kv", "new_ix", "q", "q_ix", "w", "swa_new", "o", "lse")

    def make_buffer_sets(self, graphs):
        self.sets = [{n: getattr(self, n) for n in self.IO_NAMES}, {}]
        for n in self.IO_NAMES:
            t = getattr(self, n)
            self.sets[1][n] = t.clone() if n not in ("o", "lse") else torch.empty_like(t)
        self.set_graphs = [getattr(self, "graphs", None), None]
        if graphs:
            self.use_set(1)
            self.capture()
            self.set_graphs[1] = self.graphs
            self.use_set(0)

    def use_set(self, s):
        for n, t in self.sets[s].items():
            setattr(self, n, t)
        if getattr(self, "set_graphs", None) and self.set_graphs[s] is not None:
            self.graphs = self.set_graphs[s]

    def set_io(self, s):
        d = self.sets[s]
        return [d[n] for n in ("new_kv", "new_ix", "q", "q_ix", "w", "swa_new")], [d["o"], d["lse"]]

    def attention(self, layer):
        """The attention launch of one layer alone (its entries as given indices, its window fused)."""
        self.k.csa2_sparse_attn("reuse", self.q[layer], self.q_pos, self.cache, self.spec.tau, self.N, k=self.spec.k,
                                idx_in=self.idx[layer], o=self.o[layer], lse=self.lse[layer], err=self.err,
                                swa_codes=self.swa_codes[layer], swa_scale=self.swa_scale[layer])

    def gather_bytes(self):
        """Bytes one attention launch must move: per sequence its 512 listed main entries (288 B), its 128
        window tokens (516 B), its bf16 query heads (64 KB) and fp32 output heads (128 KB + lse)."""
        return self.B * (self.spec.k * 288 + 128 * 516 + 64 * 512 * 2 + 64 * 512 * 4 + 64 * 4)

    def scan_bytes(self):
        """Algorithmic bytes of one Full-layer indexer launch: every 68-byte indexer key read once.

        The fp32 score row (4 B per entry) is an artefact of handing the scores to a separate top-k
        launch, not of the method, so it counts as traffic, not as algorithmic bytes."""
        return self.B * self.N * 68


class Model40:
    """Device state of one decode token through the pages' 40-layer stack (csa2_decode_step).

    Four caches, one per Full layer (the encoder's three at ratio 2, the decoder's at ratio 1),
    hold every token before this step's, so the step itself appends the token to each of them
    (at ratio 2 the token before it waits in the staging rows); every layer's SWA ring holds the
    127 tokens before it and the step packs this token's.
    """

    R = 128

    def __init__(self, spec, dev):
        import compressed_sparse_attention_score_b200 as k
        from workloads import configs as W
        self.k, self.spec, self.dev = k, spec, dev
        self.plan, self.ratios = k.csa2_plan_v41()
        L, B, T = len(self.plan), spec.B, spec.tokens[0]
        assert all(t == T for t in spec.tokens), "one position for every sequence"
        self.L, self.B, self.T, self.pos_ = L, B, T, T - 1
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.err = err
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        nc = len(self.ratios)
        rmax = max(self.ratios)
        self.pos = torch.full((B,), T - 1, dtype=torch.int32, device=dev)
        self.new_kv = torch.empty((nc, B, 512), dtype=torch.bfloat16, device=dev)
        self.new_ix = torch.empty((nc, B, 128), dtype=torch.bfloat16, device=dev)
        self.kv_stage = torch.zeros((nc, B, rmax, 640), dtype=torch.float32, device=dev)
        self.caches, self.max_entries, self.cache_specs = [], [], []
        for c, r in enumerate(self.ratios):
            cs = W.cache_spec(spec, c, r, shares_queries=c == nc - 1)
            n = T // r
            cache = k.GlobalKVCache(B, r, seq_stride=(n + 127) // 128 * 128)
            p0 = (T - 1) // r * r                       # first token of this step's group
            for b in range(B):
                kv, ix = W.token_latents(cs, b, dev)
                k.csa2_pack_kv(kv[None, :p0].contiguous(), ix[None, :p0].contiguous(), zero, cache.seq_view(b),
                               err=err)
                self.new_kv[c, b].copy_(kv[T - 1])
                self.new_ix[c, b].copy_(ix[T - 1])
                for t in range(p0, T - 1):              # the group's earlier tokens wait in staging
                    view = cache.seq_view(b)
                    view.num_entries.fill_(p0 // r)
                    k.csa2_append_kv(kv[t:t + 1].contiguous(), ix[t:t + 1].contiguous(),
                                     torch.full((1,), t, dtype=torch.int32, device=dev), view,
                                     stage=self.kv_stage[c, b:b + 1], err=err)
                del kv, ix
            cache.num_entries.fill_(p0 // r)
            self.caches.append(cache)
            self.max_entries.append(n)
            self.cache_specs.append(cs)
        qs = [W.query_tensors(spec, layer, dev) for layer in range(L)]
        self.q = torch.stack([t[0][:, 0] for t in qs]).contiguous()        # [L][B][64][512]
        self.q_ix = torch.stack([t[1][:, 0] for t in qs]).contiguous()     # [L][B][64][128]
        self.w = torch.stack([t[2][:, 0] for t in qs]).contiguous()        # [L][B][64]
        self.swa_codes = torch.zeros((L, B, self.R, 512), dtype=torch.uint8, device=dev)
        self.swa_scale = torch.zeros((L, B, self.R), dtype=torch.float32, device=dev)
        self.swa_x = torch.empty((L, B, 512), dtype=torch.bfloat16, device=dev)
        for layer in range(L):
            x, p = W.swa_tokens(spec, layer, dev)
            k.csa2_pack_swa(x[:, :-1].contiguous(), p[:, :-1].contiguous(), self.swa_codes[layer],
                            self.swa_scale[layer], err=err)
            self.swa_x[layer].copy_(x[:, -1])
        self.idx = torch.full((L, B, spec.k), -1, dtype=torch.int32, device=dev)
        self.pool = torch.full((nc, B, spec.pool_k), -1, dtype=torch.int32, device=dev)
        self.o = torch.empty((L, B, 64, 512), dtype=torch.float32, device=dev)
        self.lse = torch.empty((L, B, 64), dtype=torch.float32, device=dev)
        self.dstep = k.DecodeStep(self.plan, self.caches, self.max_entries, self.pos, spec.tau, spec.k, spec.pool_k,
                                  self.q, self.swa_x, self.swa_codes, self.swa_scale, self.idx, self.o, self.lse,
                                  q_ix=self.q_ix, w=self.w, pool=self.pool, new_kv=self.new_kv, new_ix=self.new_ix,
                                  kv_stage=self.kv_stage, window=128)
        self.ws = torch.empty(max(1, self.dstep.workspace_size()), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        assert k.csa2_check(err) == 0

    def step(self, graphs=False):
        if graphs:
            self.graph.replay()
        else:
            self.dstep.run(self.ws, err=self.err)

    def capture(self):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(self.graph, stream=side):
                self.dstep.run(self.ws, err=self.err, stream=side)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()

    def launches_per_step(self):
        """Kernels of one step: one append per cache, per Full layer an indexer scan and a top-k, per
        Reindex layer one launch that scores its pool and selects, and per layer one attention launch
        (which also packs the layer's window token)."""
        full = sum(1 for m, _, _ in self.plan if m == 0)
        reindex = sum(1 for m, _, _ in self.plan if m == 1)
        return len(self.ratios) + 2 * full + reindex + len(self.plan)

    def reindex_recall(self):
        """Per Reindex layer: the share of its top-k (searched inside the decoder pool) that an exact
        top-k over the whole decoder cache with the same indexer query also picks."""
        k, out = self.k, {}
        c = self.plan[next(i for i, p in enumerate(self.plan) if p[0] == 1)][2]
        for layer, (m, _, _) in enumerate(self.plan):
            if m != 1:
                continue
            s = k.csa2_index_score(self.q_ix[layer][:, None].contiguous(), self.w[layer][:, None].contiguous(),
                                   self.pos[:, None].contiguous(), self.caches[c], self.max_entries[c], err=self.err)
            exact = k.csa2_topk(s, self.spec.k)[0][:, 0]
            got = self.idx[layer]
            hit = [len(set(got[b].tolist()) & set(exact[b].tolist()) - {-1}) / self.spec.k for b in range(self.B)]
            out[layer] = sum(hit) / len(hit)
        return out


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_sources, name):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"source_sha:\s*([0-9a-f]+)", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m or not t or m.group(1) != source_sha(kernel_sources):
        return None
    return float(t.group(1))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], "measured"
    return 6650.0, "fallback"


def tensor_peaks():
    """(dense bf16 TFLOP/s as a burst, kind): the measured cuBLAS figure, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ---------------------------------------------------------------- the oracle's time (CPU baseline)
def oracle_time(spec, n_seqs=1):
    """Time the oracle, as it stands, on `n_seqs` sequences of one decode step (all five layers)."""
    import numpy as np
    from oracle import csa2 as OC
    from oracle import formats as OF
    from workloads import configs as W
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    total = 0.0
    for b in range(n_seqs):
        kv, ix = W.token_latents(spec, b, "cpu")
        n = spec.entries(b)
        c = OC.Cache(1, n, spec.ratio)
        c.num_entries[0] = n
        c.ix_codes[0], c.ix_scales[0] = OF.pack_indexer(ix.float().numpy())
        qs = [W.query_tensors(spec, layer, "cpu") for layer in range(5)]
        swa = []
        for layer in range(5):
            x, pos = W.swa_tokens(spec, layer, "cpu")
            codes, sc = OF.pack_swa(x[b].float().numpy())
            ring_c = np.zeros((128, 512), np.uint8)
            ring_s = np.zeros(128, np.float32)
            p = pos[b].numpy()
            ring_c[p % 128], ring_s[p % 128] = codes, sc
            swa.append((ring_c, ring_s))
        kvn = kv.float().numpy()

        def run():
            pos = spec.tokens[b] - 1
            t0 = time.perf_counter()
            out = OC.decode_layer("full", c, 0, pos, qs[0][0][b, 0].float().numpy(), spec.tau, swa[0],
                                  q_ix=qs[0][1][b, 0].float().numpy(), w=qs[0][2][b, 0].float().numpy(),
                                  k=spec.k, pool_k=spec.pool_k)
            rows = [out["idx"]]
            for layer in range(1, 5):
                r = OC.decode_layer("reindex", c, 0, pos, qs[layer][0][b, 0].float().numpy(), spec.tau,
                                    swa[layer], q_ix=qs[layer][1][b, 0].float().numpy(),
                                    w=qs[layer][2][b, 0].float().numpy(), k=spec.k, pool=out["pool"])
                rows.append(r["idx"])
            return time.perf_counter() - t0, rows

        # untimed: put the main entries the step will read into the oracle cache
        _, rows = run()
        need = np.unique(np.concatenate(rows))
        need = need[need >= 0]
        c.kv_codes[0, need], c.kv_scales[0, need] = OF.pack_main(kvn[need])
        dt, _ = run()
        total += dt
    return total, cores


# ---------------------------------------------------------------- main
def run_reference(args, world, rank):
    from workloads import configs as W
    if rank != 0:
        return
    spec = W.CONFIGS[args.workload]()
    n = args.cpu_sample_seqs
    times = []
    for _ in range(args.warmup + args.steps):
        dt, cores = oracle_time(spec, n)
        times.append(dt)
    t = sum(times[args.warmup:]) / max(1, args.steps)
    value = n * 5 / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(spec),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n} of {spec.B} sequences, one decode step through all 5 layers"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(spec):
    return {"workload": f"{spec.name}: hierarchical Full->Reindex decode, batch {spec.B}, "
                        f"{spec.entries(0)} entries/seq at ratio {spec.ratio}, 1 Full + 4 Reindex layers",
            "batch": spec.B, "ctx_entries": spec.entries(0), "ratio": spec.ratio, "top_k": spec.k,
            "pool_k": spec.pool_k, "heads": 64, "indexer_heads": 64, "swa_window": 128,
            "layers_per_step": 5, "parallelism": "dp (independent sequences per rank)",
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, outside step events)"}


class OneLayer:
    """Device state of one CSA2 layer call over one of the other configurations, for their own lines:
    tiny_full (Full decode, 2048 entries), reuse64k (Reuse decode, 32 x 65536 entries), mixed64 (paged,
    32 Full sequences at ratio 2 and 32 Reuse sequences at ratio 1, two calls) and prefill8k (Full mode
    for 8192 causal query tokens).  Every call runs the sliding-window branch and the merge in the same
    launch as the sparse attention."""

    def __init__(self, spec, dev):
        import compressed_sparse_attention_score_b200 as k
        from workloads import configs as W
        self.k, self.spec, self.dev, self.W = k, spec, dev, W
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        B = spec.B
        self.q, self.q_ix, self.w, self.q_pos = W.query_tensors(spec, 0, dev)
        if spec.paged:
            table, pages = W.page_layout(spec, dev)
            self.base = k.GlobalKVCache(B, 1, num_slots=pages * spec.page_size, page_table=table,
                                        page_size=spec.page_size)
        else:
            self.base = k.GlobalKVCache(B, spec.ratio, seq_stride=(spec.max_entries + 127) // 128 * 128)
        for b in range(B):
            kv, ix = W.token_latents(spec, b, dev)
            v = self.base.seq_view(b)
            v.ratio = spec.seq_ratio(b)
            k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), zero, v, err=self.err)
            self.base.num_entries[b] = spec.entries(b)
            del kv, ix
        x, pos = W.swa_tokens(spec, 0, dev)
        self.R = 128 if spec.q_len == 1 else spec.q_len + 128
        self.codes = torch.zeros((B, self.R, 512), dtype=torch.uint8, device=dev)
        self.scale = torch.zeros((B, self.R), dtype=torch.float32, device=dev)
        k.csa2_pack_swa(x, pos, self.codes, self.scale, err=self.err)
        self.calls = []   # (mode, rows tensor index or None, view, max_entries, idx_in)
        if spec.name == "mixed64":
            for mode, ratio in (("full", 2), ("reuse", 1)):
                ids = [b for b in range(B) if spec.seq_mode(b) == mode]
                sel = torch.tensor(ids, device=dev)
                view = k.GlobalKVCache(len(ids), ratio, num_slots=self.base.num_slots,
                                       page_table=self.base.page_table[sel].contiguous(), page_size=spec.page_size,
                                       planes=self.base.planes, num_entries=self.base.num_entries[sel].contiguous())
                idx = W.reuse_indices(spec, dev)[sel].contiguous() if mode == "reuse" else None
                self.calls.append((mode, sel, view, max(spec.entries(b) for b in ids), idx))
        else:
            idx = W.reuse_indices(spec, dev) if spec.mode == "reuse" else None
            self.calls.append((spec.mode if spec.mode != "prefill" else "full", None, self.base, spec.max_entries, idx))
        self.io = []
        for mode, sel, view, me, idx in self.calls:
            take = (lambda t: t) if sel is None else (lambda t, s=sel: t[s].contiguous())
            rows = take(self.q)
            o = torch.empty(rows.shape[:2] + (64, 512), dtype=torch.float32, device=dev)
            lse = torch.empty(rows.shape[:2] + (64,), dtype=torch.float32, device=dev)
            nbytes = k.csa2_workspace_size(mode, rows.shape[0], rows.shape[1], me, spec.k)
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev) if nbytes else None
            self.io.append((rows, take(self.q_ix), take(self.w), take(self.q_pos), take(self.codes),
                            take(self.scale), o, lse, ws))
        torch.cuda.synchronize()
        assert k.csa2_check(self.err) == 0

    def step(self, graphs=False):
        if graphs:
            self.graph.replay()
            return
        for (mode, _, view, me, idx), (q, q_ix, w, q_pos, codes, scale, o, lse, ws) in zip(self.calls, self.io):
            self.k.csa2_sparse_attn(mode, q, q_pos, view, self.spec.tau, me, k=self.spec.k, q_ix=q_ix, w=w,
                                    idx_in=idx, o=o, lse=lse, ws=ws, err=self.err, swa_codes=codes, swa_scale=scale)

    def capture(self):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(self.graph, stream=side):
                self.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()

    def prefill_select(self):
        """The prefill chunk's fused indexer + top-k alone (csa2_index_topk)."""
        q, q_ix, w, q_pos = self.io[0][:4]
        self.sel = self.k.csa2_index_topk(q_ix, w, q_pos, self.base, self.spec.max_entries, k=self.spec.k,
                                          idx=getattr(self, "sel", None), err=self.err)

    def prefill_attend(self):
        """The prefill chunk's attention over that selection (with its window), alone."""
        q, q_ix, w, q_pos, codes, scale, o, lse, _ = self.io[0]
        if getattr(self, "sel", None) is None:
            self.prefill_select()
        self.k.csa2_sparse_attn("reuse", q, q_pos, self.base, self.spec.tau, self.spec.max_entries, k=self.spec.k,
                                idx_in=self.sel, o=o, lse=lse, err=self.err, swa_codes=codes, swa_scale=scale)

    def query_rows(self):
        return self.spec.B * self.spec.q_len

    def launches_per_step(self):
        """Full: indexer scan, top-k and attention, or for a prefill chunk (1024 rows or more) the fused
        indexer + top-k and attention; Reuse: attention."""
        n = 0
        for (mode, *_), io in zip(self.calls, self.io):
            rows = io[0].shape[0] * io[0].shape[1]
            n += (2 if rows >= 1024 else 3) if mode == "full" else 1
        return n

    def gather_bytes(self):
        """Bytes the attention must move per step: per query row its listed main entries (288 B each),
        its window tokens (516 B each), its bf16 query (64 KB) and fp32 output (128 KB + lse)."""
        rows = self.query_rows()
        return rows * (self.spec.k * 288 + 128 * 516 + 64 * 512 * 2 + 64 * 512 * 4 + 64 * 4)

    def scan_pairs(self):
        """(query, entry) pairs the indexer scores per step (Full calls)."""
        n = 0
        for (mode, sel, view, me, _), (q, *_rest) in zip(self.calls, self.io):
            if mode != "full":
                continue
            ids = range(self.spec.B) if sel is None else sel.tolist()
            for b in ids:
                r = self.spec.seq_ratio(b)
                n += sum(min(self.spec.entries(b), (p + 1) // r) for p in self.spec.query_pos(b))
        return n


def run_one_layer(args, spec, dev, world, rank):
    """Own JSON line of one of the other configurations: query-tokens/s of one CSA2 layer call."""
    wl = OneLayer(spec, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    graphs = not args.eager
    for i in range(args.warmup):
        wl.step(graphs=graphs and i > 0)
        if graphs and i == 0:
            wl.capture()
    torch.cuda.synchronize()
    assert wl.k.csa2_check(wl.err) == 0
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        wl.step(graphs=graphs)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, world)
    assert wl.k.csa2_check(wl.err) == 0
    peak, peak_kind = peaks()
    rows = wl.query_rows()
    pairs = wl.scan_pairs()
    line = {"metric": f"{spec.name}: query-tokens/s of one CSA2 layer (sparse + SWA + merge)",
            "value": world * rows / (step_ms * 1e-3), "unit": "query-tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": spec.name, "batch": spec.B, "query_tokens": rows, "top_k": spec.k,
                       "modes": sorted({m for m, *_ in wl.calls}),
                       "launch": "eager" if args.eager else "CUDA graph of the layer's calls",
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, outside step events)"},
            "gather": {"bytes_per_step": wl.gather_bytes(),
                       "GBps_whole_step": wl.gather_bytes() / (step_ms * 1e-3) / 1e9, "peak": peak,
                       "peak_kind": peak_kind},
            "gpu_launches": wl.launches_per_step() * args.steps, "clocks": clk}
    if pairs:
        line["indexer"] = {"pairs_per_step": pairs, "fp4_tflop_per_step": pairs * 64 * 128 * 2 / 1e12,
                           "fp4_tflops_whole_step": pairs * 64 * 128 * 2 / (step_ms * 1e-3) / 1e12}
    if spec.mode == "prefill":
        # the two halves of the layer alone: the fused indexer + top-k, then the attention on its selection
        bf16, kind = tensor_peaks()
        parts = {}
        for name, fn in (("indexer", wl.prefill_select), ("attention", wl.prefill_attend)):
            pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                pev[i][0].record(stream)
                fn()
                pev[i][1].record(stream)
            torch.cuda.synchronize()
            parts[name] = sum(a.elapsed_time(b) for a, b in pev) / args.steps
        assert wl.k.csa2_check(wl.err) == 0
        fp4 = pairs * 64 * 128 * 2 / (parts["indexer"] * 1e-3) / 1e12
        attn_flop = rows * 64 * (spec.k + 128) * 512 * 4
        bf = attn_flop / (parts["attention"] * 1e-3) / 1e12
        line["indexer_roofline"] = {"bound": "tensor", "kernel": "csa2 fused prefill indexer + top-k (FP4 MMA)",
                                    "achieved": fp4, "peak": 4 * bf16, "unit": "TFLOP/s", "frac": fp4 / (4 * bf16),
                                    "peak_kind": f"4 x {kind} dense bf16 (the nominal fp4 : bf16 ratio)",
                                    "ms": parts["indexer"]}
        line["attention_roofline"] = {"bound": "tensor", "kernel": "csa2 sparse attention + SWA + merge (kind::f16)",
                                      "achieved": bf, "peak": bf16, "unit": "TFLOP/s", "frac": bf / bf16,
                                      "peak_kind": f"{kind} dense bf16", "ms": parts["attention"],
                                      "flop_per_step": attn_flop}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_model40(args, spec, dev, world, rank):
    """One decode token of each sequence through the pages' 40-layer stack, one csa2_decode_step per
    step, replayed from a CUDA graph; its own JSON line (whole-model decode per token)."""
    wl = Model40(spec, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    graphs = not args.eager
    for i in range(args.warmup):
        wl.step(graphs=graphs and i > 0)
        if graphs and i == 0:
            wl.capture()
    torch.cuda.synchronize()
    assert wl.k.csa2_check(wl.err) == 0
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        wl.step(graphs=graphs)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, world)
    assert wl.k.csa2_check(wl.err) == 0
    recall = wl.reindex_recall()
    csa2_layers = sum(1 for m, _, _ in wl.plan if m != wl.k.LAYER_SWA)
    scanned = sum(wl.B * wl.max_entries[c] for c in range(len(wl.ratios)))
    line = {"metric": "decode tokens/s through the 40-layer CSA2 stack (one csa2_decode_step per token)",
            "value": world * wl.B / (step_ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0,1) latents, planted 2% cluster)",
            "config": {"workload": f"{spec.name}: batch {spec.B}, {spec.tokens[0]} tokens/seq, 40 layers "
                                   f"(2 SWA-only, 4 Full, 4 Reindex, 30 Reuse), caches at ratios {wl.ratios}",
                       "batch": spec.B, "ctx_tokens": spec.tokens[0], "top_k": spec.k, "pool_k": spec.pool_k,
                       "launch": "eager" if args.eager else "CUDA graph of csa2_decode_step",
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, outside step events)"},
            "query_tokens_per_s_per_csa2_layer": world * wl.B * csa2_layers / (step_ms * 1e-3),
            "full_scan_entries_per_step": scanned,
            "reindex_recall": {str(k): v for k, v in recall.items()},
            "gpu_launches": wl.launches_per_step() * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    import compressed_sparse_attention_score_b200  # noqa: F401  (fails loudly without the library)
    from workloads import configs as W
    dev = torch.device("cuda", torch.cuda.current_device())
    spec = W.CONFIGS[args.workload](seed=rank)
    if args.batch:
        spec = W.scaled(spec, spec.tokens[0], B=args.batch)
    if spec.name == "model40":
        run_model40(args, spec, dev, world, rank)
        return
    if spec.name in ("tiny_full", "reuse64k", "mixed64", "prefill8k"):
        run_one_layer(args, spec, dev, world, rank)
        return
    assert spec.name == "hier1m", "bench.py times the hierarchical 1M-context decode workload"
    wl = Hier1M(spec, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    graphs = not args.eager
    for i in range(args.warmup):
        wl.step(graphs=graphs and i > 0)
        if graphs and i == 0:
            wl.capture()
    torch.cuda.synchronize()
    assert wl.k.csa2_check(wl.err) == 0

    # ---- device-resident timing
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        wl.step(scan_events=sev[i], graphs=graphs)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    scan_ms = sum(a.elapsed_time(b) for a, b in sev) / args.steps
    step_ms = max_over_ranks(step_ms, world)
    units = world * wl.B * wl.LAYERS
    value = units / (step_ms * 1e-3)

    # ---- end to end through the C ABI with host buffers
    ins, h_in, outs, h_out = wl.host_io()
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        eev[i][0].record(stream)
        for d, h in zip(ins, h_in):
            d.copy_(h, non_blocking=True)
        wl.step(graphs=graphs)
        for h, d in zip(h_out, outs):
            h.copy_(d, non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_serial_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eev) / args.steps, world)
    # ---- end to end, pipelined: step i's inputs are copied in (pinned host -> device, one copy stream)
    # while step i - 1 computes, and its outputs copied out (another copy stream) while step i + 1
    # computes; inputs and outputs double-buffered.  Timed from the first input copy to the last output
    # copy, divided by the steps.  No L2 flush: every step scans the 2.8 GB cache, far more than L2.
    wl.make_buffer_sets(graphs)
    h_outs = [h_out, [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined(n):
        h2d_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        d2h_done = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def copy_in(i):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])       # this buffer set's inputs are no longer read
                for d, h in zip(wl.set_io(i % 2)[0], h_in):
                    d.copy_(h, non_blocking=True)
                h2d_done[i].record(s_in)

        t0.record(s_in)
        copy_in(0)
        if n > 1:
            copy_in(1)
        for i in range(n):
            comp.wait_event(h2d_done[i])
            if i >= 2:
                comp.wait_event(d2h_done[i - 2])             # this buffer set's outputs have been read back
            wl.use_set(i % 2)
            wl.step(graphs=graphs)
            comp_done[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                for h, d in zip(h_outs[i % 2], wl.set_io(i % 2)[1]):
                    h.copy_(d, non_blocking=True)
                d2h_done[i].record(s_out)
            if i + 2 < n:
                copy_in(i + 2)
        s_out.wait_event(d2h_done[n - 1])
        t1.record(s_out)
        torch.cuda.synchronize()
        wl.use_set(0)
        return t0.elapsed_time(t1) / n

    pipelined(max(2, args.warmup))
    barrier(world)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(pipelined(args.steps), world)
    # the same end-to-end steps with every call made through the C ABI from Python (no graph replay)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        eev[i][0].record(stream)
        for d, h in zip(ins, h_in):
            d.copy_(h, non_blocking=True)
        wl.step(graphs=False)
        for h, d in zip(h_out, outs):
            h.copy_(d, non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_eager_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eev) / args.steps, world)
    # the gather: a Reindex layer's attention launch (512 listed entries + 128 window tokens per row)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        gev[i][0].record(stream)
        wl.attention(1)
        gev[i][1].record(stream)
    torch.cuda.synchronize()
    gather_ms = sum(a.elapsed_time(b) for a, b in gev) / args.steps
    assert wl.k.csa2_check(wl.err) == 0

    peak, peak_kind = peaks()
    gather_gbs = wl.gather_bytes() / (gather_ms * 1e-3) / 1e9
    gather = {"kernel": "csa2 sparse attention + SWA + merge (one layer, one launch)",
              "bytes_per_launch": wl.gather_bytes(), "achieved": gather_gbs, "peak": peak, "peak_kind": peak_kind,
              "unit": "GB/s", "frac": gather_gbs / peak, "launch_us": gather_ms * 1e3,
              "timing": "isolated launches, L2 flushed before each"}
    achieved = wl.scan_bytes() / (scan_ms * 1e-3) / 1e9
    traffic = profiled_traffic(["compressed_sparse_attention_score_b200/csrc/" + f
                                for f in ("index_mma.cu", "sm100.cuh", "common.cuh")], "index_score_hier1m.md")
    # context for the scan's fraction: a plain read-only stream over as many bytes (torch's sum
    # reduction over the same 570 MB), timed the same way (L2 flushed, CUDA events)
    stream_buf = torch.empty(wl.scan_bytes() // 4, dtype=torch.float32, device=dev).fill_(1.0)
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
    stream_buf.sum()
    for a, b in rev:
        flush.zero_()
        a.record(stream)
        stream_buf.sum()
        b.record(stream)
    torch.cuda.synchronize()
    read_ms = sorted(a.elapsed_time(b) for a, b in rev)[2]
    read_gbs = wl.scan_bytes() / (read_ms * 1e-3) / 1e9
    del stream_buf
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0,1) latents and queries)",
            "config": dict(config_dict(spec), launch="eager" if args.eager else
                           "CUDA graphs of the step around an eagerly launched Full-layer scan"),
            "roofline": {"bound": "hbm", "kernel": "csa2 indexer scan (Full layer)", "achieved": achieved,
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "scan_ms": scan_ms,
                         "entries_scanned_per_s": wl.B * wl.N / (scan_ms * 1e-3),
                         "read_stream": {"kernel": "torch sum over the same bytes (context, not the peak)",
                                         "GBps": read_gbs, "scan_frac_of_it": achieved / read_gbs}},
            "gather": gather,
            "e2e": {"value": units / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "copies": "overlapped with the neighbouring steps' compute (two copy streams, inputs and "
                              "outputs double-buffered); timed from the first input copy to the last output copy"},
            "e2e_serial": {"value": units / (e2e_serial_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_serial_ms,
                           "copies": "inputs in, step, outputs out, one stream, per-step events"},
            "e2e_eager": {"value": units / (e2e_eager_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                          "d2h_bytes_per_step": d2h, "ms_per_step": e2e_eager_ms,
                          "launch": "every call through the C ABI from Python, no graph replay"},
            "gpu_launches": wl.launches_per_step() * args.steps,
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del wl
        torch.cuda.empty_cache()
        dt, cores = oracle_time(spec, args.cpu_sample_seqs)
        line["cpu_baseline"] = {"value": args.cpu_sample_seqs * 5 / dt, "unit": UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"{args.cpu_sample_seqs} of {spec.B} sequences, one decode step "
                                          f"through all 5 layers (Full scan of {spec.entries(0)} keys)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
