"""ctypes binding of libcsa2.so: argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
CUDA tensors (or None for NULL) and raises RuntimeError when the call returns a
non-zero csa2_status.  All arithmetic happens in the library's CUDA kernels;
there is no CPU fallback: without the built library, importing this module fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m compressed_sparse_attention_score_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

MODE = {"full": 0, "reindex": 1, "reuse": 2, "dense": 3}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
STATUS = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "UNSUPPORTED", 4: "CUDA", 5: "INDEX", 6: "TIMEOUT"}

MAIN_DIM, MAIN_CODE_BYTES, MAIN_SCALE_BYTES = 512, 256, 32
IX_DIM, IX_CODE_BYTES, IX_SCALE_BYTES = 128, 64, 4
HEADS = IX_HEADS = 64

c_void_p, c_int32, c_int64, c_size_t, c_float = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                                   ctypes.c_size_t, ctypes.c_float)


class csa2_cache(ctypes.Structure):
    _fields_ = [("kv_codes", c_void_p), ("kv_scales", c_void_p), ("ix_codes", c_void_p),
                ("ix_scales", c_void_p), ("page_table", c_void_p), ("num_entries", c_void_p),
                ("num_slots", c_int64), ("batch", c_int32), ("ratio", c_int32),
                ("seq_stride", c_int32), ("page_size", c_int32), ("max_pages", c_int32)]


class csa2_layer_plan(ctypes.Structure):
    _fields_ = [("mode", c_int32), ("source", c_int32), ("cache", c_int32)]


class csa2_decode_args(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("plan", c_void_p), ("n_caches", c_int32), ("caches", c_void_p),
                ("max_entries", c_void_p), ("B", c_int32), ("pos", c_void_p), ("softmax_scale", c_float),
                ("k", c_int32), ("pool_k", c_int32), ("q", c_void_p), ("q_ix", c_void_p), ("w", c_void_p),
                ("new_kv", c_void_p), ("new_ix", c_void_p), ("kv_stage", c_void_p), ("swa_x", c_void_p),
                ("swa_codes", c_void_p), ("swa_scale", c_void_p), ("R", c_int32), ("window", c_int32),
                ("idx", c_void_p), ("pool", c_void_p), ("o", c_void_p), ("lse", c_void_p)]


LAYER_SWA = 4
_P = ctypes.POINTER(csa2_cache)
_PD = ctypes.POINTER(csa2_decode_args)
_SIGS = {
    "csa2_version": ([], ctypes.c_int),
    "csa2_last_error_string": ([], ctypes.c_char_p),
    "csa2_check": ([c_void_p, c_void_p], ctypes.c_int),
    "csa2_workspace_size": ([ctypes.c_int, c_int32, c_int32, c_int32, c_int32, c_int32], c_size_t),
    "csa2_pack_kv": ([c_void_p, c_void_p, ctypes.c_int, c_void_p, c_int32, c_int32, c_void_p, _P,
                      c_void_p, c_void_p], ctypes.c_int),
    "csa2_pack_swa": ([c_void_p, ctypes.c_int, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32,
                       c_void_p, c_void_p], ctypes.c_int),
    "csa2_index_score": ([c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_int32, c_int32, _P,
                          c_void_p, c_void_p, c_void_p], ctypes.c_int),
    "csa2_topk": ([c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_int32, c_void_p,
                   c_void_p, c_void_p], ctypes.c_int),
    "csa2_sparse_attn": ([ctypes.c_int, c_void_p, c_int32, c_int32, c_void_p, c_float, c_void_p, c_void_p,
                          c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, _P, c_void_p, c_void_p, c_int32,
                          c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p],
                         ctypes.c_int),
    "csa2_swa_attn": ([c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_float,
                       c_void_p, c_void_p, c_void_p, c_void_p], ctypes.c_int),
    "csa2_merge": ([c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p],
                   ctypes.c_int),
    "csa2_noalloc_scratch_bytes": ([], c_size_t),
    "csa2_sparse_attn_noalloc": ([ctypes.c_int, c_void_p, c_int32, c_int32, c_void_p, c_float, c_void_p, c_void_p,
                                  c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, _P, c_void_p, c_void_p,
                                  c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_void_p], ctypes.c_int),
    "csa2_append_kv": ([c_void_p, c_void_p, ctypes.c_int, c_int32, c_void_p, c_void_p, _P, c_void_p, c_void_p],
                       ctypes.c_int),
    "csa2_plan_v41": ([c_void_p, c_int32, c_void_p], c_int32),
    "csa2_index_topk": ([c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_int32, c_int32, _P, c_void_p, c_void_p,
                         c_void_p], ctypes.c_int),
    "csa2_pack_kv_gated": ([c_void_p, c_void_p, ctypes.c_int, c_void_p, c_void_p, c_int32, c_int32, c_void_p, _P,
                           c_void_p, c_void_p], ctypes.c_int),
    "csa2_decode_workspace_size": ([_PD], c_size_t),
    "csa2_decode_step": ([_PD, c_void_p, c_size_t, c_void_p, c_void_p], ctypes.c_int),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes, _f.restype = _args, _ret

EXPORTED = tuple(_SIGS)


def raw():
    """The ctypes library handle (for tests of the bare C ABI)."""
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("CSA2 tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("CSA2 tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ok(status, what):
    if status != 0:
        msg = _lib.csa2_last_error_string().decode()
        raise RuntimeError(f"{what} -> CSA2_{STATUS.get(status, status)}: {msg}")


class GlobalKVCache:
    """Caller-owned device planes of the shared global KV cache plus its descriptor.

    Contiguous: slot = b * seq_stride + n.  Paged: page_table [batch][max_pages]
    maps entry pages of page_size entries to physical pages.  Planes may be shared
    between several views (e.g. two page tables into one physical pool).
    """

    def __init__(self, batch, ratio, seq_stride=None, num_slots=None, page_table=None, page_size=256,
                 device="cuda", planes=None, num_entries=None):
        self.batch, self.ratio = int(batch), int(ratio)
        self.page_table = page_table
        if page_table is None:
            assert seq_stride is not None
            self.seq_stride, self.page_size, self.max_pages = int(seq_stride), 0, 0
            num_slots = batch * seq_stride if num_slots is None else num_slots
        else:
            assert num_slots is not None and page_table.dtype == torch.int32
            self.seq_stride, self.page_size, self.max_pages = 0, int(page_size), int(page_table.shape[1])
        self.num_slots = int(num_slots)
        if planes is None:
            planes = (torch.zeros((self.num_slots, MAIN_CODE_BYTES), dtype=torch.uint8, device=device),
                      torch.zeros((self.num_slots, MAIN_SCALE_BYTES), dtype=torch.uint8, device=device),
                      torch.zeros((self.num_slots, IX_CODE_BYTES), dtype=torch.uint8, device=device),
                      torch.zeros((self.num_slots, IX_SCALE_BYTES), dtype=torch.uint8, device=device))
        self.kv_codes, self.kv_scales, self.ix_codes, self.ix_scales = planes
        self.num_entries = (torch.zeros(batch, dtype=torch.int32, device=device)
                            if num_entries is None else num_entries)

    def seq_view(self, b):
        """A one-sequence descriptor over the same memory (sequence b becomes sequence 0)."""
        if self.page_table is None:
            sl = slice(b * self.seq_stride, (b + 1) * self.seq_stride)
            return GlobalKVCache(1, self.ratio, seq_stride=self.seq_stride, num_slots=self.seq_stride,
                                 planes=tuple(p[sl] for p in self.planes), num_entries=self.num_entries[b:b + 1])
        return GlobalKVCache(1, self.ratio, num_slots=self.num_slots, page_table=self.page_table[b:b + 1],
                             page_size=self.page_size, planes=self.planes, num_entries=self.num_entries[b:b + 1])

    @property
    def planes(self):
        return (self.kv_codes, self.kv_scales, self.ix_codes, self.ix_scales)

    def desc(self):
        d = csa2_cache()
        d.kv_codes, d.kv_scales = _ptr(self.kv_codes), _ptr(self.kv_scales)
        d.ix_codes, d.ix_scales = _ptr(self.ix_codes), _ptr(self.ix_scales)
        d.page_table = _ptr(self.page_table)
        d.num_entries = _ptr(self.num_entries)
        d.num_slots, d.batch, d.ratio = self.num_slots, self.batch, self.ratio
        d.seq_stride, d.page_size, d.max_pages = self.seq_stride, self.page_size, self.max_pages
        return d


def csa2_version():
    return _lib.csa2_version()


def csa2_check(err, stream=None):
    return _lib.csa2_check(_ptr(err), _stream(stream))


def csa2_workspace_size(mode, B, Q, max_entries, k, pool_k=0):
    return _lib.csa2_workspace_size(MODE[mode], B, Q, max_entries, k, pool_k)


def csa2_pack_kv(lat_kv, lat_ix, first_entry, cache, pool_w=None, err=None, stream=None):
    B, T = lat_kv.shape[0], lat_kv.shape[1]
    assert lat_kv.shape[2] == MAIN_DIM and lat_ix.shape == (B, T, IX_DIM) and lat_ix.dtype == lat_kv.dtype
    d = cache.desc()
    _ok(_lib.csa2_pack_kv(_ptr(lat_kv), _ptr(lat_ix), DTYPE[lat_kv.dtype], _ptr(pool_w), B, T,
                          _ptr(first_entry), ctypes.byref(d), _ptr(err), _stream(stream)), "csa2_pack_kv")


def csa2_pack_swa(x, pos, swa_codes, swa_scale, err=None, stream=None):
    B, T = x.shape[0], x.shape[1]
    R = swa_codes.shape[1]
    _ok(_lib.csa2_pack_swa(_ptr(x), DTYPE[x.dtype], B, T, _ptr(pos), _ptr(swa_codes), _ptr(swa_scale), R,
                           _ptr(err), _stream(stream)), "csa2_pack_swa")


def csa2_index_score(q_ix, w, q_pos, cache, max_entries, cand=None, scores=None, err=None, stream=None):
    B, Q = q_ix.shape[0], q_ix.shape[1]
    P = 0 if cand is None else cand.shape[-1]
    n_out = P if cand is not None else max_entries
    if scores is None:
        scores = torch.empty((B, Q, n_out), dtype=torch.float32, device=q_ix.device)
    d = cache.desc()
    _ok(_lib.csa2_index_score(_ptr(q_ix), _ptr(w), B, Q, _ptr(q_pos), _ptr(cand), P, max_entries,
                              ctypes.byref(d), _ptr(scores), _ptr(err), _stream(stream)), "csa2_index_score")
    return scores


def csa2_topk(scores, k, n_valid=None, idx=None, val=None, k2=0, idx2=None, val2=None, stream=None):
    """Top-k positions of each row (and optionally a second top-k2 selection in the same pass)."""
    N = scores.shape[-1]
    R = scores.numel() // N if N else 0
    if idx is None:
        idx = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    if k2 and idx2 is None:
        idx2 = torch.empty(scores.shape[:-1] + (k2,), dtype=torch.int32, device=scores.device)
    _ok(_lib.csa2_topk(_ptr(scores), _ptr(n_valid), R, N, k, _ptr(idx), _ptr(val), k2, _ptr(idx2), _ptr(val2),
                       _stream(stream)), "csa2_topk")
    return (idx, val) if not k2 else (idx, val, idx2, val2)


def csa2_sparse_attn(mode, q, q_pos, cache, softmax_scale, max_entries, k=512, q_ix=None, w=None, pool_k=0,
                     pool_io=None, idx_in=None, idx_out=None, o=None, lse=None, ws=None, err=None, stream=None,
                     swa_codes=None, swa_scale=None, window=128, swa_new=None):
    """One layer's sparse branch; with swa_codes/swa_scale the SWA window joins the same softmax (merged).
    swa_new [B][1][512] bf16 (decode): this step's window token, quantised into the ring in the same launch."""
    B, Q = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty((B, Q, HEADS, MAIN_DIM), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Q, HEADS), dtype=torch.float32, device=q.device)
    if ws is None:
        nbytes = csa2_workspace_size(mode, B, Q, max_entries, k, pool_k)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device) if nbytes else None
    d = cache.desc()
    R = 0 if swa_codes is None else swa_codes.shape[1]
    _ok(_lib.csa2_sparse_attn(MODE[mode], _ptr(q), B, Q, _ptr(q_pos), float(softmax_scale), _ptr(q_ix), _ptr(w),
                              k, pool_k, _ptr(pool_io), _ptr(idx_in), _ptr(idx_out), max_entries, ctypes.byref(d),
                              _ptr(swa_codes), _ptr(swa_scale), R, window, _ptr(swa_new), _ptr(o), _ptr(lse),
                              _ptr(ws), 0 if ws is None else ws.numel(), _ptr(err), _stream(stream)),
        "csa2_sparse_attn")
    return o, lse


def csa2_sparse_attn_noalloc(mode, q, q_pos, cache, softmax_scale, max_entries, k=512, q_ix=None, w=None,
                             pool_k=0, pool_io=None, idx_in=None, idx_out=None, o=None, lse=None, err=None,
                             stream=None, swa_codes=None, swa_scale=None, window=128):
    """csa2_sparse_attn using the library's fixed scratch instead of a workspace (see csa2.h)."""
    B, Q = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty((B, Q, HEADS, MAIN_DIM), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Q, HEADS), dtype=torch.float32, device=q.device)
    d = cache.desc()
    R = 0 if swa_codes is None else swa_codes.shape[1]
    _ok(_lib.csa2_sparse_attn_noalloc(MODE[mode], _ptr(q), B, Q, _ptr(q_pos), float(softmax_scale), _ptr(q_ix),
                                      _ptr(w), k, pool_k, _ptr(pool_io), _ptr(idx_in), _ptr(idx_out), max_entries,
                                      ctypes.byref(d), _ptr(swa_codes), _ptr(swa_scale), R, window, _ptr(o),
                                      _ptr(lse), _ptr(err), _stream(stream)), "csa2_sparse_attn_noalloc")
    return o, lse


def csa2_swa_attn(q, q_pos, swa_codes, swa_scale, softmax_scale, window=128, o=None, lse=None, err=None,
                  stream=None):
    B, Q = q.shape[0], q.shape[1]
    R = swa_codes.shape[1]
    if o is None:
        o = torch.empty((B, Q, HEADS, MAIN_DIM), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Q, HEADS), dtype=torch.float32, device=q.device)
    _ok(_lib.csa2_swa_attn(_ptr(q), B, Q, _ptr(q_pos), _ptr(swa_codes), _ptr(swa_scale), R, window,
                           float(softmax_scale), _ptr(o), _ptr(lse), _ptr(err), _stream(stream)), "csa2_swa_attn")
    return o, lse


def csa2_merge(o1, l1, o2, l2, o=None, lse=None, stream=None):
    D = o1.shape[-1]
    rows = l1.numel()
    if o is None:
        o = torch.empty_like(o1)
    if lse is None:
        lse = torch.empty_like(l1)
    _ok(_lib.csa2_merge(_ptr(o1), _ptr(l1), _ptr(o2), _ptr(l2), rows, D, _ptr(o), _ptr(lse), _stream(stream)),
        "csa2_merge")
    return o, lse


def csa2_append_kv(lat_kv, lat_ix, pos, cache, stage=None, err=None, stream=None):
    """Append one token per sequence (lat_kv [B][512], lat_ix [B][128]) at positions pos [B]."""
    B = lat_kv.shape[0]
    assert lat_kv.shape[-1] == MAIN_DIM and lat_ix.shape[-1] == IX_DIM and lat_ix.dtype == lat_kv.dtype
    d = cache.desc()
    _ok(_lib.csa2_append_kv(_ptr(lat_kv), _ptr(lat_ix), DTYPE[lat_kv.dtype], B, _ptr(pos), _ptr(stage),
                            ctypes.byref(d), _ptr(err), _stream(stream)), "csa2_append_kv")


def csa2_index_topk(q_ix, w, q_pos, cache, max_entries, k=512, idx=None, err=None, stream=None):
    """Full-mode selection of every query row (fused indexer + top-k, no scores kept): idx [B][Q][k]."""
    B, Q = q_ix.shape[0], q_ix.shape[1]
    if idx is None:
        idx = torch.empty((B, Q, k), dtype=torch.int32, device=q_ix.device)
    d = cache.desc()
    _ok(_lib.csa2_index_topk(_ptr(q_ix), _ptr(w), B, Q, _ptr(q_pos), k, max_entries, ctypes.byref(d), _ptr(idx),
                             _ptr(err), _stream(stream)), "csa2_index_topk")
    return idx


def csa2_pack_kv_gated(lat_kv, lat_ix, gate_kv, gate_ix, first_entry, cache, err=None, stream=None):
    """csa2_pack_kv with per-channel softmax gates over each entry's tokens (gate_* fp32, shaped like lat_*)."""
    B, T = lat_kv.shape[0], lat_kv.shape[1]
    assert gate_kv.shape == lat_kv.shape and gate_ix.shape == lat_ix.shape and gate_kv.dtype == torch.float32
    d = cache.desc()
    _ok(_lib.csa2_pack_kv_gated(_ptr(lat_kv), _ptr(lat_ix), DTYPE[lat_kv.dtype], _ptr(gate_kv), _ptr(gate_ix), B, T,
                                _ptr(first_entry), ctypes.byref(d), _ptr(err), _stream(stream)),
        "csa2_pack_kv_gated")


def csa2_plan_v41():
    """The pages' 40-layer plan: ([(mode, source, cache)] * 40, ratios of its 4 caches)."""
    n = _lib.csa2_plan_v41(None, 0, None)
    plan = (csa2_layer_plan * n)()
    ratios = (c_int32 * 4)()
    assert _lib.csa2_plan_v41(plan, n, ratios) == n
    return [(p.mode, p.source, p.cache) for p in plan], list(ratios)


class DecodeStep:
    """Descriptor of csa2_decode_step over caller-owned device tensors (marshalling only).

    plan: [(mode, source, cache)] per layer (mode: a MODE value or LAYER_SWA); caches: GlobalKVCache
    per cache id; max_entries: per cache.  Tensors are layer-major as csa2.h describes.
    """

    def __init__(self, plan, caches, max_entries, pos, softmax_scale, k, pool_k, q, swa_x, swa_codes, swa_scale,
                 idx, o, lse, q_ix=None, w=None, pool=None, new_kv=None, new_ix=None, kv_stage=None, window=128):
        L, nc = len(plan), len(caches)
        self._plan = (csa2_layer_plan * L)(*[csa2_layer_plan(*p) for p in plan])
        self._caches = (csa2_cache * max(nc, 1))(*[c.desc() for c in caches])
        self._maxe = (c_int32 * max(nc, 1))(*max_entries)
        self._keep = (caches, pos, q, swa_x, swa_codes, swa_scale, idx, o, lse, q_ix, w, pool, new_kv, new_ix, kv_stage)
        a = csa2_decode_args()
        a.n_layers, a.plan = L, ctypes.addressof(self._plan)
        a.n_caches, a.caches, a.max_entries = nc, ctypes.addressof(self._caches), ctypes.addressof(self._maxe)
        a.B, a.pos, a.softmax_scale, a.k, a.pool_k = q.shape[1], _ptr(pos), float(softmax_scale), k, pool_k
        a.q, a.q_ix, a.w = _ptr(q), _ptr(q_ix), _ptr(w)
        a.new_kv, a.new_ix, a.kv_stage = _ptr(new_kv), _ptr(new_ix), _ptr(kv_stage)
        a.swa_x, a.swa_codes, a.swa_scale = _ptr(swa_x), _ptr(swa_codes), _ptr(swa_scale)
        a.R, a.window = swa_codes.shape[2], window
        a.idx, a.pool, a.o, a.lse = _ptr(idx), _ptr(pool), _ptr(o), _ptr(lse)
        self.args = a

    def workspace_size(self):
        return _lib.csa2_decode_workspace_size(ctypes.byref(self.args))

    def run(self, ws, err=None, stream=None):
        _ok(_lib.csa2_decode_step(ctypes.byref(self.args), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(err),
                                  _stream(stream)), "csa2_decode_step")
