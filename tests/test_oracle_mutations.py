"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

A pin that still passes with the mistake in place would not be pinning anything.
"""
import numpy as np
import pytest

from oracle import csa2 as C
from oracle import formats as F
import tests.test_oracle_formats as TF
import tests.test_oracle_method as TM


def _fails(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_relu_dropped_is_caught(monkeypatch):
    def no_relu(q_ix, w, keys):
        qh = C.quantised_query(q_ix)
        return (np.asarray(keys, np.float64) @ qh.T) @ np.asarray(w, np.float64)
    monkeypatch.setattr(C, "indexer_scores", no_relu)
    _fails(TM.test_indexer_score_brute_force)


def test_query_left_unquantised_is_caught(monkeypatch):
    monkeypatch.setattr(C, "quantised_query", lambda q: np.asarray(q, np.float64))
    _fails(TM.test_indexer_query_is_mxfp4_quantised)


def test_nibble_order_swapped_is_caught(monkeypatch):
    monkeypatch.setattr(F, "pack_nibbles", lambda c: (np.asarray(c)[..., 1::2] | (np.asarray(c)[..., 0::2] << 4)).astype(np.uint8))
    _fails(TF.test_nibble_order_low_first)


def test_e2m1_ties_away_from_zero_is_caught(monkeypatch):
    def away(y):
        y = np.asarray(y, np.float32)
        m = np.abs(y)
        idx = np.zeros(m.shape, np.uint8)
        for p in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            idx += m >= p
        neg = np.signbit(y) & (idx > 0)
        return (idx | (neg.astype(np.uint8) << 3)).astype(np.uint8)
    monkeypatch.setattr(F, "e2m1_encode", away)
    _fails(TF.test_e2m1_grid_and_ties_brute_force)


def test_e4m3_truncation_is_caught(monkeypatch):
    orig = F.e4m3_encode

    def trunc(v):
        v = np.asarray(v, np.float32)
        c = orig(v)
        back = F.e4m3_decode(c)
        too_big = np.abs(back) > np.abs(v.astype(np.float64))
        return np.where(too_big & ((c & 0x7F) > 0), c - 1, c).astype(np.uint8)
    monkeypatch.setattr(F, "e4m3_encode", trunc)
    _fails(TF.test_e4m3_against_torch_cast)


def test_floor_exponent_is_caught(monkeypatch):
    monkeypatch.setattr(F, "e8m0_ceil_exponent",
                        lambda q: np.clip(np.floor(np.log2(np.asarray(q, np.float64))), -127, 127).astype(np.int64))
    _fails(TF.test_e8m0_ceil_exponent_brute_force)


def test_topk_tie_to_higher_index_is_caught(monkeypatch):
    def bad(scores, k, n_valid=None):
        s = np.asarray(scores, np.float64)
        n = len(s) if n_valid is None else min(int(n_valid), len(s))
        pos = np.arange(n)
        pos = pos[s[:n] != -np.inf]
        order = pos[np.lexsort((-pos, -s[pos]))]
        sel = np.sort(order[:k])
        out = np.full(k, -1, np.int64)
        out[:len(sel)] = sel
        return out
    monkeypatch.setattr(C, "topk", bad)
    _fails(TM.test_topk_against_rank_definition, 0)


def test_missing_softmax_scale_is_caught(monkeypatch):
    orig = C.attend
    monkeypatch.setattr(C, "attend", lambda q, keys, tau: orig(q, keys, 1.0))
    _fails(TM.test_attend_brute_force)


def test_merge_weight_swapped_is_caught(monkeypatch):
    orig = C.merge
    monkeypatch.setattr(C, "merge", lambda o1, l1, o2, l2: orig(o1, l2, o2, l1))
    _fails(TM.test_merge_equals_one_softmax_over_union)


def test_off_by_one_visibility_is_caught(monkeypatch):
    monkeypatch.setattr(C.Cache, "visible", lambda self, b, pos: int(min(self.num_entries[b], pos // self.ratio + 1)))
    _fails(TM.test_full_respects_causality)


def test_swa_window_off_by_one_is_caught(monkeypatch):
    def bad(q, pos, codes, scale, window, tau):
        R = codes.shape[0]
        slots = np.arange(max(0, pos - window), pos + 1) % R
        return C.attend(q, F.unpack_swa(codes[slots], scale[slots]), tau)
    monkeypatch.setattr(C, "swa_attention", bad)
    _fails(TM.test_swa_equals_dense_over_last_window)


def test_layer_without_its_window_branch_is_caught(monkeypatch):
    orig = C.swa_attention
    monkeypatch.setattr(C, "swa_attention",
                        lambda q, pos, codes, scale, window, tau: C.attend(q, np.zeros((0, 512)), tau))
    _fails(TM.test_decode_layer_is_one_softmax_over_entries_and_window, "reuse")
    monkeypatch.setattr(C, "swa_attention", orig)


def test_layer_with_the_default_window_is_caught(monkeypatch):
    orig = C.swa_attention
    monkeypatch.setattr(C, "swa_attention",
                        lambda q, pos, codes, scale, window, tau: orig(q, pos, codes, scale, 128, tau))
    _fails(TM.test_decode_layer_is_one_softmax_over_entries_and_window, "full")


def test_gate_softmax_over_channels_is_caught(monkeypatch):
    def over_channels(lat, gate, ratio):
        lat, gate = np.asarray(lat, np.float32), np.asarray(gate, np.float32)
        n = lat.shape[0] // ratio
        out = np.empty((n,) + lat.shape[1:], np.float32)
        for j in range(n):
            g = gate[j * ratio:(j + 1) * ratio]
            e = C.exp_fp32((g - g.max(axis=1, keepdims=True)).astype(np.float32))
            w = (e / e.sum(axis=1, keepdims=True)).astype(np.float32)
            out[j] = (w * lat[j * ratio:(j + 1) * ratio]).sum(axis=0).astype(np.float32)
        return out
    monkeypatch.setattr(C, "compress_gated", over_channels)
    _fails(TM.test_gated_compressor_reductions)


def test_stack_reusing_the_wrong_layer_is_caught(monkeypatch):
    orig = C.decode_layer

    def first_full(mode, cache, b, pos, q, tau, swa, window=128, **kw):
        if mode == "reuse" and "idx" in kw:   # every Reuse layer takes layer 2's entries instead
            kw["idx"] = first_full.layer2
        r = orig(mode, cache, b, pos, q, tau, swa, window, **kw)
        if mode == "full" and not hasattr(first_full, "layer2"):
            first_full.layer2 = r["idx"]
        return r
    monkeypatch.setattr(C, "decode_layer", first_full)
    _fails(TM.test_decode_model_follows_the_layer_schedule)


def test_stack_without_the_decoder_pool_is_caught(monkeypatch):
    monkeypatch.setattr(C, "pool_layer", lambda: 2)
    with pytest.raises((AssertionError, TypeError, IndexError)):
        TM.test_decode_model_follows_the_layer_schedule()


def test_layer_that_skips_its_listed_entries_is_caught(monkeypatch):
    monkeypatch.setattr(C, "sparse_attention", lambda cache, b, q, idx, tau: C.attend(q, np.zeros((0, 512)), tau))
    _fails(TM.test_decode_layer_is_one_softmax_over_entries_and_window, "reindex")
