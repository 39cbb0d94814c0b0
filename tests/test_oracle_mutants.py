"""Plant plausible mistakes in the oracle (on the CPU, by monkeypatching) and
check that at least one pin fails for each: the pins are strong enough to
trust the oracle as the parity reference."""

import numpy as np
import pytest

from oracle import attention, codecs
from tests import test_oracle_attention as ta
from tests import test_oracle_codecs as tc


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_dropped_softmax_scale_is_caught(monkeypatch):
    def mutant(q, K, V, scale):
        x = K @ q
        w = np.exp(x - np.max(x)) if len(x) else x
        return (w @ V) / np.sum(w) if len(x) else np.zeros(V.shape[1])
    monkeypatch.setattr(attention, "softmax_weighted_sum", mutant)
    assert _fails(ta.test_paged_equals_contiguous_brute_force, 1)


def test_scores_against_values_is_caught(monkeypatch):
    orig = attention.softmax_weighted_sum
    monkeypatch.setattr(attention, "softmax_weighted_sum", lambda q, K, V, s: orig(q, V, V, s))
    assert _fails(ta.test_paged_equals_contiguous_brute_force, 1)


def test_interleaved_gqa_mapping_is_caught(monkeypatch):
    orig = attention.gather_sequence

    def paged_mutant(q, k_cache, v_cache, block_tables, context_lens, scale, heads=None):
        S, Hq, D = q.shape
        Hkv = k_cache.shape[1]
        out = np.zeros((S, Hq, D))
        for s in range(S):
            for h in range(Hq):
                g = h % Hkv                      # wrong grouping
                L = int(context_lens[s])
                K = orig(k_cache, block_tables[s], L, g)
                V = orig(v_cache, block_tables[s], L, g)
                out[s, h] = attention.softmax_weighted_sum(q[s, h], K, V, scale)
        return out
    monkeypatch.setattr(attention, "paged_decode_f64", paged_mutant)
    assert _fails(ta.test_paged_equals_contiguous_brute_force, 2)


def test_wrong_in_block_offset_is_caught(monkeypatch):
    def mutant(cache, row, L, g):
        bs = cache.shape[2]
        rows = [cache[int(row[j // bs]), g, (bs - 1 - j % bs), :] for j in range(L)]
        return np.stack(rows) if rows else np.zeros((0, cache.shape[3]))
    monkeypatch.setattr(attention, "gather_sequence", mutant)
    assert _fails(ta.test_page1_block_table_gather_order)


def test_wrong_e4m3_bias_is_caught(monkeypatch):
    monkeypatch.setattr(codecs, "decode_e4m3",
                        lambda c: codecs._decode_binary(c, 4, 3, 8, False, True))
    assert _fails(tc.test_e4m3_every_code_matches_torch)


def test_truncating_encoder_is_caught(monkeypatch):
    orig_rint = np.rint
    monkeypatch.setattr(codecs.np, "rint", np.floor)
    try:
        assert _fails(tc.test_e4m3_encode_ties_go_to_even)
    finally:
        monkeypatch.setattr(codecs.np, "rint", orig_rint)
