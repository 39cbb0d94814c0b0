"""Plant plausible mistakes in the oracle (on the CPU, by monkeypatching) and
check that at least one pin fails for each: the pins are strong enough to
trust the oracle as the parity reference. Covered: decode attention, codecs,
multi-query (extend / prefill) attention, the block pool with copy-on-write,
beam re-selection and the prefix cache."""

import numpy as np
import pytest

from oracle import attention, codecs
from oracle import pool as opool
from oracle.pool import BlockPool, PoolError
from oracle.prefix_cache import PrefixCache
from tests import test_beam as tb
from tests import test_oracle_attention as ta
from tests import test_oracle_codecs as tc
from tests import test_oracle_extend as te
from tests import test_oracle_pool as tp
from tests import test_prefix_cache as tpc


def _fails(fn, *args):
    """A pin catches a mutant by failing an assertion or by the pool refusing a state."""
    try:
        fn(*args)
    except (AssertionError, PoolError):
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


def test_softmax_without_the_maximum_subtracted_is_caught(monkeypatch):
    def mutant(q, K, V, scale):
        if K.shape[0] == 0:
            return np.zeros(V.shape[1])
        with np.errstate(over="ignore", invalid="ignore"):
            w = np.exp(scale * (K @ q))                 # overflows for large scores
            return (w @ V) / np.sum(w)
    monkeypatch.setattr(attention, "softmax_weighted_sum", mutant)
    assert _fails(ta.test_huge_scores_stay_finite)


def test_wrong_bf16_bias_is_caught(monkeypatch):
    monkeypatch.setattr(codecs, "decode_bf16", lambda c: codecs._decode_binary(c, 8, 7, 126, True))
    assert _fails(tc.test_bf16_every_code_matches_torch)


def test_e4m3_read_with_ieee_specials_is_caught(monkeypatch):
    # the all-ones exponent as inf / NaN (E4M3 keeps 256..448 there and has no inf)
    monkeypatch.setattr(codecs, "decode_e4m3", lambda c: codecs._decode_binary(c, 4, 3, 7, True))
    assert _fails(tc.test_e4m3_every_code_matches_torch)


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


# ---- multi-query (extend / prefill) attention --------------------------------------

def _extend_mutant(visible):
    """paged_extend with the number of context tokens a query sees given by
    visible(L, Q, i) instead of L - Q + i + 1."""
    def mutant(q_codes, q_dtype, k_codes, v_codes, kv_dtype, k_scale, v_scale, block_tables,
               context_lens, query_start, scale, rows=None):
        q = codecs.decode(q_codes, q_dtype)
        T, Hq, D = q.shape
        G = Hq // k_codes.shape[1]
        out = np.zeros((T, Hq, D))
        for s in range(len(context_lens)):
            L, q0, q1 = int(context_lens[s]), int(query_start[s]), int(query_start[s + 1])
            for t in range(q0, q1):
                n = visible(L, q1 - q0, t - q0)
                for h in range(Hq):
                    K = codecs.decode(attention.gather_sequence(k_codes, block_tables[s], n, h // G), kv_dtype) * k_scale
                    V = codecs.decode(attention.gather_sequence(v_codes, block_tables[s], n, h // G), kv_dtype) * v_scale
                    out[t, h] = attention.softmax_weighted_sum(q[t, h], K, V, scale)
        return out
    return mutant


def test_extend_mutants_reproduce_the_oracle_when_unmutated(monkeypatch):
    # the harness itself is faithful: the true rule passes every extend pin
    monkeypatch.setattr(attention, "paged_extend", _extend_mutant(lambda L, Q, i: L - Q + i + 1))
    for pin in (te.test_matches_dense_causal_attention, te.test_first_prompt_token_returns_its_value_row,
                te.test_brute_force_loops, te.test_single_query_is_decode):
        pin()


def test_extend_query_not_seeing_itself_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "paged_extend", _extend_mutant(lambda L, Q, i: L - Q + i))
    assert _fails(te.test_first_prompt_token_returns_its_value_row)
    assert _fails(te.test_brute_force_loops)


def test_extend_position_from_context_start_is_caught(monkeypatch):
    # chunked prefill mistake: query i placed at position i instead of L - Q + i
    monkeypatch.setattr(attention, "paged_extend", _extend_mutant(lambda L, Q, i: i + 1))
    assert _fails(te.test_matches_dense_causal_attention)
    assert _fails(te.test_single_query_is_decode)


def test_extend_without_causal_mask_is_caught(monkeypatch):
    monkeypatch.setattr(attention, "paged_extend", _extend_mutant(lambda L, Q, i: L))
    assert _fails(te.test_matches_dense_causal_attention)
    assert _fails(te.test_first_prompt_token_returns_its_value_row)


# ---- block pool -------------------------------------------------------------------

def _append_mutant(cow, drop_old):
    def seq_append(self, row, pos, block_size):
        lb, off = divmod(pos, block_size)
        cs = cd = -1
        if off == 0:
            row.append(self.alloc())
        elif cow and self.refcnt[row[lb]] > 1:
            new = self.alloc()
            if drop_old:
                self.decref(row[lb])
            cs, cd = row[lb], new
            row[lb] = new
        return row[lb] * block_size + off, cs, cd
    return seq_append


def test_pool_mutant_harness_is_faithful(monkeypatch):
    monkeypatch.setattr(BlockPool, "seq_append", _append_mutant(True, True))
    tp.test_copy_on_write_of_shared_partial_block()
    tp.test_prefix_sharing_cow_count_is_sharers_minus_one()


def test_writing_into_a_shared_block_is_caught(monkeypatch):
    monkeypatch.setattr(BlockPool, "seq_append", _append_mutant(False, True))
    assert _fails(tp.test_copy_on_write_of_shared_partial_block)
    assert _fails(tp.test_prefix_sharing_cow_count_is_sharers_minus_one)


def test_copy_on_write_keeping_the_old_reference_is_caught(monkeypatch):
    monkeypatch.setattr(BlockPool, "seq_append", _append_mutant(True, False))
    assert _fails(tp.test_copy_on_write_of_shared_partial_block)
    assert _fails(tp.test_prefix_sharing_cow_count_is_sharers_minus_one)


def test_fifo_free_list_is_caught(monkeypatch):
    def decref(self, b):
        self._check(b)
        if self.refcnt[b] == 0:
            raise PoolError("STATE", "decref of free block")
        self.refcnt[b] -= 1
        if self.refcnt[b] == 0:
            self.free.insert(0, b)          # queue instead of stack
    monkeypatch.setattr(BlockPool, "decref", decref)
    assert _fails(tp.test_lifo_order_and_errors)


def test_reorder_dropping_old_references_first_is_caught(monkeypatch):
    def reorder(pool, rows, lens, parents):
        for r in rows:
            for b in r:
                pool.decref(b)
        new_rows = [list(rows[p]) for p in parents]
        for r in new_rows:
            for b in r:
                pool.incref(b)
        return new_rows, [lens[p] for p in parents]
    monkeypatch.setattr(opool, "reorder", reorder)
    assert _fails(tb.test_reorder_keeps_chosen_beams_and_frees_dropped_ones)


# ---- prefix cache -----------------------------------------------------------------

def test_prefix_key_of_the_block_alone_is_caught(monkeypatch):
    def key_of_block(self, k, tokens):
        return tuple(tokens[k * self.bs:(k + 1) * self.bs])

    def match(self, pool, tokens, row):
        n = 0
        for k in range(len(tokens) // self.bs):
            b = self.entries.get(key_of_block(self, k, tokens))
            if b is None:
                break
            pool.incref(b)
            row.append(b)
            n += 1
        return n

    def insert(self, pool, tokens, row):
        added = 0
        for k in range(len(tokens) // self.bs):
            key = key_of_block(self, k, tokens)
            if key in self.entries:
                continue
            pool.incref(row[k])
            self.entries[key] = row[k]
            self.order.append(key)
            added += 1
        return added
    monkeypatch.setattr(PrefixCache, "match", match)
    monkeypatch.setattr(PrefixCache, "insert", insert)
    assert _fails(tpc.test_a_block_repeated_at_another_position_is_not_reused)


def test_match_without_a_reference_is_caught(monkeypatch):
    orig = PrefixCache.match

    def match(self, pool, tokens, row):
        n = orig(self, pool, tokens, row)
        for b in row[len(row) - n:]:
            pool.decref(b)                  # the hit no longer holds its block
        return n
    monkeypatch.setattr(PrefixCache, "match", match)
    assert _fails(tpc.test_page3_shared_history_case)
