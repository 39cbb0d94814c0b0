"""Pins for the oracle's paged decode attention: worked examples, closed forms,
invariants and an independent brute force."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention, codecs
from tests.conftest import GOLDEN


def _one_seq(K, V, BS=4, perm=None):
    """Lay one sequence's K/V rows out in a paged cache of one kv head."""
    L, D = K.shape
    nb = -(-L // BS)
    order = list(range(nb)) if perm is None else list(perm)
    kc = np.full((max(order) + 1 if order else 1, 1, BS, D), np.nan)
    vc = np.full_like(kc, np.nan)
    for j in range(L):
        kc[order[j // BS], 0, j % BS] = K[j]
        vc[order[j // BS], 0, j % BS] = V[j]
    bt = np.array([order + [0]], dtype=np.int64)
    return kc, vc, bt


def test_hand_worked_two_tokens():
    # scores 0 and ln 3 -> weights 1/4 and 3/4
    q = np.array([[[1.0, 0.0]]])
    K = np.array([[0.0, 0.0], [math.log(3.0), 0.0]])
    V = np.array([[1.0, 0.0], [0.0, 1.0]])
    kc, vc, bt = _one_seq(K, V, BS=16)
    out = attention.paged_decode_f64(q, kc, vc, bt, [2], 1.0)
    assert np.allclose(out[0, 0], [0.25, 0.75], atol=1e-15)


def test_equal_scores_average():
    q = np.array([[[0.3, -2.0, 1.0]]])
    K = np.zeros((5, 3))
    V = np.arange(15, dtype=np.float64).reshape(5, 3)
    kc, vc, bt = _one_seq(K, V, BS=2)
    out = attention.paged_decode_f64(q, kc, vc, bt, [5], 0.7)
    assert np.allclose(out[0, 0], V.mean(axis=0), atol=1e-12)


def test_single_token_returns_its_value_row_exactly():
    rng = np.random.default_rng(1)
    for _ in range(20):
        D = int(rng.integers(1, 9))
        q = rng.normal(size=(1, 1, D))
        K = rng.normal(size=(1, D)) * 50
        V = rng.normal(size=(1, D))
        kc, vc, bt = _one_seq(K, V, BS=16, perm=[int(rng.integers(0, 5))])
        out = attention.paged_decode_f64(q, kc, vc, bt, [1], float(rng.uniform(0.01, 3)))
        assert np.array_equal(out[0, 0], V[0])


def test_constant_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    D, L = 8, 37
    q = rng.normal(size=(1, 1, D))
    K = np.tile(rng.normal(size=(1, D)), (L, 1))
    V = rng.normal(size=(L, D))
    kc, vc, bt = _one_seq(K, V, BS=16)
    out = attention.paged_decode_f64(q, kc, vc, bt, [L], 0.125)
    assert np.allclose(out[0, 0], V.mean(axis=0), atol=1e-12, rtol=0)


def test_huge_scores_stay_finite():
    q = np.array([[[1000.0]]])
    K = np.array([[1.0], [0.999], [0.5]])
    V = np.array([[1.0], [2.0], [3.0]])
    kc, vc, bt = _one_seq(K, V, BS=2)
    out = attention.paged_decode_f64(q, kc, vc, bt, [3], 1.0)
    w = np.array([1.0, math.exp(-1.0), math.exp(-500.0)])
    assert np.isclose(out[0, 0, 0], (w @ V[:, 0]) / w.sum(), rtol=1e-14)


def test_empty_context_gives_zero_row():
    kc = np.ones((2, 1, 4, 3))
    out = attention.paged_decode_f64(np.ones((1, 1, 3)), kc, kc, np.zeros((1, 1), np.int64), [0], 1.0)
    assert np.array_equal(out, np.zeros((1, 1, 3)))


def _brute(q, K_by_head, V_by_head, lens, scale, G):
    """Independent loop version: contiguous per-(seq, kv head) rows, math.exp."""
    S, Hq, D = q.shape
    out = np.zeros((S, Hq, D))
    for s in range(S):
        for h in range(Hq):
            g = h // G
            L = lens[s]
            if L == 0:
                continue
            xs = []
            for j in range(L):
                acc = 0.0
                for d in range(D):
                    acc += q[s, h, d] * K_by_head[s][g][j][d]
                xs.append(scale * acc)
            mx = max(xs)
            ws = [math.exp(x - mx) for x in xs]
            tot = sum(ws)
            for d in range(D):
                out[s, h, d] = sum(ws[j] * V_by_head[s][g][j][d] for j in range(L)) / tot
    return out


@pytest.mark.parametrize("G", [1, 2, 4])
def test_paged_equals_contiguous_brute_force(G):
    rng = np.random.default_rng(10 + G)
    S, Hkv, D, BS = 3, 2, 5, 4
    Hq = Hkv * G
    lens = [1, 9, 14]
    NB = 12
    perm = rng.permutation(NB)
    q = rng.normal(size=(S, Hq, D))
    Kc = [[rng.normal(size=(L, D)) for _ in range(Hkv)] for L in lens]
    Vc = [[rng.normal(size=(L, D)) for _ in range(Hkv)] for L in lens]
    kc = np.full((NB, Hkv, BS, D), np.nan)
    vc = np.full_like(kc, np.nan)
    bt = np.zeros((S, 4), dtype=np.int64)
    nxt = 0
    for s, L in enumerate(lens):
        for lb in range(-(-L // BS)):
            bt[s, lb] = perm[nxt]
            nxt += 1
        for g in range(Hkv):
            for j in range(L):
                kc[bt[s, j // BS], g, j % BS] = Kc[s][g][j]
                vc[bt[s, j // BS], g, j % BS] = Vc[s][g][j]
    got = attention.paged_decode_f64(q, kc, vc, bt, lens, 0.37)
    want = _brute(q, Kc, Vc, lens, 0.37, G)
    assert np.allclose(got, want, atol=1e-12, rtol=0)


def test_block_permutation_gives_identical_bits():
    rng = np.random.default_rng(4)
    S, H, D, BS, NB = 2, 2, 6, 4, 10
    lens = [7, 13]
    kc = rng.normal(size=(NB, H, BS, D))
    vc = rng.normal(size=(NB, H, BS, D))
    bt = np.array([[0, 1, 0, 0], [2, 3, 4, 5]])
    q = rng.normal(size=(S, H, D))
    base = attention.paged_decode_f64(q, kc, vc, bt, lens, 0.5)
    perm = rng.permutation(NB)              # physical block b moves to perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    moved = attention.paged_decode_f64(q, kc2, vc2, perm[bt], lens, 0.5)
    assert np.array_equal(base, moved)


def test_gqa_equals_mha_with_duplicated_kv_heads():
    rng = np.random.default_rng(5)
    S, Hkv, G, D, BS, NB = 2, 2, 3, 4, 4, 6
    kc = rng.normal(size=(NB, Hkv, BS, D))
    vc = rng.normal(size=(NB, Hkv, BS, D))
    q = rng.normal(size=(S, Hkv * G, D))
    bt = np.array([[5, 1], [0, 2]])
    lens = [6, 8]
    gqa = attention.paged_decode_f64(q, kc, vc, bt, lens, 0.3)
    mha = attention.paged_decode_f64(q, np.repeat(kc, G, axis=1), np.repeat(vc, G, axis=1), bt, lens, 0.3)
    assert np.array_equal(gqa, mha)


def test_page1_block_table_gather_order():
    fx = json.load(open(os.path.join(GOLDEN, "block_table_example.json")))
    BS, D = 4, 2
    # each physical row holds (block id, offset) so the gather shows its addressing
    kc = np.zeros((5, 1, BS, D))
    for b in range(5):
        for o in range(BS):
            kc[b, 0, o] = (b, o)
    for name, row in fx["tables"].items():
        L = len(row) * BS
        got = attention.gather_sequence(kc, row, L, 0)
        want = np.array([(row[j // BS], j % BS) for j in range(L)], dtype=np.float64)
        assert np.array_equal(got, want)
    # seq_2 reads physical 2, then the shared physical 1, then 4
    g2 = attention.gather_sequence(kc, fx["tables"]["seq_2"], 3 * BS, 0)
    assert [int(g2[j * BS, 0]) for j in range(3)] == [2, 1, 4]


def test_pool_diagram_gather_follows_logical_order():
    fx = json.load(open(os.path.join(GOLDEN, "pool_diagram_12_blocks.json")))
    BS = 2
    kc = np.zeros((fx["num_blocks"], 1, BS, 1))
    for b in range(fx["num_blocks"]):
        kc[b, 0, :, 0] = b
    got = attention.gather_sequence(kc, fx["tables"]["A"], 3 * BS, 0)[::BS, 0]
    assert got.tolist() == [0.0, 4.0, 8.0]


def test_code_level_decode_applies_scales_and_codecs():
    """Codes + per-tensor scales, checked by loops over torch's own fp8/bf16 decoders."""
    rng = np.random.default_rng(6)
    S, H, D, BS, NB = 2, 2, 4, 8, 5
    k_codes = rng.integers(0, 256, size=(NB, H, BS, D), dtype=np.uint8)
    v_codes = rng.integers(0, 256, size=(NB, H, BS, D), dtype=np.uint8)
    k_codes[(k_codes & 0x7F) == 0x7F] = 0x11   # no NaN codes in a cache
    v_codes[(v_codes & 0x7F) == 0x7F] = 0x22
    q32 = rng.normal(size=(S, H, D)).astype(np.float32)
    q_codes = torch.from_numpy(q32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bt = np.array([[3, 0], [4, 1]])
    lens = [11, 16]
    ks, vs = 0.0123, 0.0456
    got = attention.paged_decode(q_codes, "bf16", k_codes, v_codes, "e4m3", ks, vs, bt, lens, 0.5)
    kf = torch.from_numpy(k_codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * ks
    vf = torch.from_numpy(v_codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * vs
    qf = torch.from_numpy(q_codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    Kh = [[[kf[bt[s, j // BS], g, j % BS] for j in range(lens[s])] for g in range(H)] for s in range(S)]
    Vh = [[[vf[bt[s, j // BS], g, j % BS] for j in range(lens[s])] for g in range(H)] for s in range(S)]
    want = _brute(qf, Kh, Vh, lens, 0.5, 1)
    assert np.allclose(got, want, atol=1e-12, rtol=0)
