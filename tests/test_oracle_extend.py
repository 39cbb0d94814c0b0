"""Pins for the oracle's multi-query (extend / chunked prefill) attention."""

import math

import numpy as np
import torch

from oracle import attention


def _bf16_codes(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_vals(codes):
    return torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _layout(rng, lens, Hkv, D, BS, NB):
    kc = _bf16_codes(rng.normal(size=(NB, Hkv, BS, D)))
    vc = _bf16_codes(rng.normal(size=(NB, Hkv, BS, D)))
    perm = rng.permutation(NB)
    MB = max(-(-L // BS) for L in lens)
    bt = np.zeros((len(lens), MB), np.int64)
    nxt = 0
    for s, L in enumerate(lens):
        for k in range(-(-L // BS)):
            bt[s, k] = perm[nxt]
            nxt += 1
    return kc, vc, bt


def test_single_query_is_decode():
    rng = np.random.default_rng(1)
    lens, Hkv, G, D, BS = [5, 33, 70], 2, 2, 8, 4
    kc, vc, bt = _layout(rng, lens, Hkv, D, BS, 40)
    q = _bf16_codes(rng.normal(size=(3, Hkv * G, D)))
    ext = attention.paged_extend(q, "bf16", kc, vc, "bf16", 1.0, 1.0, bt, lens, [0, 1, 2, 3], 0.3)
    dec = attention.paged_decode(q, "bf16", kc, vc, "bf16", 1.0, 1.0, bt, lens, 0.3)
    assert np.array_equal(ext, dec)


def test_matches_dense_causal_attention():
    """Identity tables: the textbook causal softmax(Q K^T * scale + mask) V, written
    as a masked matrix product."""
    rng = np.random.default_rng(2)
    L, Qn, Hkv, G, D, BS = 37, 9, 1, 3, 6, 4
    kc, vc, _ = _layout(rng, [L], Hkv, D, BS, 10)
    bt = np.arange(10, dtype=np.int64)[None, :]
    q = _bf16_codes(rng.normal(size=(Qn, Hkv * G, D)))
    got = attention.paged_extend(q, "bf16", kc, vc, "bf16", 1.0, 1.0, bt, [L], [0, Qn], 0.45)
    K = _bf16_vals(kc)[:, 0].reshape(-1, D)[:L]
    V = _bf16_vals(vc)[:, 0].reshape(-1, D)[:L]
    Q = _bf16_vals(q)
    for h in range(G):
        S = 0.45 * Q[:, h] @ K.T                                  # [Qn, L]
        pos = L - Qn + np.arange(Qn)
        mask = np.arange(L)[None, :] > pos[:, None]
        S = np.where(mask, -np.inf, S)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        want = (P / P.sum(axis=1, keepdims=True)) @ V
        assert np.allclose(got[:, h], want, atol=1e-12, rtol=0)


def test_first_prompt_token_returns_its_value_row():
    """Prefill of a whole prompt: query 0 sees only token 0."""
    rng = np.random.default_rng(3)
    L, D, BS = 20, 8, 4
    kc, vc, bt = _layout(rng, [L], 1, D, BS, 8)
    q = _bf16_codes(rng.normal(size=(L, 1, D)) * 30)
    out = attention.paged_extend(q, "bf16", kc, vc, "bf16", 1.0, 1.0, bt, [L], [0, L], 1.0)
    assert np.array_equal(out[0, 0], _bf16_vals(vc)[bt[0, 0], 0, 0])


def test_brute_force_loops():
    rng = np.random.default_rng(4)
    lens, qlens, Hkv, G, D, BS = [6, 11], [3, 4], 2, 2, 3, 4
    kc, vc, bt = _layout(rng, lens, Hkv, D, BS, 12)
    qs = [0, 3, 7]
    q = _bf16_codes(rng.normal(size=(7, Hkv * G, D)))
    got = attention.paged_extend(q, "bf16", kc, vc, "bf16", 1.0, 1.0, bt, lens, qs, 0.7)
    Kv, Vv, Qv = _bf16_vals(kc), _bf16_vals(vc), _bf16_vals(q)
    for s in range(2):
        for i in range(qlens[s]):
            t = qs[s] + i
            pos = lens[s] - qlens[s] + i
            for h in range(Hkv * G):
                g = h // G
                xs = []
                for j in range(pos + 1):
                    row = Kv[bt[s, j // BS], g, j % BS]
                    xs.append(0.7 * sum(Qv[t, h, d] * row[d] for d in range(D)))
                mx = max(xs)
                ws = [math.exp(x - mx) for x in xs]
                for d in range(D):
                    num = sum(ws[j] * Vv[bt[s, j // BS], g, j % BS, d] for j in range(pos + 1))
                    assert abs(got[t, h, d] - num / sum(ws)) < 1e-12
