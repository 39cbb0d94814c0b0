"""What rounding P to bf16 does to extend / prefill outputs, on the CPU.

The extend and prefill kernels feed the softmax probabilities P to the tensor cores
rounded to the cache's 16-bit type (the A and B operands of one MMA share a type) and
keep everything else in binary32. This test restates that arithmetic in numpy -- 128-token
tiles, a reference maximum that moves only by more than 2^8, P rounded to bf16 for P V,
the running sum over the binary32 p -- and compares it with float64 attention at the
parity tolerance |err| <= 2e-3 + 1e-2 |ref| on N(0, 1) inputs, as the GPU tests draw them.

Rows that see 16 or more tokens stay inside the tolerance. Rows that see only a few can
leave it: one 2^-9 rounding of a dominant weight moves the output by up to 2^-9 |v| while
cancelling V values keep |ref| small. Adding the bf16 remainder p - bf16(p) for the
context's first tile (a second P V product) brings those rows inside again. This is the
basis of the known gap and of its planned fix; it runs no GPU code.
"""

import numpy as np
import torch

TILE = 128


def bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def kernel_arithmetic(q, K, V, qpos, scale, remainder_first_tile=False):
    s_mul = np.float32(scale * 1.4426950408889634)
    R, D = q.shape
    m = np.full(R, -np.inf, np.float32)
    l = np.zeros(R, np.float32)
    O = np.zeros((R, D), np.float32)
    for j in range(-(-K.shape[0] // TILE)):
        lo, hi = j * TILE, min(K.shape[0], (j + 1) * TILE)
        S = q @ K[lo:hi].T
        S = np.where(np.arange(lo, hi)[None, :] > qpos[:, None], -np.inf, S)
        with np.errstate(invalid="ignore"):
            mx = S.max(axis=1) * s_mul
            up = mx > m + 8
            corr = np.where(up, np.exp2(m - mx), 1.0).astype(np.float32)
        l, O, m = np.where(up, l * corr, l), np.where(up[:, None], O * corr[:, None], O), np.where(up, mx, m)
        p = np.exp2(S * s_mul - np.where(m == -np.inf, 0, m)[:, None]).astype(np.float32)
        l = l + p.sum(axis=1)
        P = bf16(p)
        if remainder_first_tile and j == 0:
            P = P + bf16(p - P)
        O = O + P @ V[lo:hi]
    return bf16(O / l[:, None])          # the output is stored in bf16


def float64_attention(q, K, V, qpos, scale):
    x = scale * (q.astype(np.float64) @ K.T.astype(np.float64))
    x = np.where(np.arange(K.shape[0])[None, :] > qpos[:, None], -np.inf, x)
    w = np.exp(x - x.max(axis=1, keepdims=True))
    return (w @ V.astype(np.float64)) / w.sum(axis=1, keepdims=True)


def _excess(n_tokens, qpos, seed, **kw):
    rng = np.random.default_rng(seed)
    D = 128
    q = bf16(rng.normal(size=(len(qpos), D)))
    K, V = bf16(rng.normal(size=(n_tokens, D))), bf16(rng.normal(size=(n_tokens, D)))
    got = kernel_arithmetic(q, K, V, qpos, 1 / np.sqrt(D), **kw)
    ref = float64_attention(q, K, V, qpos, 1 / np.sqrt(D))
    return np.abs(got - ref) - (2e-3 + 1e-2 * np.abs(ref))


def test_rows_that_see_sixteen_or_more_tokens_stay_inside_the_tolerance():
    worst = -1.0
    for seed in range(24):
        n = 16 + (seed * 97) % 600
        qpos = np.sort(np.random.default_rng(seed).integers(15, n, size=128))
        worst = max(worst, float(_excess(n, qpos, seed).max()))
    assert worst <= 0, worst


def test_short_rows_and_the_first_tile_remainder():
    plain, fixed = [], []
    for seed in range(60):
        qpos = np.repeat(np.arange(15), 9)[:128]          # every row sees 1..15 tokens
        plain.append(float(_excess(15, qpos, 1000 + seed).max()))
        fixed.append(float(_excess(15, qpos, 1000 + seed, remainder_first_tile=True).max()))
    assert max(fixed) <= 0, max(fixed)
    # with P rounded alone some of these tiles leave the tolerance (the known gap), and the
    # typical row comes much closer to the bound than with the remainder
    assert max(plain) > 0
    assert np.median(plain) > np.median(fixed) + 2.5e-4
