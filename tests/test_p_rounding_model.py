"""How the extend / prefill kernels feed P to the tensor cores, checked on the CPU.

The softmax probabilities P enter the P V tensor-core product as 16-bit values (the A and
B operands of one MMA share a type); everything else is binary32. This test restates the
kernels' arithmetic in numpy and compares it with float64 attention at the parity
tolerance |err| <= 2e-3 + 1e-2 |ref|, on N(0, 1) inputs as the GPU tests draw them, with
score scales from flat to peaked (scale * sqrt(D) = 1, 4, 12):

* P rounded to bf16 alone (the arithmetic before the fix) leaves the tolerance: a rounding
  of up to 2^-8 of a dominant weight moves the output by up to 2^-8 |v| while cancelling V
  values keep |ref| small. Rows that see few tokens and rows with peaked scores both do;
* the tcgen05 kernel's arithmetic -- 128-token tiles whose two 64-column halves keep
  separate running sums, a reference maximum that moves only by more than 2^8, P as p
  rounded to bf16 and the bf16 remainder p - bf16(p), added as a second product to the
  rows of every group of 32 (one warp's rows) where some row has a weight above 1/8 of
  its running sum (the two halves' sums, exchanged with the maxima), zeros to the other
  rows of the tile -- stays inside for every element;
* the mma.sync kernels' arithmetic -- 16-token slices, the running maximum, P and its bf16
  remainder for every slice where some row has a weight above 1/8 of its running sum,
  the running sum over what enters the products -- stays inside;
* f16 P (rounding up to 2^-11 of p) stays inside without a remainder.
It runs no GPU code.
"""

import numpy as np
import pytest
import torch

TILE = 128
SHARE = 0.125      # the tcgen05 kernel's threshold for the remainder product


def _round(x, dt):
    t = torch.bfloat16 if dt == "bf16" else torch.float16
    return torch.from_numpy(np.asarray(x, np.float32)).to(t).to(torch.float32).numpy()


def tcgen05_arithmetic(q, K, V, qpos, scale, dt, remainder):
    """remainder: None (P rounded alone), "adaptive" (the kernel's rule) or "always"."""
    s_mul = np.float32(scale * 1.4426950408889634)
    R, D = q.shape
    m = np.full(R, -np.inf, np.float32)
    lh = np.zeros((2, R), np.float32)          # running sums of the two 64-column halves
    O = np.zeros((R, D), np.float32)
    flagged = 0
    for j in range(-(-K.shape[0] // TILE)):
        lo, hi = j * TILE, min(K.shape[0], (j + 1) * TILE)
        S = q @ K[lo:hi].T
        S = np.where(np.arange(lo, hi)[None, :] > qpos[:, None], -np.inf, S)
        with np.errstate(invalid="ignore"):
            mx = S.max(axis=1) * s_mul
            up = mx > m + 8
            corr = np.where(up, np.exp2(m - mx), 1.0).astype(np.float32)
        lh, O, m = np.where(up, lh * corr, lh), np.where(up[:, None], O * corr[:, None], O), np.where(up, mx, m)
        ref = np.where(m == -np.inf, 0, m)
        p = np.exp2(S * s_mul - ref[:, None]).astype(np.float32)
        with np.errstate(invalid="ignore"):
            pmax = np.exp2(mx - ref).astype(np.float32)
        # per group of 32 rows (one warp's rows), before this tile's sums
        need_row = pmax > SHARE * (lh.sum(axis=0) + pmax)
        need = np.repeat(need_row.reshape(-1, 32).any(axis=1), 32) if R % 32 == 0 else np.full(R, need_row.any())
        halves = [p[:, :64], p[:, 64:]]
        lh = lh + np.stack([np.pad(x, ((0, 0), (0, 64 - x.shape[1]))).sum(axis=1) for x in halves])
        P = _round(p, dt)
        rem = _round(p - P, dt) if dt == "bf16" else None
        if rem is not None and remainder == "always":
            flagged += 1
            P = P + rem
        elif rem is not None and remainder == "adaptive" and need.any():
            flagged += 1
            P = P + np.where(need[:, None], rem, 0)
        O = O + P @ V[lo:hi]
    return _round(O / lh.sum(axis=0)[:, None], dt), flagged


def mma_sync_arithmetic(q, K, V, qpos, scale, dt, adaptive=True):
    """16-token slices, the running maximum (rescale whenever it grows), P and, for a
    slice where some row's largest weight exceeds 1/8 of its running sum (adaptive) or
    always, its bf16 remainder; the running sum over what enters the products. (The
    kernel decides per warp from each lane's share of a row, which flags at least the
    slices this row-wise rule flags.)"""
    s_mul = np.float32(scale * 1.4426950408889634)
    R, D = q.shape
    m = np.full(R, -np.inf, np.float32)
    l = np.zeros(R, np.float32)
    O = np.zeros((R, D), np.float32)
    for j in range(-(-K.shape[0] // 16)):
        lo, hi = j * 16, min(K.shape[0], (j + 1) * 16)
        S = (q @ K[lo:hi].T) * s_mul
        S = np.where(np.arange(lo, hi)[None, :] > qpos[:, None], -np.inf, S)
        mx = S.max(axis=1)
        grow = mx > m
        with np.errstate(invalid="ignore"):
            corr = np.where(grow, np.exp2(m - mx), 1.0).astype(np.float32)
        l, O, m = np.where(grow, l * corr, l), np.where(grow[:, None], O * corr[:, None], O), np.where(grow, mx, m)
        p = np.exp2(S - np.where(m == -np.inf, 0, m)[:, None]).astype(np.float32)
        P = _round(p, dt)
        if dt == "bf16":
            rem = _round(p - P, dt)
            with np.errstate(invalid="ignore"):
                need = np.any(p.max(axis=1) > SHARE * (l + (P + rem).sum(axis=1)))
            if need or not adaptive:
                P = P + rem
        l = l + P.sum(axis=1)
        O = O + P @ V[lo:hi]
    return _round(O / l[:, None], dt)


def float64_attention(q, K, V, qpos, scale):
    x = scale * (q.astype(np.float64) @ K.T.astype(np.float64))
    x = np.where(np.arange(K.shape[0])[None, :] > qpos[:, None], -np.inf, x)
    w = np.exp(x - x.max(axis=1, keepdims=True))
    return (w @ V.astype(np.float64)) / w.sum(axis=1, keepdims=True)


def _draw(seed, short, dt):
    """128 query rows: every row seeing 1-15 tokens, or rows at random positions of a
    16-1500-token context."""
    rng = np.random.default_rng(seed)
    if short:
        n, qpos = 15, np.repeat(np.arange(15), 9)[:128]
    else:
        n = int(rng.integers(16, 1500))
        qpos = np.sort(rng.integers(15, n, size=128))
    D = 128
    q, K, V = (_round(rng.normal(size=s), dt) for s in ((128, D), (n, D), (n, D)))
    return q, K, V, qpos


def _excess(got, q, K, V, qpos, scale):
    ref = float64_attention(q, K, V, qpos, scale)
    return float((np.abs(got - ref) - (2e-3 + 1e-2 * np.abs(ref))).max())


@pytest.mark.parametrize("mult", [1.0, 4.0, 12.0])
def test_bf16_p_alone_leaves_the_tolerance(mult):
    """The arithmetic before the fix: some element leaves the tolerance at every scale."""
    worst = -1.0
    for seed in range(40):
        q, K, V, qpos = _draw(2000 + seed, seed % 2 == 0, "bf16")
        scale = mult / np.sqrt(128)
        worst = max(worst, _excess(tcgen05_arithmetic(q, K, V, qpos, scale, "bf16", None)[0], q, K, V, qpos, scale))
        if worst > 0:
            break
    assert worst > 0


@pytest.mark.parametrize("mult", [1.0, 4.0, 12.0])
def test_tcgen05_arithmetic_with_the_remainder_stays_inside(mult):
    scale = mult / np.sqrt(128)
    worst, flagged, tiles = -1.0, 0, 0
    for seed in range(24):
        q, K, V, qpos = _draw(3000 + seed, seed % 3 == 0, "bf16")
        got, f = tcgen05_arithmetic(q, K, V, qpos, scale, "bf16", "adaptive")
        worst = max(worst, _excess(got, q, K, V, qpos, scale))
        flagged, tiles = flagged + f, tiles + -(-K.shape[0] // TILE)
    assert worst <= 0, worst
    if mult == 1.0:   # flat scores: the product is needed for few tiles
        assert flagged < 0.5 * tiles


@pytest.mark.parametrize("mult", [1.0, 4.0, 12.0])
def test_mma_sync_arithmetic_with_the_remainder_stays_inside(mult):
    scale = mult / np.sqrt(128)
    worst = -1.0
    for seed in range(16):
        q, K, V, qpos = _draw(4000 + seed, seed % 2 == 0, "bf16")
        worst = max(worst, _excess(mma_sync_arithmetic(q, K, V, qpos, scale, "bf16"), q, K, V, qpos, scale))
    assert worst <= 0, worst


@pytest.mark.parametrize("mult", [1.0, 4.0, 12.0])
def test_f16_p_stays_inside_without_a_remainder(mult):
    scale = mult / np.sqrt(128)
    worst = -1.0
    for seed in range(16):
        q, K, V, qpos = _draw(5000 + seed, seed % 2 == 0, "f16")
        got = tcgen05_arithmetic(q, K, V, qpos, scale, "f16", None)[0]
        worst = max(worst, _excess(got, q, K, V, qpos, scale))
        worst = max(worst, _excess(mma_sync_arithmetic(q, K, V, qpos, scale, "f16"), q, K, V, qpos, scale))
    assert worst <= 0, worst
