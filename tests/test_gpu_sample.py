"""bi_sample on the GPU: parity with the fp64 oracle (same Philox draw, same
nucleus rule), greedy rows equal to bi_argmax, bitwise batch invariance and
repeatability, and softmax frequencies.

The kernel decides in fp32 and the oracle in fp64, so a draw that lands
within rounding of a boundary (the nucleus threshold, or a step of the
cumulative distribution) may pick a neighbour; such rows are allowed only
when the boundary is that close, and must then still be a valid draw."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import DEV
from synth import rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


def dev(a, dtype):
    return torch.as_tensor(np.ascontiguousarray(a)).to(DEV).to(dtype)


def case(seed, T, V=32000):
    g = rng(seed)
    logits = (g.standard_normal((T, V)) * 2.0).astype(np.float32)
    temp = g.choice([0.5, 0.8, 1.0, 1.3], size=T).astype(np.float32)
    top_p = g.choice([0.1, 0.5, 0.9, 0.95, 1.0], size=T).astype(np.float32)
    seeds = g.integers(0, 2 ** 63, size=T, dtype=np.int64).astype(np.uint64)
    offs = g.integers(0, 2 ** 20, size=T).astype(np.uint64)
    return logits, temp, top_p, seeds, offs


def run(L, logits, temp, top_p, seeds, offs):
    return L.bi_sample(dev(logits, torch.float32), dev(temp, torch.float32),
                       dev(top_p, torch.float32), dev(seeds.view(np.int64), torch.int64),
                       dev(offs.view(np.int64), torch.int64)).cpu().numpy()


def margin(logits_row, temp, top_p, r):
    """How close (relative to the total weight) the oracle's draw r and the
    nucleus threshold come to a boundary: the smallest distance from r to a
    step of the kept cumulative distribution, and from top_p to a step of
    the sorted cumulative weights."""
    z = logits_row.astype(np.float64) / float(temp)
    w = np.exp(z - z.max())
    tot = w.sum()
    srt = np.sort(w)[::-1]
    cs = np.cumsum(srt) / tot
    d_thr = np.min(np.abs(cs - float(top_p)))
    k = np.searchsorted(cs, float(top_p))  # the threshold's rank
    tau = srt[min(k, len(srt) - 1)]
    kept = w >= tau
    cdf = np.cumsum(np.where(kept, w, 0.0)) / tot
    d_cdf = np.min(np.abs(cdf[kept] - r))
    return min(d_thr, d_cdf)


def test_sample_matches_the_oracle(L):
    logits, temp, top_p, seeds, offs = case(150, 400)
    got = run(L, logits, temp, top_p, seeds, offs)
    want, r, _ = oracle.sample(logits, temp, top_p, seeds, offs, details=True)
    bad = np.nonzero(got != want)[0]
    print("rows decided differently at a boundary: %d of %d" % (len(bad), len(got)))
    assert len(bad) <= 4, bad
    for t in bad:  # only at a rounding-close boundary
        assert margin(logits[t], temp[t], top_p[t], r[t]) < 1e-5, t


def test_temperature_zero_rows_are_greedy(L):
    logits, _, top_p, seeds, offs = case(151, 64)
    logits[5, 100] = logits[5].max() + 1.0
    logits[5, 7] = logits[5, 100]  # a tie: the lower index wins
    got = run(L, logits, np.zeros(64, np.float32), top_p, seeds, offs)
    want = L.bi_argmax(dev(logits, torch.float32)).cpu().numpy()
    assert np.array_equal(got, want) and got[5] == 7


def test_rows_do_not_depend_on_the_batch(L):
    logits, temp, top_p, seeds, offs = case(152, 256)
    full = run(L, logits, temp, top_p, seeds, offs)
    g = rng(153)
    for B in (1, 3, 17, 100):
        sel = g.choice(256, size=B, replace=False)
        part = run(L, logits[sel], temp[sel], top_p[sel], seeds[sel], offs[sel])
        assert np.array_equal(part, full[sel]), B
    for _ in range(20):
        assert np.array_equal(run(L, logits, temp, top_p, seeds, offs), full)


def test_frequencies_follow_the_softmax(L):
    row = np.array([1.0, 0.0, -1.0, 2.0, 0.5, -3.0, 0.25, 1.5], dtype=np.float32)
    n = 40000
    logits = np.repeat(row[None], n, axis=0)
    got = run(L, logits, np.full(n, 0.7, np.float32), np.ones(n, np.float32),
              np.arange(n, dtype=np.uint64), np.full(n, 42, np.uint64))
    p = np.exp(row.astype(np.float64) / 0.7)
    p /= p.sum()
    for k in range(len(row)):
        f = (got == k).mean()
        assert abs(f - p[k]) < 4.5 * np.sqrt(p[k] * (1 - p[k]) / n), (k, f, p[k])


def test_degenerate_cases(L):
    g = rng(154)
    # one-token vocabulary, odd vocabulary sizes, an empty batch
    for V in (1, 3, 31999):
        logits = g.standard_normal((7, V)).astype(np.float32)
        got = run(L, logits, np.full(7, 0.9, np.float32), np.full(7, 0.9, np.float32),
                  np.arange(7, dtype=np.uint64), np.zeros(7, np.uint64))
        want = oracle.sample(logits, 0.9, 0.9, np.arange(7, dtype=np.uint64), 0)
        assert np.array_equal(got, want), V
    empty = L.bi_sample(torch.empty((0, 10), device=DEV), 1.0, 1.0, 0, 0)
    assert empty.shape == (0,)
    # top_p 0 keeps only the largest weight(s); a tiny temperature is greedy
    logits = g.standard_normal((50, 1000)).astype(np.float32)
    greedy = L.bi_argmax(dev(logits, torch.float32)).cpu().numpy()
    seeds = np.arange(50, dtype=np.uint64)
    assert np.array_equal(run(L, logits, np.ones(50, np.float32), np.zeros(50, np.float32),
                              seeds, seeds), greedy)
    assert np.array_equal(run(L, logits, np.full(50, 1e-6, np.float32), np.ones(50, np.float32),
                              seeds, seeds), greedy)
