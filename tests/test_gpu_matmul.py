"""bi_matmul on the GPU (tcgen05 + TMA): parity with the fp64 oracle, exact
cases, and bitwise batch invariance across M = 1..2048 and row positions."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import TOL_BF16, TOL_F32, dev_bf16, rowwise_normwise, same_bytes, to_f64
from synth import f32_to_bf16_bits, norm_matmul, normal_bf16, rng, tiny_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


def parity(L, a, w, out_dtype=torch.bfloat16, rows=None):
    c = L.bi_matmul(dev_bf16(a), dev_bf16(w), out_dtype=out_dtype)
    torch.cuda.synchronize()
    if rows is None:
        rows = np.arange(a.shape[0])
    ref = oracle.matmul(a[rows], w)
    err = rowwise_normwise(to_f64(c)[rows], ref)
    tol = TOL_BF16 if out_dtype == torch.bfloat16 else TOL_F32
    assert err.max() <= tol, "worst row %d: %.3g" % (rows[err.argmax()], err.max())
    return err.max()


def test_tiny_layer_parity(L):
    c = tiny_layer()
    for B in c["batch_sizes"]:
        parity(L, c["x"][:B], c["W"])
        parity(L, c["x"][:B], c["W"], torch.float32)


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (3, 264, 72), (129, 512, 136), (200, 776, 1000),
                                   (257, 256, 64), (130, 4096, 4096)])
def test_ragged_shapes(L, M, N, K):
    g = rng(M * 7 + N + K)
    a = normal_bf16(g, (M, K))
    w = normal_bf16(g, (N, K), std=0.02)
    parity(L, a, w)
    parity(L, a, w, torch.float32)


@pytest.mark.parametrize("N", [4096, 12288])
def test_hidden_4096_full_size_sampled_rows(L, N):
    c = norm_matmul(M=2048, N=N)
    # the tile edges plus 256 random rows (each row is checked element by element)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, 2047], rng(3).integers(0, 2048, 256)]))
    parity(L, c["x"], c["W"], rows=rows)
    parity(L, c["x"], c["W"], torch.float32, rows=rows)


def test_identity_weight_is_exact(L):
    g = rng(1)
    a = normal_bf16(g, (300, 256))
    eye = f32_to_bf16_bits(np.eye(256, dtype=np.float32))
    out = L.bi_matmul(dev_bf16(a), dev_bf16(eye))
    assert same_bytes(out, dev_bf16(a))


def test_small_integers_are_exact(L):
    # |a|,|w| <= 8, K = 256: every partial sum is an integer below 2^24
    g = rng(2)
    a = f32_to_bf16_bits(g.integers(-8, 9, size=(150, 256)).astype(np.float32))
    w = f32_to_bf16_bits(g.integers(-8, 9, size=(264, 256)).astype(np.float32))
    out = L.bi_matmul(dev_bf16(a), dev_bf16(w), out_dtype=torch.float32)
    np.testing.assert_array_equal(to_f64(out), oracle.matmul(a, w))


def test_every_batch_size_gives_the_same_row_bits(L):
    c = norm_matmul(M=2048, N=4096)
    x, W = dev_bf16(c["x"]), dev_bf16(c["W"])
    full = L.bi_matmul(x, W)
    bad = []
    for M in range(1, 2049):
        if not same_bytes(L.bi_matmul(x[:M], W), full[:M]):
            bad.append(M)
    assert not bad, "batch sizes whose rows differ from M=2048: %s" % bad[:20]


def test_wide_n_batch_sizes(L):
    c = norm_matmul(M=2048, N=12288)
    x, W = dev_bf16(c["x"]), dev_bf16(c["W"])
    full = L.bi_matmul(x, W)
    full32 = L.bi_matmul(x, W, out_dtype=torch.float32)
    for M in (1, 2, 5, 64, 127, 128, 129, 500, 1024, 1999):
        assert same_bytes(L.bi_matmul(x[:M], W), full[:M]), M
        assert same_bytes(L.bi_matmul(x[:M], W, out_dtype=torch.float32), full32[:M]), M


def test_row_position_does_not_matter(L):
    """The tensor core gives a row the same bits at any row of the tile."""
    c = norm_matmul(M=512, N=1024)
    x, W = dev_bf16(c["x"]), dev_bf16(c["W"])
    full = L.bi_matmul(x, W, out_dtype=torch.float32)
    perm = torch.randperm(512, generator=torch.Generator().manual_seed(1)).to(x.device)
    y = L.bi_matmul(x[perm].contiguous(), W, out_dtype=torch.float32)
    assert same_bytes(y, full[perm])
    # one row copied into every row position of a 128-row tile, random neighbours
    other = dev_bf16(normal_bf16(rng(4), (128, 4096)))
    for pos in (0, 1, 31, 32, 63, 64, 100, 127):
        mix = other.clone()
        mix[pos] = x[9]
        assert same_bytes(L.bi_matmul(mix, W, out_dtype=torch.float32)[pos], full[9]), pos


def test_repeat_runs_are_identical(L):
    c = norm_matmul(M=700, N=4096)
    x, W = dev_bf16(c["x"]), dev_bf16(c["W"])
    a = L.bi_matmul(x, W)
    for _ in range(10):
        assert same_bytes(L.bi_matmul(x, W), a)
    assert L.bi_device_status() == bi.Status.OK
