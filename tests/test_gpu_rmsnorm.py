"""bi_rmsnorm on the GPU: parity with the fp64 oracle and bitwise batch
invariance (each row byte-compared across every batch size M = 1..2048 and
across row positions)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import TOL_BF16, TOL_F32, dev_bf16, rowwise_normwise, same_bytes, to_f64
from synth import norm_matmul, normal_bf16, rng, tiny_layer, uniform_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


def check_parity(L, x_bits, w_bits, eps, out_dtype=torch.bfloat16):
    y = L.bi_rmsnorm(dev_bf16(x_bits), dev_bf16(w_bits), eps, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(x_bits, w_bits, eps)
    err = rowwise_normwise(to_f64(y), ref)
    tol = TOL_BF16 if out_dtype == torch.bfloat16 else TOL_F32
    assert err.max() <= tol, "worst row %d: %.3g" % (err.argmax(), err.max())
    return err.max()


def test_tiny_layer_parity(L):
    c = tiny_layer()
    for B in c["batch_sizes"]:
        check_parity(L, c["x"][:B], c["w"], c["eps"])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_hidden_4096_parity_ragged(L, out_dtype):
    c = norm_matmul(M=2048)
    for M in (1, 7, 300, 2048):
        check_parity(L, c["x"][:M], c["w"], c["eps"], out_dtype)


@pytest.mark.parametrize("H", [8, 24, 264, 4104, 14336, 65536])
def test_odd_and_extreme_widths(L, H):
    g = rng(100 + H)
    x = normal_bf16(g, (5, H))
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    check_parity(L, x, w, 1e-6)
    check_parity(L, x, w, 1e-6, torch.float32)


def test_constant_row_closed_form(L):
    # x = c*1 -> y = c/sqrt(c^2+eps)*w, which rounds to the bf16 of w (|c| >= 1)
    H = 4096
    g = rng(5)
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    x = np.zeros((3, H), dtype=np.uint16)
    x[0] = 0x3F80   # 1.0
    x[1] = 0xC020   # -2.5
    x[2] = 0x4140   # 12
    y = L.bi_rmsnorm(dev_bf16(x), dev_bf16(w), 1e-6, out_dtype=torch.float32)
    wf = to_f64(dev_bf16(w))
    got = to_f64(y)
    np.testing.assert_allclose(got[0], wf, rtol=2e-6)
    np.testing.assert_allclose(got[1], -wf, rtol=2e-6)
    np.testing.assert_allclose(got[2], wf, rtol=2e-6)


def test_every_batch_size_gives_the_same_row_bits(L):
    c = norm_matmul(M=2048)
    x = dev_bf16(c["x"])
    w = dev_bf16(c["w"])
    full = L.bi_rmsnorm(x, w, c["eps"])
    full32 = L.bi_rmsnorm(x, w, c["eps"], out_dtype=torch.float32)
    bad = []
    for M in range(1, 2049):
        y = L.bi_rmsnorm(x[:M], w, c["eps"])
        if not same_bytes(y, full[:M]):
            bad.append(M)
    for M in (1, 2, 3, 100, 1000, 2047):
        if not same_bytes(L.bi_rmsnorm(x[:M], w, c["eps"], out_dtype=torch.float32), full32[:M]):
            bad.append(-M)
    assert not bad, "batch sizes whose rows differ from M=2048: %s" % bad[:20]


def test_row_position_and_neighbours_do_not_matter(L):
    c = norm_matmul(M=512)
    x = dev_bf16(c["x"])
    w = dev_bf16(c["w"])
    full = L.bi_rmsnorm(x, w, c["eps"])
    perm = torch.randperm(512, generator=torch.Generator().manual_seed(0)).to(x.device)
    y = L.bi_rmsnorm(x[perm].contiguous(), w, c["eps"])
    assert same_bytes(y, full[perm])
    # the same row amid other rows drawn fresh
    other = dev_bf16(normal_bf16(rng(9), (64, 4096)))
    mix = torch.cat([other[:31], x[17:18], other[31:]]).contiguous()
    assert same_bytes(L.bi_rmsnorm(mix, w, c["eps"])[31], full[17])


def test_repeat_runs_are_identical(L):
    c = norm_matmul(M=300)
    x, w = dev_bf16(c["x"]), dev_bf16(c["w"])
    a = L.bi_rmsnorm(x, w, c["eps"])
    for _ in range(20):
        assert same_bytes(L.bi_rmsnorm(x, w, c["eps"]), a)
