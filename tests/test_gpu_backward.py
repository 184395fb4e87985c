"""The backward passes on the GPU: RMSNorm backward (parity with the fp64
oracle, dx rows independent of the batch, dw the same bits on every run),
the transpose (a bit copy), and the matmul backward on the invariant GEMM
(parity with the oracle's products, exact on small integers, dA rows
independent of the batch), and the SwiGLU and RoPE backward (parity with
the oracle, rows independent of the batch, head sets inside wider rows)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import TOL_BF16, TOL_F32, dev_bf16, host_bits, normwise, rowwise_normwise, same_bytes, to_f64
from synth import bf16_bits_to_f32, f32_to_bf16_bits, normal_bf16, rng, uniform_bf16

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module")
def L():
    return bi.load()


def scaled_rows(g, M, K):
    x = normal_bf16(g, (M, K))
    s = np.exp2(g.uniform(-4, 4, size=(M, 1))).astype(np.float32)
    return f32_to_bf16_bits(bf16_bits_to_f32(x) * s)


@pytest.mark.parametrize("M,H", [(1, 256), (3, 4096), (300, 1000), (257, 4096), (600, 64)])
def test_rmsnorm_backward_parity(L, M, H):
    g = rng(500 + M + H)
    x, w, dy = scaled_rows(g, M, H), uniform_bf16(g, (H,), 0.5, 1.5), normal_bf16(g, (M, H))
    rdx, rdw = oracle.rmsnorm_backward(x, w, dy, EPS)
    for dt, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        dx, dw = L.bi_rmsnorm_backward(dev_bf16(x), dev_bf16(w), dev_bf16(dy), EPS, out_dtype=dt)
        assert rowwise_normwise(to_f64(dx), rdx).max() <= tol, dt
        assert normwise(to_f64(dw), rdw) <= tol, dt


def test_rmsnorm_backward_dx_rows_do_not_depend_on_the_batch(L):
    g = rng(510)
    x, w, dy = scaled_rows(g, 700, 4096), uniform_bf16(g, (4096,), 0.5, 1.5), normal_bf16(g, (700, 4096))
    xd, wd, dyd = dev_bf16(x), dev_bf16(w), dev_bf16(dy)
    full, dw_full = L.bi_rmsnorm_backward(xd, wd, dyd, EPS)
    for M in (1, 2, 255, 256, 257, 699):
        dx, _ = L.bi_rmsnorm_backward(xd[:M], wd, dyd[:M], EPS)
        assert same_bytes(dx, full[:M]), M
    for _ in range(5):  # dw sums over the rows: the same bits on every run
        _, dw = L.bi_rmsnorm_backward(xd, wd, dyd, EPS)
        assert same_bytes(dw, dw_full)


def test_transpose_is_a_bit_copy(L):
    g = rng(520)
    for R, C, ld in ((37, 70, 40), (1, 8, 8), (256, 300, 256), (1000, 33, 1000)):
        a = normal_bf16(g, (R, C))
        out = host_bits(L.bi_transpose(dev_bf16(a), ld_out=ld))
        np.testing.assert_array_equal(out[:, :R], a.T)
        assert np.all(out[:, R:] == 0)


@pytest.mark.parametrize("M,N,K", [(3, 264, 72), (129, 512, 136), (300, 776, 1000), (257, 1024, 512)])
def test_matmul_backward_parity(L, M, N, K):
    g = rng(530 + M + N + K)
    dc, a, w = normal_bf16(g, (M, N)), normal_bf16(g, (M, K)), normal_bf16(g, (N, K), std=0.05)
    rda = oracle.matmul(dc, np.ascontiguousarray(w.T))    # dC W
    rdw = oracle.matmul(np.ascontiguousarray(dc.T), np.ascontiguousarray(a.T))  # dC^T A
    for dt, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        da, dw = L.bi_matmul_backward(dev_bf16(dc), dev_bf16(a), dev_bf16(w), out_dtype=dt)
        assert rowwise_normwise(to_f64(da), rda).max() <= tol, dt
        assert rowwise_normwise(to_f64(dw), rdw).max() <= tol, dt


def test_matmul_backward_small_integers_are_exact(L):
    g = rng(540)
    ints = lambda shape: f32_to_bf16_bits(g.integers(-4, 5, size=shape).astype(np.float32))  # noqa: E731
    dc, a, w = ints((37, 64)), ints((37, 48)), ints((64, 48))
    da, dw = L.bi_matmul_backward(dev_bf16(dc), dev_bf16(a), dev_bf16(w), out_dtype=torch.float32)
    np.testing.assert_array_equal(to_f64(da), oracle.matmul(dc, np.ascontiguousarray(w.T)))
    np.testing.assert_array_equal(to_f64(dw), oracle.matmul(np.ascontiguousarray(dc.T),
                                                            np.ascontiguousarray(a.T)))


def test_matmul_backward_da_rows_do_not_depend_on_the_batch(L):
    g = rng(550)
    dc, a, w = normal_bf16(g, (600, 1024)), normal_bf16(g, (600, 512)), normal_bf16(g, (1024, 512), std=0.05)
    dcd, ad, wd = dev_bf16(dc), dev_bf16(a), dev_bf16(w)
    full, dw_full = L.bi_matmul_backward(dcd, ad, wd)
    for M in (1, 3, 256, 257, 599):
        da, _ = L.bi_matmul_backward(dcd[:M], ad[:M], wd, want_dw=False)
        assert same_bytes(da, full[:M]), M
    _, dw = L.bi_matmul_backward(dcd, ad, wd, want_da=False)
    assert same_bytes(dw, dw_full)


@pytest.mark.parametrize("T,F", [(1, 8), (37, 1408), (300, 120), (5, 14336)])
def test_swiglu_backward_parity(L, T, F):
    g = rng(560 + T + F)
    gate = normal_bf16(g, (T, F), std=2.0)
    gate[0, :4] = f32_to_bf16_bits(np.array([-100.0, -20.0, 20.0, 100.0], dtype=np.float32))[: min(4, F)]
    gu = np.concatenate([gate, normal_bf16(g, (T, F))], axis=1)
    dout = normal_bf16(g, (T, F))
    ref = oracle.swiglu_backward(gu, dout)
    for dt, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        out = L.bi_swiglu_backward(dev_bf16(gu), dev_bf16(dout), out_dtype=dt)
        assert np.all(np.isfinite(to_f64(out)))
        assert rowwise_normwise(to_f64(out), ref).max() <= tol, dt


def test_swiglu_backward_rows_do_not_depend_on_the_batch(L):
    g = rng(570)
    gu, dout = normal_bf16(g, (300, 2 * 1408), std=2.0), normal_bf16(g, (300, 1408))
    gud, dd = dev_bf16(gu), dev_bf16(dout)
    full = L.bi_swiglu_backward(gud, dd)
    for M in (1, 7, 299):
        assert same_bytes(L.bi_swiglu_backward(gud[:M], dd[:M]), full[:M]), M


@pytest.mark.parametrize("nh,d", [(8, 128), (32, 128), (3, 64)])
def test_rope_backward_parity(L, nh, d):
    g = rng(580 + nh + d)
    T = 77
    dy = normal_bf16(g, (T, nh, d))
    pos = g.integers(0, 32768, size=T).astype(np.int32)
    pos[0] = 0
    ref = oracle.rope_backward(dy, pos)
    pd = torch.from_numpy(pos).to("cuda")
    for dt, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        out = L.bi_rope_backward(dev_bf16(dy), pd, out_dtype=dt)
        assert rowwise_normwise(to_f64(out).reshape(T, -1), ref.reshape(T, -1)).max() <= tol, dt
    # position 0 is the identity
    out = L.bi_rope_backward(dev_bf16(dy), pd, out_dtype=torch.float32)
    np.testing.assert_array_equal(to_f64(out)[0], bf16_bits_to_f32(dy[0]).astype(np.float64))


def test_rope_backward_reads_and_writes_head_sets_of_wider_rows(L):
    # the q heads (first 32) and the k heads (next 8) of a fused q/k/v
    # gradient [T, (32 + 2 * 8) * 128], rotated in place of a copy
    g = rng(590)
    T, Hq, Hkv, d = 40, 32, 8, 128
    dqkv = normal_bf16(g, (T, (Hq + 2 * Hkv) * d))
    pos = torch.from_numpy(g.integers(0, 4096, size=T).astype(np.int32)).to("cuda")
    src = dev_bf16(dqkv)
    out = torch.zeros_like(src)
    v3 = lambda t, h0, n: t.view(T, Hq + 2 * Hkv, d)[:, h0:h0 + n]  # noqa: E731
    L.bi_rope_backward(v3(src, 0, Hq), pos, out=v3(out, 0, Hq))
    L.bi_rope_backward(v3(src, Hq, Hkv), pos, out=v3(out, Hq, Hkv))
    q_ref = L.bi_rope_backward(v3(src, 0, Hq).contiguous(), pos)
    k_ref = L.bi_rope_backward(v3(src, Hq, Hkv).contiguous(), pos)
    assert same_bytes(v3(out, 0, Hq).contiguous(), q_ref)
    assert same_bytes(v3(out, Hq, Hkv).contiguous(), k_ref)
    assert torch.count_nonzero(v3(out, Hq + Hkv, Hkv)) == 0  # the v part is untouched
