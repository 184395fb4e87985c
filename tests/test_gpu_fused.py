"""The fused matmul forms on the GPU: the norm-weight fold (bit-exact: the
correctly rounded product), RMSNorm folded into the matmul (parity with the
fp64 oracle, bitwise batch invariance, its row statistics bi_rmsnorm's own)
and the residual matmul (equal bit for
bit to bi_matmul followed by the addition; parity with the oracle)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import (TOL_BF16, TOL_F32, dev_bf16, host_bits, rowwise_normwise, same_bytes,
                      to_f64)
from synth import bf16_bits_to_f32, f32_to_bf16_bits, norm_matmul, normal_bf16, rng, uniform_bf16

pytestmark = pytest.mark.gpu

EPS = 1e-6
SHAPES = [(1, 8, 8), (3, 264, 72), (129, 512, 136), (200, 776, 1000), (257, 256, 64),
          (300, 4096, 4096), (600, 1024, 8), (2048, 8192, 64)]


@pytest.fixture(scope="module")
def L():
    return bi.load()


def scaled_rows(g, M, K):
    """N(0, 1) rows times per-row scales 2^U(-6, 6): the norm has work to do."""
    x = normal_bf16(g, (M, K))
    s = np.exp2(g.uniform(-6, 6, size=(M, 1))).astype(np.float32)
    return f32_to_bf16_bits(bf16_bits_to_f32(x) * s)


def test_fold_is_the_correctly_rounded_product(L):
    g = rng(300)
    W = normal_bf16(g, (777, 520), std=0.02)
    w = uniform_bf16(g, (520,), 0.5, 1.5)
    want = f32_to_bf16_bits(oracle.fold_norm_weight(W, w).astype(np.float32))  # exact in fp32
    got = host_bits(L.bi_fold_norm_weight(dev_bf16(W), dev_bf16(w)))
    np.testing.assert_array_equal(got, want)
    Wd = dev_bf16(W)
    L.bi_fold_norm_weight(Wd, dev_bf16(w), out=Wd)  # in place
    np.testing.assert_array_equal(host_bits(Wd), want)


@pytest.mark.parametrize("M,K", [(1, 64), (37, 256), (300, 4096), (2048, 4096)])
def test_rmsnorm_matmul_row_scale_is_the_rmsnorm_rstd(L, M, K):
    # With the identity as the folded weight the product is x itself (exact
    # in fp32), so the fused form is round(r * x) -- which must equal
    # bi_rmsnorm with unit weights, round((x * rstd) * 1), exactly: the row
    # statistics are bi_rmsnorm's own reduction.  (Exactly in value: where x
    # holds -0 the tensor core's sum of +-0 products is +0, so only the sign
    # of such a zero may differ.)
    g = rng(310 + M + K)
    x = dev_bf16(scaled_rows(g, M, K))
    eye = dev_bf16(f32_to_bf16_bits(np.eye(K, dtype=np.float32)))
    ones = dev_bf16(f32_to_bf16_bits(np.ones(K, dtype=np.float32)))
    for dt in (torch.bfloat16, torch.float32):
        f = L.bi_rmsnorm_matmul(x, eye, EPS, out_dtype=dt)
        r = L.bi_rmsnorm(x, ones, EPS, out_dtype=dt)
        assert not torch.isnan(f).any()
        assert torch.equal(f, r), dt  # == on values: -0 equals +0
        nonzero = f != 0
        assert same_bytes(f[nonzero], r[nonzero]), dt


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_rmsnorm_matmul_parity(L, M, N, K):
    g = rng(310 + M + N + K)
    x = scaled_rows(g, M, K)
    wf = normal_bf16(g, (N, K), std=0.05)
    rows = np.arange(M) if M <= 300 else np.unique(np.concatenate(
        [[0, 127, 128, 255, 256, M - 1], g.integers(0, M, 40)]))
    ref = oracle.rmsnorm_matmul(x[rows], wf, EPS)
    for dt, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        c = L.bi_rmsnorm_matmul(dev_bf16(x), dev_bf16(wf), EPS, out_dtype=dt)
        err = rowwise_normwise(to_f64(c)[rows], ref)
        assert err.max() <= tol, (dt, rows[err.argmax()], err.max())


def test_rmsnorm_matmul_full_size_sampled_rows(L):
    c = norm_matmul(M=2048, N=12288)
    g = rng(320)
    w = c["w"]
    wf = L.bi_fold_norm_weight(dev_bf16(c["W"]), dev_bf16(w))
    rows = np.unique(np.concatenate([[0, 127, 128, 2047], g.integers(0, 2048, 24)]))
    ref = oracle.rmsnorm_matmul(c["x"][rows], host_bits(wf), EPS)
    out = L.bi_rmsnorm_matmul(dev_bf16(c["x"]), wf, EPS)
    err = rowwise_normwise(to_f64(out)[rows], ref)
    assert err.max() <= TOL_BF16, err.max()
    # the composition the fold stands for: RMSNorm with weight w, then W
    ref2 = oracle.matmul(f32_to_bf16_bits(oracle.rmsnorm(c["x"][rows], w, EPS).astype(np.float32)),
                         c["W"])
    assert rowwise_normwise(to_f64(out)[rows], ref2).max() <= TOL_BF16


def test_rmsnorm_matmul_rows_do_not_depend_on_the_batch(L):
    g = rng(330)
    x = dev_bf16(scaled_rows(g, 2048, 4096))
    wf = dev_bf16(normal_bf16(g, (4096, 4096), std=0.02))
    full = L.bi_rmsnorm_matmul(x, wf, EPS)
    for M in (1, 2, 3, 31, 127, 128, 129, 255, 256, 257, 1000, 1500, 2047):
        assert same_bytes(L.bi_rmsnorm_matmul(x[:M], wf, EPS), full[:M]), M
    perm = torch.from_numpy(g.permutation(2048)).to(x.device)
    assert same_bytes(L.bi_rmsnorm_matmul(x[perm].contiguous(), wf, EPS), full[perm])
    for _ in range(5):
        assert same_bytes(L.bi_rmsnorm_matmul(x, wf, EPS), full)


def test_rmsnorm_matmul_edge_rows(L):
    g = rng(340)
    x = scaled_rows(g, 5, 256)
    x[1] = 0                       # a zero row: rsqrt(eps) * 0 = 0
    x[3] = f32_to_bf16_bits(np.full(256, 3.0, np.float32))  # constant row: y = sign
    wf = normal_bf16(g, (264, 256), std=0.1)
    c = to_f64(L.bi_rmsnorm_matmul(dev_bf16(x), dev_bf16(wf), EPS, out_dtype=torch.float32))
    assert np.all(c[1] == 0.0)
    ref = oracle.rmsnorm_matmul(x, wf, EPS)
    assert rowwise_normwise(c, ref).max() <= TOL_F32
    assert L.bi_rmsnorm_matmul(dev_bf16(x[:0]), dev_bf16(wf), EPS).shape == (0, 264)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_residual_equals_matmul_then_add(L, M, N, K):
    g = rng(350 + M + N + K)
    a = dev_bf16(normal_bf16(g, (M, K)))
    w = dev_bf16(normal_bf16(g, (N, K), std=0.05))
    r = dev_bf16(normal_bf16(g, (M, N)))
    want = (r.float() + L.bi_matmul(a, w).float()).to(torch.bfloat16)
    assert same_bytes(L.bi_matmul_residual(a, w, r), want)
    r2 = r.clone()
    L.bi_matmul_residual(a, w, r2, out=r2)  # in place
    assert same_bytes(r2, want)


def test_residual_parity_with_the_oracle(L):
    g = rng(360)
    a, w, r = normal_bf16(g, (300, 1000)), normal_bf16(g, (776, 1000), std=0.05), \
        normal_bf16(g, (300, 776))
    out = L.bi_matmul_residual(dev_bf16(a), dev_bf16(w), dev_bf16(r))
    err = rowwise_normwise(to_f64(out), oracle.matmul_residual(r, a, w))
    assert err.max() <= TOL_BF16, err.max()


def test_residual_rows_do_not_depend_on_the_batch(L):
    c = norm_matmul(M=2048, N=4096)
    g = rng(370)
    a, w = dev_bf16(c["x"]), dev_bf16(c["W"])
    r = dev_bf16(normal_bf16(g, (2048, 4096)))
    full = L.bi_matmul_residual(a, w, r)
    for M in (1, 3, 129, 256, 257, 2047):
        assert same_bytes(L.bi_matmul_residual(a[:M], w, r[:M]), full[:M]), M


def test_fused_argument_errors(L):
    x = torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        L.bi_rmsnorm_matmul(x, torch.zeros((8, 12), dtype=torch.bfloat16, device="cuda"), EPS)
    x = torch.zeros((4, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        L.bi_rmsnorm_matmul(x, torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda"), -1.0)
    with pytest.raises(RuntimeError):
        L.bi_matmul_residual(x, torch.zeros((12, 16), dtype=torch.bfloat16, device="cuda"),
                             torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda"))


# ---------------------------------------------------------------- QKV epilogue

THETA = 10000.0


def qkv_case(seed, T, Hq, Hkv, d, K, num_pages=64, max_pos=4096):
    g = rng(seed)
    x = scaled_rows(g, T, K)
    wf = normal_bf16(g, ((Hq + 2 * Hkv) * d, K), std=0.05)
    pos = g.integers(0, max_pos, size=T).astype(np.int32)
    slots = g.permutation(num_pages * 16)[:T].astype(np.int64)  # one slot per token
    slots[::7] = -1                                           # rows that write no cache
    return x, wf, pos, slots


def caches(num_pages, Hkv, d):
    return [torch.zeros((num_pages, Hkv, 16, d), dtype=torch.bfloat16, device="cuda")
            for _ in range(2)]


@pytest.mark.parametrize("T,Hq,Hkv,d,K", [(1, 32, 8, 128, 4096), (3, 8, 2, 64, 512),
                                          (130, 32, 8, 128, 4096), (300, 8, 2, 128, 1000),
                                          (257, 4, 4, 64, 256), (129, 3, 1, 128, 256)])
def test_qkv_epilogue_equals_the_two_launches(L, T, Hq, Hkv, d, K):
    # one tile may hold q and k heads, or k and v heads; N need not fill the last tile
    x, wf, pos, slots = qkv_case(400 + T + d, T, Hq, Hkv, d, K, num_pages=max(64, T // 8))
    np_ = max(64, T // 8)
    table = L.bi_rope_table(4096, d, THETA)
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    k1, v1 = caches(np_, Hkv, d)
    k2, v2 = caches(np_, Hkv, d)
    xd, wd = dev_bf16(x), dev_bf16(wf)
    pd, sd = torch.from_numpy(pos).cuda(), torch.from_numpy(slots).cuda()
    L.bi_device_status()
    q1 = L.bi_rmsnorm_matmul_rope_kv(xd, wd, EPS, bi.PagedKV(k1, v1, bt), table, pd, sd, Hq)
    qkv = L.bi_rmsnorm_matmul(xd, wd, EPS)
    q2 = L.bi_rope_kv_write(bi.PagedKV(k2, v2, bt), qkv, pd, sd, Hq, THETA)
    assert L.bi_device_status() == bi.Status.OK
    assert same_bytes(q1, q2)
    assert same_bytes(k1, k2) and same_bytes(v1, v2)
    if (slots >= 0).any():  # some row wrote its slot
        assert bool(torch.any(k1 != 0)) and bool(torch.any(v1 != 0))


def test_qkv_epilogue_parity_with_the_oracle(L):
    T, Hq, Hkv, d, K = 40, 8, 2, 128, 512
    x, wf, pos, slots = qkv_case(410, T, Hq, Hkv, d, K)
    table = L.bi_rope_table(4096, d, THETA)
    q = L.bi_rmsnorm_matmul_rope_kv(dev_bf16(x), dev_bf16(wf), EPS,
                                    bi.PagedKV(*caches(64, Hkv, d),
                                               torch.zeros((1, 1), dtype=torch.int32,
                                                           device="cuda")),
                                    table, torch.from_numpy(pos).cuda(),
                                    torch.from_numpy(slots).cuda(), Hq)
    # the oracle's chain: RMSNorm -> matmul (rounded to bf16, as the fused op's
    # product is) -> RoPE at each token's position
    prod = f32_to_bf16_bits(oracle.rmsnorm_matmul(x, wf, EPS).astype(np.float32))
    want = oracle.rope(prod[:, :Hq * d].reshape(T, Hq, d), pos, THETA)
    err = rowwise_normwise(to_f64(q).reshape(T, -1), want.reshape(T, -1))
    assert err.max() <= TOL_BF16, err.max()


def test_qkv_epilogue_rows_do_not_depend_on_the_batch(L):
    T, Hq, Hkv, d, K = 300, 32, 8, 128, 4096
    x, wf, pos, slots = qkv_case(420, T, Hq, Hkv, d, K)
    slots[:] = -1  # q only
    table = L.bi_rope_table(4096, d, THETA)
    kv = bi.PagedKV(*caches(64, Hkv, d), torch.zeros((1, 1), dtype=torch.int32, device="cuda"))
    xd, wd = dev_bf16(x), dev_bf16(wf)
    pd, sd = torch.from_numpy(pos).cuda(), torch.from_numpy(slots).cuda()
    full = L.bi_rmsnorm_matmul_rope_kv(xd, wd, EPS, kv, table, pd, sd, Hq)
    for M in (1, 2, 129, 256, 257):
        part = L.bi_rmsnorm_matmul_rope_kv(xd[:M], wd, EPS, kv, table, pd[:M], sd[:M], Hq)
        assert same_bytes(part, full[:M]), M


def test_rope_table_is_the_rounded_angles(L):
    for d in (64, 128):
        got = L.bi_rope_table(3000, d, THETA).cpu().numpy().astype(np.float64)
        want = oracle.rope_angles(3000, d, THETA)
        ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(got - want) <= ulp), d


def test_qkv_epilogue_bad_position_and_slot(L):
    T, Hq, Hkv, d, K = 20, 4, 2, 64, 256
    x, wf, pos, slots = qkv_case(430, T, Hq, Hkv, d, K, max_pos=100)
    table = L.bi_rope_table(100, d, THETA)
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    kv = bi.PagedKV(*caches(64, Hkv, d), bt)
    pos[5] = 100           # past the table: the row writes nothing
    slots[6] = 64 * 16     # past the cache: q is written, k and v are not
    q = torch.zeros((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    L.bi_device_status()
    L.bi_rmsnorm_matmul_rope_kv(dev_bf16(x), dev_bf16(wf), EPS, kv, table,
                                torch.from_numpy(pos).cuda(), torch.from_numpy(slots).cuda(), Hq,
                                q_out=q)
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX
    assert not bool(torch.any(q[5] != 0)) and bool(torch.any(q[6] != 0))
