"""The toy decoder's glue kernels on the GPU (bi_add_rmsnorm, bi_embedding,
bi_rope_kv_write, bi_swiglu, bi_argmax): parity with the fp64 oracle on the
same seeded inputs, and bitwise batch invariance (a row's output bytes do not
depend on the other rows of the call)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import DEV, TOL_BF16, TOL_F32, dev_bf16, host_bits, rowwise_normwise, same_bytes, to_f64
from synth import (bf16_bits_to_f32, kv_from_blocks, normal_bf16, page_table, rng, slot_mapping,
                   uniform_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


def i32(a):
    return torch.as_tensor(np.asarray(a, dtype=np.int32)).to(DEV)


def i64(a):
    return torch.as_tensor(np.asarray(a, dtype=np.int64)).to(DEV)


# ---------------------------------------------------------------- residual + RMSNorm


@pytest.mark.parametrize("H,M", [(4096, 1), (4096, 37), (4096, 600), (256, 9), (16384, 5)])
def test_add_rmsnorm_parity(L, H, M):
    g = rng(60 + M)
    x, delta = normal_bf16(g, (M, H)), normal_bf16(g, (M, H), std=0.5)
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    xd = dev_bf16(x)
    y = L.bi_add_rmsnorm(xd, dev_bf16(delta), dev_bf16(w), 1e-6)
    torch.cuda.synchronize()
    s_ref, y_ref = oracle.add_rmsnorm(x, delta, w, 1e-6)
    assert rowwise_normwise(to_f64(xd), s_ref).max() <= TOL_BF16
    assert rowwise_normwise(to_f64(y), y_ref).max() <= TOL_BF16
    # the residual is round(fp32(x) + fp32(delta)): within half a bf16 ulp
    assert np.all(np.abs(to_f64(xd) - s_ref) <= np.abs(s_ref) * 2.0 ** -8 * 1.01 + 1e-30)


def test_add_rmsnorm_fp32_output_parity(L):
    g = rng(66)
    x, delta = normal_bf16(g, (64, 4096)), normal_bf16(g, (64, 4096))
    w = uniform_bf16(g, (4096,), 0.5, 1.5)
    xd = dev_bf16(x)
    y = L.bi_add_rmsnorm(xd, dev_bf16(delta), dev_bf16(w), 1e-6, out_dtype=torch.float32)
    # the fp32 output normalises the rounded residual: compare with the
    # oracle's RMSNorm of the device's residual row
    ref = oracle.rmsnorm(host_bits(xd), w, 1e-6)
    assert rowwise_normwise(to_f64(y), ref).max() <= TOL_F32


def test_add_rmsnorm_equals_plain_rmsnorm_of_the_updated_rows(L):
    g = rng(67)
    x, delta = normal_bf16(g, (300, 4096)), normal_bf16(g, (300, 4096))
    w = dev_bf16(uniform_bf16(g, (4096,), 0.5, 1.5))
    xd = dev_bf16(x)
    y = L.bi_add_rmsnorm(xd, dev_bf16(delta), w, 1e-6)
    assert same_bytes(y, L.bi_rmsnorm(xd, w, 1e-6))


def test_add_rmsnorm_rows_independent_of_batch(L):
    g = rng(68)
    x, delta = normal_bf16(g, (2048, 4096)), normal_bf16(g, (2048, 4096))
    w = dev_bf16(uniform_bf16(g, (4096,), 0.5, 1.5))
    xf = dev_bf16(x)
    yf = L.bi_add_rmsnorm(xf, dev_bf16(delta), w, 1e-6)
    for M in (1, 2, 3, 64, 255, 1000):
        xm = dev_bf16(x[:M])
        ym = L.bi_add_rmsnorm(xm, dev_bf16(delta[:M]), w, 1e-6)
        assert same_bytes(xm, xf[:M]) and same_bytes(ym, yf[:M]), M


# ---------------------------------------------------------------- embedding


def test_embedding_bit_exact(L):
    g = rng(70)
    table = normal_bf16(g, (32000, 4096), std=0.02)
    ids = g.integers(0, 32000, size=300).astype(np.int32)
    out = L.bi_embedding(dev_bf16(table), i32(ids))
    assert np.array_equal(host_bits(out), oracle.embedding(table, ids))


def test_embedding_bad_id_flags_status(L):
    table = dev_bf16(normal_bf16(rng(71), (10, 64)))
    L.bi_device_status()  # clear
    out = torch.zeros((2, 64), dtype=torch.bfloat16, device=DEV)
    L.bi_embedding(table, i32([3, 10]), out=out)
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX
    assert same_bytes(out[0], table[3]) and not bool(out[1].view(torch.int16).any())


# ---------------------------------------------------------------- RoPE + KV write


def _rope_case(seed, T, Hq, Hkv, d, max_pos=32768):
    g = rng(seed)
    qkv = normal_bf16(g, (T, (Hq + 2 * Hkv) * d))
    pos = g.integers(0, max_pos, size=T).astype(np.int32)
    bt, num_pages = page_table(g, [T], extra_pages=3)
    slots = slot_mapping(bt, 0, np.arange(T))
    return qkv, pos, bt, num_pages, slots


@pytest.mark.parametrize("T,Hq,Hkv,d", [(1, 32, 8, 128), (77, 32, 8, 128), (300, 4, 1, 64),
                                         (40, 64, 4, 128)])
def test_rope_kv_write_parity(L, T, Hq, Hkv, d):
    qkv, pos, bt, num_pages, slots = _rope_case(80 + T, T, Hq, Hkv, d)
    kc = torch.zeros((num_pages, Hkv, 16, d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    kv = bi.PagedKV(kc, vc, i32(bt))
    q = L.bi_rope_kv_write(kv, dev_bf16(qkv), i32(pos), i64(slots), Hq)
    torch.cuda.synchronize()
    parts = qkv.reshape(T, Hq + 2 * Hkv, d)
    q_ref = oracle.rope(np.ascontiguousarray(parts[:, :Hq]), pos)
    k_ref = oracle.rope(np.ascontiguousarray(parts[:, Hq:Hq + Hkv]), pos)
    assert rowwise_normwise(to_f64(q).reshape(T * Hq, d), q_ref.reshape(T * Hq, d)).max() <= TOL_BF16
    k_logical = kv_from_blocks(host_bits(kc))
    v_logical = kv_from_blocks(host_bits(vc))
    k_rows = np.stack([k_logical[s // 16, :, s % 16] for s in slots])  # [T, Hkv, d]
    v_rows = np.stack([v_logical[s // 16, :, s % 16] for s in slots])
    k_dev = bf16_bits_to_f32(k_rows).astype(np.float64)
    assert rowwise_normwise(k_dev.reshape(T * Hkv, d), k_ref.reshape(T * Hkv, d)).max() <= TOL_BF16
    assert np.array_equal(v_rows, np.ascontiguousarray(parts[:, Hq + Hkv:]))


def test_rope_position_zero_is_exact(L):
    qkv, _, bt, num_pages, slots = _rope_case(90, 5, 8, 2, 128)
    kv = bi.PagedKV(torch.zeros((num_pages, 2, 16, 128), dtype=torch.bfloat16, device=DEV),
                    torch.zeros((num_pages, 2, 16, 128), dtype=torch.bfloat16, device=DEV),
                    i32(bt))
    q = L.bi_rope_kv_write(kv, dev_bf16(qkv), i32([0] * 5), i64(slots), 8)
    assert np.array_equal(host_bits(q), qkv.reshape(5, 12, 128)[:, :8])


def test_rope_rows_independent_of_batch(L):
    T, Hq, Hkv, d = 200, 32, 8, 128
    qkv, pos, bt, num_pages, slots = _rope_case(91, T, Hq, Hkv, d)

    def run(sel):
        kv = bi.PagedKV(torch.zeros((num_pages, Hkv, 16, d), dtype=torch.bfloat16, device=DEV),
                        torch.zeros((num_pages, Hkv, 16, d), dtype=torch.bfloat16, device=DEV),
                        i32(bt))
        q = L.bi_rope_kv_write(kv, dev_bf16(qkv[sel]), i32(pos[sel]), i64(slots[sel]), Hq)
        return q, kv

    q_all, kv_all = run(np.arange(T))
    for sel in (np.array([17]), np.arange(5, 9), np.array([199, 3, 50])):
        q, kv = run(sel)
        assert same_bytes(q, q_all[torch.as_tensor(sel).to(DEV)])
        kb, kab = kv_from_blocks(host_bits(kv.k_cache)), kv_from_blocks(host_bits(kv_all.k_cache))
        for s in slots[sel]:
            assert np.array_equal(kb[s // 16, :, s % 16], kab[s // 16, :, s % 16])


def test_rope_bad_slot_flags_status(L):
    qkv, pos, bt, num_pages, slots = _rope_case(92, 3, 4, 1, 64)
    kv = bi.PagedKV(torch.zeros((num_pages, 1, 16, 64), dtype=torch.bfloat16, device=DEV),
                    torch.zeros((num_pages, 1, 16, 64), dtype=torch.bfloat16, device=DEV), i32(bt))
    L.bi_device_status()
    slots = slots.copy()
    slots[1] = num_pages * 16
    L.bi_rope_kv_write(kv, dev_bf16(qkv), i32(pos), i64(slots), 4)
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX


# ---------------------------------------------------------------- SwiGLU


@pytest.mark.parametrize("T,F", [(1, 14336), (33, 14336), (5, 512)])
def test_swiglu_parity(L, T, F):
    g = rng(100 + T)
    gu = normal_bf16(g, (T, 2 * F), std=2.0)
    out = L.bi_swiglu(dev_bf16(gu))
    assert rowwise_normwise(to_f64(out), oracle.swiglu(gu)).max() <= TOL_BF16


def test_swiglu_extreme_gates(L):
    # very negative gates: silu -> -0 (e^-g overflows to inf), no NaN
    gu = np.concatenate([np.full((1, 8), 0xC700, np.uint16),   # gate -32768
                         np.full((1, 8), 0x3F80, np.uint16)], axis=1)  # up 1.0
    out = to_f64(L.bi_swiglu(dev_bf16(gu)))
    assert np.all(np.isfinite(out)) and np.all(out == 0.0)


def test_swiglu_rows_independent_of_batch(L):
    g = rng(110)
    gu = normal_bf16(g, (257, 2 * 14336), std=2.0)
    full = L.bi_swiglu(dev_bf16(gu))
    for sel in (slice(0, 1), slice(100, 103), slice(256, 257)):
        assert same_bytes(L.bi_swiglu(dev_bf16(gu[sel])), full[sel])


# ---------------------------------------------------------------- argmax


@pytest.mark.parametrize("T", [1, 7, 600])
def test_argmax_matches_oracle(L, T):
    g = rng(120 + T)
    logits = (g.standard_normal((T, 32000)) * 1.3).astype(np.float32)
    out = L.bi_argmax(torch.from_numpy(logits).to(DEV))
    assert np.array_equal(out.cpu().numpy(), oracle.argmax(logits))


def test_argmax_ties_and_infinities(L):
    g = rng(130)
    logits = g.integers(-3, 4, size=(64, 32000)).astype(np.float32)  # many ties
    logits[5] = -np.inf
    logits[6, 31999] = np.inf
    logits[7, :] = 2.0
    out = L.bi_argmax(torch.from_numpy(logits).to(DEV)).cpu().numpy()
    assert np.array_equal(out, oracle.argmax(logits))
    assert out[5] == 0 and out[6] == 31999 and out[7] == 0
