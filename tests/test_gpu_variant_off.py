"""Negative controls: the variant-off build (split-K matmul, load-dependent
RMSNorm strategy, decode split ranges whose size follows the load, each
block pre-merging its own range) must
FAIL the invariance checks that the batch-invariant build passes.  This shows
the byte comparisons can detect a batch-dependent reduction order, and that
the invariant build passes them for the reason it is built for (float
addition is not associative: the same numbers summed in another grouping
give other bits)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
from gpu_util import DEV, TOL_BF16, dev_bf16, rowwise_normwise, same_bytes, to_f64
from synth import kv_to_blocks, norm_matmul, normal_bf16, paged_kv, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    lib = bi.load(variant=True)
    assert lib.bi_build_invariant() == 0
    return lib


@pytest.fixture(scope="module")
def L():
    return bi.load()


def test_float_addition_is_not_associative():
    # The mechanism the pages name: (a + b) + c != a + (b + c).
    a, b, c = np.float32(1e8), np.float32(-1e8), np.float32(1.0)
    assert (a + b) + c != a + (b + c)


def test_variant_matmul_rows_change_with_batch_size(V, L):
    c = norm_matmul(M=2048, N=4096)
    x, W = dev_bf16(c["x"]), dev_bf16(c["W"])
    full_v = V.bi_matmul(x, W, out_dtype=torch.float32)
    full_i = L.bi_matmul(x, W, out_dtype=torch.float32)
    small_v = V.bi_matmul(x[:8], W, out_dtype=torch.float32)  # split-K at small M
    small_i = L.bi_matmul(x[:8], W, out_dtype=torch.float32)
    assert same_bytes(small_i, full_i[:8])
    assert not same_bytes(small_v, full_v[:8])
    # both are still correct results
    err = rowwise_normwise(to_f64(small_v), to_f64(full_v[:8]))
    assert err.max() < 1e-4


def test_variant_rmsnorm_rows_change_with_batch_size(V, L):
    c = norm_matmul(M=2048)
    x, w = dev_bf16(c["x"]), dev_bf16(c["w"])
    full_v = V.bi_rmsnorm(x, w, c["eps"], out_dtype=torch.float32)
    small_v = V.bi_rmsnorm(x[:16], w, c["eps"], out_dtype=torch.float32)
    full_i = L.bi_rmsnorm(x, w, c["eps"], out_dtype=torch.float32)
    small_i = L.bi_rmsnorm(x[:16], w, c["eps"], out_dtype=torch.float32)
    assert same_bytes(small_i, full_i[:16])
    assert not same_bytes(small_v, full_v[:16])


def _dev_kv(kv):
    return bi.PagedKV(dev_bf16(kv_to_blocks(kv.k_cache)), dev_bf16(kv_to_blocks(kv.v_cache)),
                      torch.from_numpy(np.ascontiguousarray(kv.block_table)).to(DEV))


def test_variant_decode_bits_change_with_work_division(V, L):
    g = rng(81)
    lens = [4000, 2500, 3000]
    kv = paged_kv(g, lens, 4, 128)
    q = dev_bf16(normal_bf16(g, (3, 64, 128)))
    dkv, sl = _dev_kv(kv), torch.tensor(lens, dtype=torch.int32, device=DEV)
    ref_i = L.bi_attention_decode(dkv, q, sl, 4000, splits_per_cta=100)
    ref_v = V.bi_attention_decode(dkv, q, sl, 4000, splits_per_cta=100)
    assert same_bytes(ref_i, ref_v)  # one block per sequence: the same arithmetic
    differs = False
    for spc in (1, 2, 3, 5):
        assert same_bytes(L.bi_attention_decode(dkv, q, sl, 4000, splits_per_cta=spc), ref_i)
        o_v = V.bi_attention_decode(dkv, q, sl, 4000, splits_per_cta=spc)
        differs |= not same_bytes(o_v, ref_v)
        err = rowwise_normwise(to_f64(o_v).reshape(3, -1), to_f64(ref_v).reshape(3, -1))
        assert err.max() <= TOL_BF16
    assert differs


def test_variant_decode_split_size_follows_the_load(V, L):
    # The variant-off decode cuts each sequence into ranges of ceil(L / count)
    # keys (count chosen from the load), so a token's decode output differs
    # from its prefill output -- the mismatch the invariant build removes
    # (there, decode of the last token equals prefill bit for bit).
    from synth import page_table, slot_mapping
    g = rng(82)
    S, Hq, Hkv, d = 2900, 8, 2, 128
    q = normal_bf16(g, (S, Hq, d))
    k, v = normal_bf16(g, (S, Hkv, d)), normal_bf16(g, (S, Hkv, d))
    bt, npg = page_table(g, [S])
    i32 = lambda a: torch.tensor(a, dtype=torch.int32, device=DEV)  # noqa: E731
    differs = False
    for lib, invariant in ((L, True), (V, False)):
        kv = bi.PagedKV(torch.zeros((npg, Hkv, 16, d), dtype=torch.bfloat16, device=DEV),
                        torch.zeros((npg, Hkv, 16, d), dtype=torch.bfloat16, device=DEV),
                        torch.from_numpy(bt).to(DEV))
        lib.bi_kv_write(kv, dev_bf16(k), dev_bf16(v),
                        torch.from_numpy(slot_mapping(bt, 0, np.arange(S))).to(DEV))
        op = lib.bi_attention_prefill(kv, dev_bf16(q), i32([0, S]), i32([0]), S)
        # the last token decoded in a batch of 16 copies: 16 x 2 kv heads
        # against 148 SMs gives 6 blocks per sequence, so the variant cuts
        # the 2900 keys into ranges of 496 (pieces at 0, 256, 496, 752, ...)
        dec = bi.PagedKV(kv.k_cache, kv.v_cache, torch.from_numpy(np.repeat(bt, 16, axis=0)).to(DEV))
        qd = dev_bf16(np.repeat(q[S - 1:], 16, axis=0))
        od = lib.bi_attention_decode(dec, qd, i32([S] * 16), S)
        same = same_bytes(od[0], op[S - 1])
        if invariant:
            assert same
        else:
            differs = not same
            err = rowwise_normwise(to_f64(od[0]).reshape(1, -1), to_f64(op[S - 1]).reshape(1, -1))
            assert err.max() <= TOL_BF16
    assert differs
