"""Negative controls: the variant-off build (split-K matmul, load-dependent
RMSNorm strategy, decode blocks that pre-merge their own split range) must
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
