"""Paged attention on the GPU: decode and (chunked) prefill against the fp64
oracle, and bitwise invariance across work division, batch composition,
page placement, pool contents and processing mode."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import DEV, TOL_BF16, dev_bf16, host_bits, rowwise_normwise, same_bytes, to_f64
from synth import (PagedKV, kv_from_blocks, kv_to_blocks, normal_bf16, page_table, paged_kv, rng,
                   slot_mapping, tiny_layer)

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-5


@pytest.fixture(scope="module")
def L():
    return bi.load()


def dev_kv(kv: PagedKV) -> bi.PagedKV:
    """Upload a logical cache in the device's page-block layout."""
    return bi.PagedKV(dev_bf16(kv_to_blocks(kv.k_cache)), dev_bf16(kv_to_blocks(kv.v_cache)),
                      torch.from_numpy(np.ascontiguousarray(kv.block_table)).to(DEV))


def i32(a):
    return torch.tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def decode_parity(L, kv: PagedKV, q_bits, **kw):
    B, Hq, d = q_bits.shape
    dkv = dev_kv(kv)
    o, lse = L.bi_attention_decode(dkv, dev_bf16(q_bits), i32(kv.seq_lens),
                                   int(kv.seq_lens.max()), want_lse=True, **kw)
    torch.cuda.synchronize()
    rows = oracle.decode_rows(q_bits, kv.seq_lens)
    ro, rl = oracle.attention(*rows, Hq, kv.k_cache, kv.v_cache, kv.block_table, want_lse=True)
    g = to_f64(o).reshape(B, Hq * d)
    err = rowwise_normwise(g, ro.reshape(B, Hq * d))
    assert err.max() <= TOL_BF16, "request %d: %.3g" % (err.argmax(), err.max())
    gl = to_f64(lse).reshape(B, Hq)
    lerr = rowwise_normwise(gl, rl.reshape(B, Hq))
    assert lerr.max() <= TOL_LSE, "lse of request %d: %.3g" % (lerr.argmax(), lerr.max())
    return o, lse


def test_decode_tiny_layer(L):
    c = tiny_layer()
    decode_parity(L, c["kv"], c["q"])


def test_decode_gqa_64_4(L):
    g = rng(21)
    lens = [1, 17, 256, 257, 1000, 3001]
    kv = paged_kv(g, lens, 4, 128, extra_pages=7)
    q = normal_bf16(g, (len(lens), 64, 128))
    decode_parity(L, kv, q)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_split_boundaries(L, d):
    g = rng(22 + d)
    lens = [1, 15, 16, 17, 255, 256, 257, 511, 512, 513, 768, 1025]
    kv = paged_kv(g, lens, 2, d)
    q = normal_bf16(g, (len(lens), 8, d))
    decode_parity(L, kv, q)
    decode_parity(L, kv, q, splits_per_cta=1)


@pytest.mark.parametrize("Hq,Hkv", [(40, 2), (48, 1), (100, 1), (128, 1)])
def test_decode_large_groups(L, Hq, Hkv):
    # Groups of 20, 48, 100 and 128 query heads: 5, 12, 25 and 32 rows in a
    # TMEM lane quarter, so the quarter's second softmax warp (rows 16..31)
    # and the upper 8 rows of each warp are used in decode too; the last
    # quarter of the 100-head group is ragged.  Oracle parity, and decode of
    # a sequence's last token equals its prefill bit for bit.
    g = rng(24 + Hq)
    lens = [1, 300, 777, 2049]
    kv = paged_kv(g, lens, Hkv, 128)
    q = normal_bf16(g, (len(lens), Hq, 128))
    o, _ = decode_parity(L, kv, q)
    S = lens[-1]
    qp = normal_bf16(rng(25 + Hq), (S, Hq, 128))
    qp[S - 1] = q[-1]
    one = PagedKV(kv.k_cache, kv.v_cache, kv.block_table[-1:], kv.seq_lens[-1:], Hkv, 128)
    op = L.bi_attention_prefill(dev_kv(one), dev_bf16(qp), i32([0, S]), i32([0]), S)
    assert same_bytes(op[S - 1], o[-1])


def test_decode_bits_do_not_depend_on_work_division(L):
    g = rng(23)
    lens = [5, 700, 2049, 4000, 300, 1]
    kv = paged_kv(g, lens, 4, 128)
    kv.block_table = np.pad(kv.block_table, ((0, 0), (0, 600 - kv.block_table.shape[1])),
                            constant_values=-1)
    q = dev_bf16(normal_bf16(g, (len(lens), 64, 128)))
    dkv, sl = dev_kv(kv), i32(kv.seq_lens)
    ref_o, ref_l = L.bi_attention_decode(dkv, q, sl, 4000, want_lse=True)
    for spc in (1, 2, 3, 5, 7, 16, 100):
        o, l = L.bi_attention_decode(dkv, q, sl, 4000, want_lse=True, splits_per_cta=spc)
        assert same_bytes(o, ref_o), spc
        assert same_bytes(l, ref_l), spc
    # a larger declared maximum changes the grid, not the bits
    o, l = L.bi_attention_decode(dkv, q, sl, 9000, want_lse=True)
    assert same_bytes(o, ref_o) and same_bytes(l, ref_l)


def relayout(kv: PagedKV, seed: int, extra: int, fill: str):
    """Same logical K/V, different physical pages, a pool of a different size,
    unused slots filled with `fill`."""
    g = rng(seed)
    bt, num_pages = page_table(g, kv.seq_lens, extra_pages=extra)
    shape = (num_pages,) + kv.k_cache.shape[1:]
    val = {"nan": 0x7FC0, "zero": 0, "inf": 0x7F80}[fill]
    k = np.full(shape, val, dtype=np.uint16)
    v = np.full(shape, val, dtype=np.uint16)
    for b, Lb in enumerate(kv.seq_lens):
        for j in range(int(Lb)):
            k[bt[b, j // 16], :, j % 16] = kv.k_cache[kv.block_table[b, j // 16], :, j % 16]
            v[bt[b, j // 16], :, j % 16] = kv.v_cache[kv.block_table[b, j // 16], :, j % 16]
    return PagedKV(k, v, bt, kv.seq_lens, kv.num_kv_heads, kv.head_dim)


def test_decode_bits_do_not_depend_on_batch_pages_or_pool(L):
    g = rng(24)
    lens = [300, 1, 2000, 513, 64, 1500, 9, 1024]
    kv = paged_kv(g, lens, 4, 128)
    q = normal_bf16(g, (len(lens), 64, 128))
    full_o = L.bi_attention_decode(dev_kv(kv), dev_bf16(q), i32(kv.seq_lens), 2000)
    # each request alone, on relocated pages in a NaN-filled pool
    for b in range(len(lens)):
        one = PagedKV(kv.k_cache, kv.v_cache, kv.block_table[b:b + 1], kv.seq_lens[b:b + 1], 4, 128)
        moved = relayout(one, seed=100 + b, extra=50, fill="nan")
        o = L.bi_attention_decode(dev_kv(moved), dev_bf16(q[b:b + 1]), i32(moved.seq_lens),
                                  int(lens[b]))
        assert same_bytes(o[0], full_o[b]), b
    # reversed batch order amid new neighbours
    g2 = rng(25)
    others = paged_kv(g2, [4000, 33, 700], 4, 128)
    qo = normal_bf16(g2, (3, 64, 128))
    big_lens = list(others.seq_lens) + lens[::-1]
    nk = others.k_cache.shape[0]
    k = np.concatenate([others.k_cache, kv.k_cache])
    v = np.concatenate([others.v_cache, kv.v_cache])
    mp = max(others.block_table.shape[1], kv.block_table.shape[1])
    bt = np.full((len(big_lens), mp), -1, dtype=np.int32)
    bt[:3, :others.block_table.shape[1]] = others.block_table
    rev = kv.block_table[::-1]
    bt[3:, :rev.shape[1]] = np.where(rev >= 0, rev + nk, -1)
    mix = PagedKV(k, v, bt, np.array(big_lens, dtype=np.int32), 4, 128)
    qq = np.concatenate([qo, q[::-1]])
    o = L.bi_attention_decode(dev_kv(mix), dev_bf16(qq), i32(mix.seq_lens), 4000)
    for i, b in enumerate(range(len(lens) - 1, -1, -1)):
        assert same_bytes(o[3 + i], full_o[b]), b


def test_decode_stale_nan_pool_never_leaks(L):
    g = rng(26)
    lens = [17, 250, 511, 1]
    kv = paged_kv(g, lens, 2, 128, extra_pages=5)
    q = normal_bf16(g, (4, 8, 128))
    zero = relayout(kv, 7, 5, "zero")
    nan = PagedKV(zero.k_cache.copy(), zero.v_cache.copy(), zero.block_table, zero.seq_lens, 2, 128)
    used = np.zeros(zero.k_cache.shape[0] * 16, dtype=bool)
    for b, Lb in enumerate(lens):
        for j in range(Lb):
            used[zero.block_table[b, j // 16] * 16 + j % 16] = True
    kf = nan.k_cache.reshape(-1, 2, 16, 128).transpose(0, 2, 1, 3).reshape(-1, 2, 128)
    vf = nan.v_cache.reshape(-1, 2, 16, 128).transpose(0, 2, 1, 3).reshape(-1, 2, 128)
    kf[~used] = 0x7FC0
    vf[~used] = 0x7F80
    nan.k_cache[:] = kf.reshape(-1, 16, 2, 128).transpose(0, 2, 1, 3)
    nan.v_cache[:] = vf.reshape(-1, 16, 2, 128).transpose(0, 2, 1, 3)
    oz = L.bi_attention_decode(dev_kv(zero), dev_bf16(q), i32(zero.seq_lens), 511)
    on = L.bi_attention_decode(dev_kv(nan), dev_bf16(q), i32(nan.seq_lens), 511)
    assert torch.isfinite(on.float()).all()
    assert same_bytes(oz, on)


# ---------------------------------------------------------------- prefill


def write_sequence(L, S, Hkv, d, k_bits, v_bits, chunk=None, seed=0, fill="nan"):
    """A fresh NaN-filled paged cache with one sequence written by bi_kv_write,
    chunk by chunk.  Returns (device cache, block table (host))."""
    g = rng(seed)
    bt, num_pages = page_table(g, [S], extra_pages=3)
    val = 0x7FC0 if fill == "nan" else 0
    k = torch.from_numpy(np.full((num_pages, Hkv, 16, d), val, dtype=np.uint16).view(np.int16))
    v = torch.from_numpy(np.full((num_pages, Hkv, 16, d), val, dtype=np.uint16).view(np.int16))
    dkv = bi.PagedKV(k.to(DEV).view(torch.bfloat16), v.to(DEV).view(torch.bfloat16),
                     torch.from_numpy(bt).to(DEV))
    chunk = chunk or S
    kd, vd = dev_bf16(k_bits), dev_bf16(v_bits)
    for c0 in range(0, S, chunk):
        n = min(chunk, S - c0)
        slots = torch.from_numpy(slot_mapping(bt, 0, np.arange(c0, c0 + n))).to(DEV)
        L.bi_kv_write(dkv, kd[c0:c0 + n].contiguous(), vd[c0:c0 + n].contiguous(), slots)
    return dkv, bt


def host_cache(dkv):
    """Download a device cache as logical [num_pages, Hkv, 16, d] arrays."""
    return kv_from_blocks(host_bits(dkv.k_cache)), kv_from_blocks(host_bits(dkv.v_cache))


def test_prefill_parity_with_context(L):
    g = rng(31)
    S, Hq, Hkv, d = 700, 8, 2, 128
    q = normal_bf16(g, (S, Hq, d))
    k = normal_bf16(g, (S, Hkv, d))
    v = normal_bf16(g, (S, Hkv, d))
    dkv, bt = write_sequence(L, S, Hkv, d, k, v)
    kc, vc = host_cache(dkv)
    # a chunk [300, 700) over a 300-token context, and the full sequence
    for c0 in (0, 300):
        n = S - c0
        o, lse = L.bi_attention_prefill(dkv, dev_bf16(q[c0:]), i32([0, n]), i32([c0]), n,
                                        want_lse=True)
        torch.cuda.synchronize()
        rs = np.zeros(n * Hq)
        rh = np.tile(np.arange(Hq), n)
        rp = np.repeat(np.arange(c0, S), Hq)
        ro, rl = oracle.attention(q[c0:].reshape(n * Hq, d), rs, rh, rp, Hq, kc, vc, bt,
                                  want_lse=True)
        err = rowwise_normwise(to_f64(o).reshape(n, Hq * d), ro.reshape(n, Hq * d))
        assert err.max() <= TOL_BF16, (c0, err.argmax(), err.max())
        lerr = rowwise_normwise(to_f64(lse).reshape(n, Hq), rl.reshape(n, Hq))
        assert lerr.max() <= TOL_LSE


def test_prefill_batch_of_sequences(L):
    g = rng(32)
    Hq, Hkv, d = 4, 4, 64
    lens = [130, 1, 257, 600]       # chunk lengths
    ctx = [0, 40, 300, 0]           # tokens already cached
    kv = paged_kv(g, [c + n for c, n in zip(ctx, lens)], Hkv, d)
    T = sum(lens)
    q = normal_bf16(g, (T, Hq, d))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    dkv = dev_kv(kv)
    o = L.bi_attention_prefill(dkv, dev_bf16(q), i32(cu), i32(ctx), max(lens))
    torch.cuda.synchronize()
    rs = np.repeat(np.repeat(np.arange(4), lens), Hq)
    rh = np.tile(np.arange(Hq), T)
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(ctx, lens)])
    rp = np.repeat(pos, Hq)
    ro = oracle.attention(q.reshape(T * Hq, d), rs, rh, rp, Hq, kv.k_cache, kv.v_cache,
                          kv.block_table)
    err = rowwise_normwise(to_f64(o).reshape(T, Hq * d), ro.reshape(T, Hq * d))
    assert err.max() <= TOL_BF16
    # each sequence alone gives the same bits
    for b in range(4):
        sub = PagedKV(kv.k_cache, kv.v_cache, kv.block_table[b:b + 1], kv.seq_lens[b:b + 1], Hkv, d)
        ob = L.bi_attention_prefill(dev_kv(sub), dev_bf16(q[cu[b]:cu[b + 1]]), i32([0, lens[b]]),
                                    i32([ctx[b]]), lens[b])
        assert same_bytes(ob, o[cu[b]:cu[b + 1]]), b


@pytest.mark.parametrize("d", [64, 128])
def test_decode_prefill_and_chunked_prefill_agree_bitwise(L, d):
    g = rng(33 + d)
    S, Hq, Hkv = 1100, 8, 2
    q = normal_bf16(g, (S, Hq, d))
    k = normal_bf16(g, (S, Hkv, d))
    v = normal_bf16(g, (S, Hkv, d))
    qd = dev_bf16(q)
    # full prefill
    dkv, bt = write_sequence(L, S, Hkv, d, k, v, seed=1)
    full_o, full_l = L.bi_attention_prefill(dkv, qd, i32([0, S]), i32([0]), S, want_lse=True)
    # chunked prefill, the cache written chunk by chunk before each chunk
    for chunk in (256, 512, 333):
        ckv, _ = write_sequence(L, S, Hkv, d, k, v, chunk=chunk, seed=2)
        outs, lses = [], []
        for c0 in range(0, S, chunk):
            n = min(chunk, S - c0)
            o, l = L.bi_attention_prefill(ckv, qd[c0:c0 + n].contiguous(), i32([0, n]), i32([c0]),
                                          n, want_lse=True)
            outs.append(o)
            lses.append(l)
        assert same_bytes(torch.cat(outs), full_o), chunk
        assert same_bytes(torch.cat(lses), full_l), chunk
    # decode of every token: request t sees keys 0..t
    dec_bt = torch.from_numpy(np.repeat(bt, S, axis=0)).to(DEV)
    dkv_dec = bi.PagedKV(dkv.k_cache, dkv.v_cache, dec_bt)
    o, l = L.bi_attention_decode(dkv_dec, qd, i32(np.arange(1, S + 1)), S, want_lse=True)
    assert same_bytes(o, full_o)
    assert same_bytes(l, full_l)


# ---------------------------------------------------------------- kv write / status


def test_kv_write_is_a_bit_exact_scatter(L):
    g = rng(41)
    kv = paged_kv(g, [40, 5, 77], 4, 128, extra_pages=4)
    kn = normal_bf16(g, (9, 4, 128))
    vn = normal_bf16(g, (9, 4, 128))
    slots = np.concatenate([slot_mapping(kv.block_table, 0, [0, 16, 39]), [-1],
                            slot_mapping(kv.block_table, 2, [3, 4, 5, 60, 76])])
    dkv = dev_kv(kv)
    L.bi_kv_write(dkv, dev_bf16(kn), dev_bf16(vn), torch.from_numpy(slots).to(DEV))
    kw, vw = kv.k_cache.copy(), kv.v_cache.copy()
    oracle.kv_write(kw, vw, kn, vn, slots)
    kd, vd = host_cache(dkv)
    np.testing.assert_array_equal(kd, kw)
    np.testing.assert_array_equal(vd, vw)
    assert L.bi_device_status() == bi.Status.OK


def test_kv_write_out_of_range_slot_is_flagged(L):
    g = rng(42)
    kv = paged_kv(g, [20], 1, 64)
    dkv = dev_kv(kv)
    before = host_bits(dkv.k_cache).copy()
    kn = normal_bf16(g, (1, 1, 64))
    L.bi_kv_write(dkv, dev_bf16(kn), dev_bf16(kn), torch.tensor([kv.num_pages * 16], device=DEV))
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX
    np.testing.assert_array_equal(host_bits(dkv.k_cache), before)  # untouched, any layout
    assert L.bi_device_status() == bi.Status.OK  # read-and-clear


def test_bad_page_id_is_flagged_not_faulted(L):
    g = rng(43)
    kv = paged_kv(g, [100], 1, 64)
    bt = kv.block_table.copy()
    bt[0, 3] = kv.num_pages + 1000
    bad = PagedKV(kv.k_cache, kv.v_cache, bt, kv.seq_lens, 1, 64)
    q = normal_bf16(g, (1, 1, 64))
    L.bi_attention_decode(dev_kv(bad), dev_bf16(q), i32([100]), 100)
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX
    decode_parity(L, kv, q)  # the context is still usable


def test_bounded_wait_gives_up_and_the_context_survives(L):
    L.bi_debug_bounded_wait(50_000_000)  # 50 ms on a barrier nothing arrives at
    assert L.bi_device_status() == bi.Status.TIMEOUT
    assert L.bi_device_status() == bi.Status.OK
    c = tiny_layer()
    decode_parity(L, c["kv"], c["q"])


def test_repeat_runs_are_identical(L):
    # the same decode and prefill calls made 100 times give the same bytes
    g = rng(51)
    lens = [5000, 1, 300, 2600]
    kv = paged_kv(g, lens, 4, 128)
    q = dev_bf16(normal_bf16(g, (4, 64, 128)))
    dkv, sl = dev_kv(kv), i32(kv.seq_lens)
    ref = L.bi_attention_decode(dkv, q, sl, 5000)
    S = 700
    qp = dev_bf16(normal_bf16(g, (S, 8, 128)))
    kp, vp = normal_bf16(g, (S, 2, 128)), normal_bf16(g, (S, 2, 128))
    pkv, _ = write_sequence(L, S, 2, 128, kp, vp, seed=5)
    refp = L.bi_attention_prefill(pkv, qp, i32([0, S]), i32([0]), S)
    for _ in range(100):
        assert same_bytes(L.bi_attention_decode(dkv, q, sl, 5000), ref)
        assert same_bytes(L.bi_attention_prefill(pkv, qp, i32([0, S]), i32([0]), S), refp)


def test_decode_long_sequence_merged_in_many_chunks(L):
    """A 70 001-key request has 274 split records per row: the ordered merge
    runs through several staged chunks, of 64 records when the batch has at
    most 512 rows and of 32 beyond.  Against the oracle alone, and the same
    bits alone and amid eleven other requests (768 rows)."""
    g = rng(31)
    lens = [70001] + [int(x) for x in g.integers(1, 6000, 11)]
    kv = paged_kv(g, lens, 4, 128)
    q = normal_bf16(g, (len(lens), 64, 128))
    one = PagedKV(kv.k_cache, kv.v_cache, kv.block_table[:1], kv.seq_lens[:1], 4, 128)
    alone, alone_l = decode_parity(L, one, q[:1])
    o, lse = L.bi_attention_decode(dev_kv(kv), dev_bf16(q), i32(kv.seq_lens), 70001, want_lse=True)
    assert same_bytes(o[0], alone[0])
    assert same_bytes(lse[0], alone_l[0])
    # and a work division that leaves every block one split
    o1, l1 = L.bi_attention_decode(dev_kv(kv), dev_bf16(q), i32(kv.seq_lens), 70001, want_lse=True,
                                   splits_per_cta=1)
    assert same_bytes(o1, o) and same_bytes(l1, lse)
    assert L.bi_device_status() == bi.Status.OK
