"""Attention backward on the GPU (bi_attention_backward): dq, dk and dv
against the fp64 oracle's backward, the same bits on every run, and each
sequence's gradients independent of the rest of the batch.

The parity measure is the attention one: normwise per sequence (its rows of
dq over all heads and positions; its keys' dk and dv over all kv heads).
dq, dk and dv are bf16 outputs (P and dS enter the tensor core as bf16, as
the forward's P does), so the bar is the bf16 one."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import DEV, TOL_BF16, dev_bf16, host_bits, normwise, same_bytes, to_f64
from synth import PagedKV, bf16_bits_to_f32, kv_from_blocks, kv_to_blocks, normal_bf16, paged_kv, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


def i32(a):
    return torch.tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def dev_kv(kv: PagedKV) -> bi.PagedKV:
    return bi.PagedKV(dev_bf16(kv_to_blocks(kv.k_cache)), dev_bf16(kv_to_blocks(kv.v_cache)),
                      torch.from_numpy(np.ascontiguousarray(kv.block_table)).to(DEV))


def case(seed, lens, ctx, Hq, Hkv, d, fill="normal"):
    g = rng(seed)
    kv = paged_kv(g, [c + n for c, n in zip(ctx, lens)], Hkv, d, extra_pages=3, fill_unused=fill)
    T = int(sum(lens))
    q = normal_bf16(g, (T, Hq, d))
    dout = normal_bf16(g, (T, Hq, d))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return kv, q, dout, cu


def run(L, kv, q, dout, cu, ctx, dkv=None):
    dkv = dkv or dev_kv(kv)
    lens = np.diff(cu)
    qd, dd = dev_bf16(q), dev_bf16(dout)
    o, lse = L.bi_attention_prefill(dkv, qd, i32(cu), i32(ctx), int(lens.max()), want_lse=True)
    max_kv = int(max(c + n for c, n in zip(ctx, lens)))
    dq, dk, dv = L.bi_attention_backward(dkv, qd, o, dd, lse, i32(cu), i32(ctx), int(lens.max()),
                                         max_kv)
    torch.cuda.synchronize()
    assert L.bi_device_status() == bi.Status.OK
    return dq, dk, dv


def oracle_rows(q, dout, cu, ctx, Hq):
    T, _, d = q.shape
    lens = np.diff(cu)
    seq = np.repeat(np.arange(len(lens)), lens)
    pos = np.concatenate([np.arange(c, c + n) for c, n in zip(ctx, lens)])
    return (q.reshape(T * Hq, d), dout.reshape(T * Hq, d), np.repeat(seq, Hq),
            np.tile(np.arange(Hq), T), np.repeat(pos, Hq))


def check_parity(kv, q, dout, cu, ctx, dq, dk, dv):
    T, Hq, d = q.shape
    qr, dr, rs, rh, rp = oracle_rows(q, dout, cu, ctx, Hq)
    rdq, rdk, rdv = oracle.attention_backward(qr, dr, rs, rh, rp, Hq, kv.k_cache, kv.v_cache,
                                              kv.block_table)
    gdq = to_f64(dq).reshape(T * Hq, d)
    gdk = bf16_bits_to_f32(kv_from_blocks(host_bits(dk))).astype(np.float64)
    gdv = bf16_bits_to_f32(kv_from_blocks(host_bits(dv))).astype(np.float64)
    worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for b in range(len(cu) - 1):
        rows = slice(int(cu[b]) * Hq, int(cu[b + 1]) * Hq)
        worst["dq"] = max(worst["dq"], normwise(gdq[rows], rdq[rows]))
        L_b = int(ctx[b] + cu[b + 1] - cu[b])
        pages = kv.block_table[b, :(L_b + 15) // 16]
        keys = np.zeros((len(pages), 16), dtype=bool)
        keys.reshape(-1)[:L_b] = True
        for name, gx, rx in (("dk", gdk, rdk), ("dv", gdv, rdv)):
            sel_g = gx[pages].transpose(0, 2, 1, 3)[keys]   # [keys, Hkv, d]
            sel_r = rx[pages].transpose(0, 2, 1, 3)[keys]
            worst[name] = max(worst[name], normwise(sel_g, sel_r))
            # slots past the sequence's end in its last page are written as 0
            tail = gx[pages].transpose(0, 2, 1, 3)[~keys]
            assert np.all(tail == 0), (name, b)
    for name, e in worst.items():
        assert e <= TOL_BF16, (name, e)
    return worst


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (2, 2, 64), (4, 1, 128)])
def test_backward_parity_split_and_block_edges(L, Hq, Hkv, d):
    # chunk lengths cross the 128-row tile and 128-key block edges (127/128/129)
    # and the forward's 256-key splits (255/256/257)
    lens = [1, 127, 129, 256, 257]
    ctx = [0, 0, 0, 0, 0]
    kv, q, dout, cu = case(600 + Hq + d, lens, ctx, Hq, Hkv, d)
    dq, dk, dv = run(L, kv, q, dout, cu, ctx)
    check_parity(kv, q, dout, cu, ctx, dq, dk, dv)


def test_backward_parity_with_context_and_stale_pool(L):
    # chunks over cached context (the keys of earlier chunks get gradients
    # from this chunk's rows only); the unused slots of the pool hold NaN
    lens = [100, 1, 300]
    ctx = [200, 511, 40]
    kv, q, dout, cu = case(610, lens, ctx, 8, 2, 128, fill="nan")
    dq, dk, dv = run(L, kv, q, dout, cu, ctx)
    check_parity(kv, q, dout, cu, ctx, dq, dk, dv)


def test_backward_decoder_shapes(L):
    # the toy decoder's attention: 32 query and 8 kv heads of 128
    lens = [300, 45]
    ctx = [0, 0]
    kv, q, dout, cu = case(620, lens, ctx, 32, 8, 128)
    dq, dk, dv = run(L, kv, q, dout, cu, ctx)
    check_parity(kv, q, dout, cu, ctx, dq, dk, dv)


def test_backward_same_bits_every_run_and_independent_of_the_batch(L):
    lens = [200, 37, 400]
    ctx = [0, 60, 0]
    Hq, Hkv, d = 8, 2, 128
    kv, q, dout, cu = case(630, lens, ctx, Hq, Hkv, d)
    dkv = dev_kv(kv)
    dq, dk, dv = run(L, kv, q, dout, cu, ctx, dkv)
    for _ in range(3):
        dq2, dk2, dv2 = run(L, kv, q, dout, cu, ctx, dkv)
        assert same_bytes(dq2, dq) and same_bytes(dk2, dk) and same_bytes(dv2, dv)
    # each sequence alone (its own page table row) gives the same bits for
    # its rows of dq and its pages of dk and dv
    for b in range(len(lens)):
        sub = PagedKV(kv.k_cache, kv.v_cache, kv.block_table[b:b + 1], kv.seq_lens[b:b + 1], Hkv, d)
        dsub = bi.PagedKV(dkv.k_cache, dkv.v_cache,
                          torch.from_numpy(np.ascontiguousarray(sub.block_table)).to(DEV))
        rows = slice(int(cu[b]), int(cu[b + 1]))
        dqb, dkb, dvb = run(L, sub, q[rows], dout[rows], np.array([0, lens[b]], dtype=np.int32),
                            [ctx[b]], dsub)
        assert same_bytes(dqb, dq[rows]), b
        pages = torch.from_numpy(kv.block_table[b, :(ctx[b] + lens[b] + 15) // 16].astype(np.int64)).to(DEV)
        assert same_bytes(dkb[pages], dk[pages]), b
        assert same_bytes(dvb[pages], dv[pages]), b


def test_backward_dq_rows_do_not_depend_on_the_chunking(L):
    # the same query rows processed as one chunk or as the tail chunk over a
    # cached context give the same dq bits (the rows see the same keys; the
    # key blocks are aligned to key 0 in both)
    g = rng(640)
    S, Hq, Hkv, d = 400, 4, 2, 128
    kv = paged_kv(g, [S], Hkv, d)
    q = normal_bf16(g, (S, Hq, d))
    dout = normal_bf16(g, (S, Hq, d))
    dkv = dev_kv(kv)
    dq_full, _, _ = run(L, kv, q, dout, np.array([0, S], dtype=np.int32), [0], dkv)
    c0 = 130
    dq_tail, _, _ = run(L, kv, q[c0:], dout[c0:], np.array([0, S - c0], dtype=np.int32), [c0], dkv)
    assert same_bytes(dq_tail, dq_full[c0:])
