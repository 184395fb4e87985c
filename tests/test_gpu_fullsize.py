"""Attention at the workloads' full sizes.

* Paged decode, GQA 64/4, d = 128, lengths U(1, 32768): four target requests
  drawn once are byte-compared in every batch size from 1 to 256, each batch
  filled with other random requests (random lengths, random pages of a
  shared pool, random queries), so the work division the launch picks from
  the load changes with B.  The targets are also checked against the fp64
  oracle, every head.
* Causal prefill of one 8192-token prompt, 32/8 heads, d = 128: full
  prefill, chunked prefill with chunks 256, 512 and 1024, and decode of
  every token give the same bytes for every token; sampled tokens are
  checked against the oracle.
"""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import (DEV, TOL_BF16, TOL_F32, dev_bf16, host_bits, normwise, rowwise_normwise,
                      same_bytes, to_f64)
from synth import (kv_from_blocks, normal_bf16, prefill, rng, slot_mapping,
                   torch_normal_bf16)

pytestmark = pytest.mark.gpu

HQ, HKV, D, PAGE, MAXLEN = 64, 4, 128, 16, 32768


@pytest.fixture(scope="module")
def L():
    return bi.load()


def i32(a):
    return torch.as_tensor(np.asarray(a, dtype=np.int32)).to(DEV)


def test_decode_targets_identical_in_every_batch_size_1_to_256(L):
    g = rng(200)
    pool = 40000                                   # pages shared by every batch
    shape = (pool, HKV, PAGE, D)
    k = torch_normal_bf16(shape, 3000, DEV)
    v = torch_normal_bf16(shape, 3001, DEV)
    max_pages = MAXLEN // PAGE
    # four targets: one key, a partial split, a long one, the longest
    t_lens = np.array([1, 257, 16389, MAXLEN], dtype=np.int32)
    t_pages = [g.choice(pool, size=(n + PAGE - 1) // PAGE, replace=False).astype(np.int32)
               for n in t_lens]
    t_q = normal_bf16(g, (4, HQ, D))

    def run(B, seed):
        gb = rng(seed)
        lens = gb.integers(1, MAXLEN + 1, size=B).astype(np.int32)
        q = normal_bf16(gb, (B, HQ, D))
        bt = np.full((B, max_pages), -1, dtype=np.int32)
        for b in range(B):
            n = (lens[b] + PAGE - 1) // PAGE
            bt[b, :n] = gb.integers(0, pool, size=n)
        slots = gb.permutation(B)[:min(4, B)]    # where the targets sit
        for i, s in enumerate(slots):
            lens[s] = t_lens[i]
            q[s] = t_q[i]
            bt[s] = -1
            bt[s, :len(t_pages[i])] = t_pages[i]
        kv = bi.PagedKV(k, v, torch.from_numpy(bt).to(DEV))
        o = L.bi_attention_decode(kv, dev_bf16(q), i32(lens), MAXLEN)
        return o, slots

    ref, slots = run(4, 0)
    ref = [ref[slots[i]].clone() for i in range(4)]
    for B in range(1, 257):
        o, slots = run(B, 1000 + B)
        for i, s in enumerate(slots):
            assert same_bytes(o[s], ref[i]), (B, i)
    assert L.bi_device_status() == bi.Status.OK

    # the targets against the fp64 oracle, all 64 heads
    for i in range(4):
        pages = torch.from_numpy(t_pages[i].astype(np.int64)).to(DEV)
        kc = kv_from_blocks(host_bits(k.index_select(0, pages)))
        vc = kv_from_blocks(host_bits(v.index_select(0, pages)))
        bt1 = np.arange(len(t_pages[i]), dtype=np.int32)[None, :]
        rows = oracle.decode_rows(t_q[i:i + 1], [int(t_lens[i])])
        want = oracle.attention(*rows, HQ, kc, vc, bt1)
        err = rowwise_normwise(to_f64(ref[i]).reshape(HQ, D), want)
        assert err.max() <= TOL_BF16, (i, err.max())


def test_prefill_8192_modes_bitwise_and_sampled_parity(L):
    c = prefill(seed=3)
    S, Hq, Hkv, d = 8192, c["Hq"], c["Hkv"], c["d"]
    q, kbits, vbits = dev_bf16(c["q"]), dev_bf16(c["k"]), dev_bf16(c["v"])
    bt_np = c["block_table"]

    def fresh_cache():
        shape = (c["num_pages"], Hkv, PAGE, d)
        nan = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=DEV)
        return bi.PagedKV(nan, nan.clone(), torch.from_numpy(bt_np).to(DEV))

    def write(kv, c0, n):
        slots = torch.from_numpy(slot_mapping(bt_np, 0, np.arange(c0, c0 + n))).to(DEV)
        L.bi_kv_write(kv, kbits[c0:c0 + n].contiguous(), vbits[c0:c0 + n].contiguous(), slots)

    kv = fresh_cache()
    write(kv, 0, S)
    full_o, full_l = L.bi_attention_prefill(kv, q, i32([0, S]), i32([0]), S, want_lse=True)
    for chunk in (256, 512, 1024):
        ckv = fresh_cache()
        outs, lses = [], []
        for c0 in range(0, S, chunk):
            write(ckv, c0, chunk)
            o, l = L.bi_attention_prefill(ckv, q[c0:c0 + chunk].contiguous(), i32([0, chunk]),
                                          i32([c0]), chunk, want_lse=True)
            outs.append(o)
            lses.append(l)
        assert same_bytes(torch.cat(outs), full_o), chunk
        assert same_bytes(torch.cat(lses), full_l), chunk
    # decode of every token: request t is the prompt's first t + 1 tokens
    dec = bi.PagedKV(kv.k_cache, kv.v_cache, torch.from_numpy(np.repeat(bt_np, S, axis=0)).to(DEV))
    od, ld = L.bi_attention_decode(dec, q, i32(np.arange(1, S + 1)), S, want_lse=True)
    assert same_bytes(od, full_o)
    assert same_bytes(ld, full_l)
    assert L.bi_device_status() == bi.Status.OK

    # sampled tokens and heads against the fp64 oracle
    kc, vc = kv_from_blocks(host_bits(kv.k_cache)), kv_from_blocks(host_bits(kv.v_cache))
    # the split and tile edges in every head, plus 256 random (token, head)
    # pairs over the whole prompt
    ts = np.array([0, 1, 127, 128, 255, 256, 257, 4095, 8191])
    tt, hh = np.meshgrid(ts, np.arange(Hq), indexing="ij")
    gs = np.random.default_rng(7)
    tt = np.concatenate([tt.ravel(), gs.integers(0, S, 256)])
    hh = np.concatenate([hh.ravel(), gs.integers(0, Hq, 256)])
    rows = np.stack([c["q"][t, h] for t, h in zip(tt, hh)])
    want, want_lse = oracle.attention(rows, np.zeros(len(tt)), hh, tt, Hq, kc, vc, bt_np,
                                      want_lse=True)
    got = to_f64(full_o)[tt, hh]
    assert rowwise_normwise(got, want).max() <= TOL_BF16
    got_l = full_l.cpu().numpy().astype(np.float64)[tt, hh]
    assert normwise(got_l, want_lse) <= TOL_F32
