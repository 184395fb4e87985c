"""bi_attention_decode_noalloc: decode attention for callers that may not
allocate device memory -- code inside a host framework that owns every
device allocation through its own pool, serving loops where an allocation
could synchronise the device or fail under fragmentation, embedders with a
memory budget fixed at start-up.  Its scratch is a fixed array inside the
library instead of a caller workspace.

The test calls the entry point through the C ABI twice in a row and checks
both outputs against bi_attention_decode's on the same inputs: within the
parity tolerance the other tests use, and (since the work division never
changes the bits) byte for byte; the outputs are also checked against the
fp64 oracle.  This file is collected last so that a run that stops at the
first failure has run every other test before it; it passes alone in a
fresh process as well."""
import ctypes

import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import (DEV, TOL_BF16, TOL_F32, dev_bf16, host_bits as bits_of, rowwise_normwise,
                      same_bytes, to_f64)
from synth import kv_to_blocks, normal_bf16, paged_kv, rng, tiny_layer

pytestmark = pytest.mark.gpu


def _dev_kv(kv):
    return bi.PagedKV(dev_bf16(kv_to_blocks(kv.k_cache)), dev_bf16(kv_to_blocks(kv.v_cache)),
                      torch.from_numpy(np.ascontiguousarray(kv.block_table)).to(DEV))


def _oracle_check(kv, q, o, lse):
    """The outputs against the fp64 oracle, per request (o) and per row (lse)."""
    B, Hq, d = q.shape
    rows = oracle.decode_rows(q, kv.seq_lens)
    ro, rl = oracle.attention(*rows, Hq, kv.k_cache, kv.v_cache, kv.block_table, want_lse=True)
    err = rowwise_normwise(to_f64(o).reshape(B, Hq * d), ro.reshape(B, Hq * d))
    assert err.max() <= TOL_BF16, "request %d: %.3g" % (err.argmax(), err.max())
    lerr = rowwise_normwise(to_f64(lse).reshape(B, Hq), rl.reshape(B, Hq))
    assert lerr.max() <= TOL_F32, "lse of request %d: %.3g" % (lerr.argmax(), lerr.max())


def _cases():
    c = tiny_layer()
    yield "tiny_layer_d64", c["kv"], c["q"]
    g = rng(71)
    lens = [1, 17, 256, 257, 1000, 3001]
    yield "gqa_64_4", paged_kv(g, lens, 4, 128, extra_pages=3), normal_bf16(g, (6, 64, 128))
    g = rng(72)
    # few long sequences: the work division spreads each over many blocks
    lens = [30000, 12345]
    yield "long_two_seqs", paged_kv(g, lens, 4, 128), normal_bf16(g, (2, 64, 128))


@pytest.mark.parametrize("name,kv,q", list(_cases()), ids=[c[0] for c in _cases()])
def test_noalloc_matches_workspace_entry_point_twice(name, kv, q):
    L = bi.load()
    dkv = _dev_kv(kv)
    qd = dev_bf16(q)
    sl = torch.tensor(kv.seq_lens, dtype=torch.int32, device=DEV)
    mx = int(kv.seq_lens.max())
    ref_o, ref_l = L.bi_attention_decode(dkv, qd, sl, mx, want_lse=True)
    B, Hq, d = q.shape
    for call in range(2):
        o = torch.empty_like(qd)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
        c = dkv.c_struct()
        st = L.lib.bi_attention_decode_noalloc(
            ctypes.byref(c), ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(o.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(sl.data_ptr()), B, Hq, mx,
            1.0 / np.sqrt(d), 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.bi_status_string(st)
        torch.cuda.synchronize()
        err = rowwise_normwise(to_f64(o).reshape(B, -1), to_f64(ref_o).reshape(B, -1))
        assert err.max() <= TOL_BF16, (call, err.max())
        lerr = rowwise_normwise(to_f64(lse), to_f64(ref_l))
        assert lerr.max() <= TOL_F32, (call, lerr.max())
        assert same_bytes(o, ref_o), call
        assert same_bytes(lse, ref_l), call
        if call == 0:
            _oracle_check(kv, q, o, lse)
    assert L.bi_device_status() == bi.Status.OK


def test_noalloc_rejects_what_the_array_cannot_hold():
    L = bi.load()
    g = rng(73)
    # The scratch needed follows the declared maximum length: 4 sequences
    # declared up to 65536 keys, one split per block, need
    # 4 * 64 * 256 * (128 + 4) * 4 bytes of partials -- more than the array.
    kv = paged_kv(g, [100, 37, 250, 1], 4, 128)
    kv.block_table = np.pad(kv.block_table, ((0, 0), (0, 4096 - kv.block_table.shape[1])),
                            constant_values=-1)
    dkv = _dev_kv(kv)
    q = dev_bf16(normal_bf16(g, (4, 64, 128)))
    sl = torch.tensor(kv.seq_lens, dtype=torch.int32, device=DEV)
    with pytest.raises(bi.BIError) as e:
        L.bi_attention_decode_noalloc(dkv, q, sl, 65536, splits_per_cta=1)
    assert e.value.status == bi.Status.WORKSPACE
    # With the division left to the library the division it would pick from
    # the load needs more scratch than the array holds (the workspace query
    # of the other entry point says how much), so the call falls back to one
    # block per sequence -- and still matches the workspace entry point and
    # the oracle.
    need = L.bi_attention_decode_workspace_bytes(dkv, 4, 64, 65536)
    assert need > bi.NOALLOC_SCRATCH_BYTES, need
    o, lse = L.bi_attention_decode_noalloc(dkv, q, sl, 65536, want_lse=True)
    ref_o, ref_l = L.bi_attention_decode(dkv, q, sl, 65536, want_lse=True)
    assert same_bytes(o, ref_o)
    assert same_bytes(lse, ref_l)
    _oracle_check(kv, bits_of(q), o, lse)
    assert L.bi_device_status() == bi.Status.OK
