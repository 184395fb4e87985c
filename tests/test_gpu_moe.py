"""The mixture-of-experts kernels on the GPU: routing and dispatch exact
against the oracle (the same fp32 router logits), gate weights and the
combine within the parity bar, and a whole MoE feed-forward whose token rows
do not depend on the batch (the tokens each expert receives change with
it)."""
import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import DEV, TOL_BF16, TOL_F32, dev_bf16, host_bits, rowwise_normwise, same_bytes, to_f64
from invariant_bi_rmsnorm_03_b200.decoder import DecoderConfig, ToyDecoder, weight_shapes
from synth import normal_bf16, rng, toy_decoder_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return bi.load()


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (300, 16, 4), (257, 128, 8), (64, 256, 16)])
def test_route_and_dispatch_match_the_oracle(L, T, E, k):
    g = rng(170 + E)
    logits = g.integers(-6, 7, size=(T, E)).astype(np.float32)  # ties included
    logits += (g.standard_normal((T, E)) * 0.01).astype(np.float32) * (g.random((T, E)) < 0.5)
    ex, w = L.bi_moe_route(torch.from_numpy(logits).to(DEV), k)
    oex, ow = oracle.moe_route(logits, k)
    assert np.array_equal(ex.cpu().numpy(), oex)
    assert rowwise_normwise(w.cpu().numpy().astype(np.float64), ow).max() <= TOL_F32
    off, order, pos, tok = L.bi_moe_dispatch(ex, E)
    o_off, o_order, o_pos = oracle.moe_dispatch(oex, E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(order.cpu().numpy(), o_order)
    assert np.array_equal(pos.cpu().numpy(), o_pos)
    assert np.array_equal(tok.cpu().numpy(), o_order // k)
    assert L.bi_device_status() == bi.Status.OK


def test_combine_matches_the_oracle(L):
    g = rng(180)
    T, k, H = 97, 4, 4096
    y = normal_bf16(g, (T * k, H))
    pos = g.permutation(T * k).astype(np.int64)
    w = g.random((T, k)).astype(np.float32)
    w /= w.sum(axis=1, keepdims=True)
    out = L.bi_moe_combine(dev_bf16(y), torch.from_numpy(pos).to(DEV), torch.from_numpy(w).to(DEV))
    want = oracle.moe_combine(y, pos, w.astype(np.float64))
    assert rowwise_normwise(to_f64(out), want).max() <= TOL_BF16


def test_moe_feed_forward_rows_do_not_depend_on_the_batch(L):
    cfg = DecoderConfig(hidden=1024, layers=1, n_heads=8, n_kv_heads=2, head_dim=128, vocab=1000,
                        n_experts=16, top_k=4, expert_ffn=512)
    w = toy_decoder_weights(weight_shapes(cfg), seed=9, device=DEV)
    model = ToyDecoder(L, cfg, w, 4, DEV)
    g = rng(181)
    h = dev_bf16(normal_bf16(g, (300, cfg.hidden)))
    full = model._moe(h, 0)
    for sel in (np.array([5]), np.arange(10, 40), g.choice(300, 150, replace=False)):
        part = model._moe(h[torch.from_numpy(sel).to(DEV)].contiguous(), 0)
        assert same_bytes(part, full[torch.from_numpy(sel).to(DEV)]), len(sel)
    # and one token against the oracle: route, its k experts' feed-forwards, combine
    rl = L.bi_matmul(h[:1], w["l0.router"], out_dtype=torch.float32).cpu().numpy()
    ex, gw = oracle.moe_route(rl, cfg.top_k)
    acc = np.zeros(cfg.hidden)
    for i, e in enumerate(ex[0]):
        gu = L.bi_matmul(h[:1], w["l0.moe_wgu"][e])
        f = L.bi_swiglu(gu)
        want_f = oracle.swiglu(host_bits(gu))
        assert rowwise_normwise(to_f64(f), want_f).max() <= TOL_BF16
        yd = oracle.matmul(host_bits(f), host_bits(w["l0.moe_wdown"][e]))
        acc += gw[0, i] * yd[0]
    assert rowwise_normwise(to_f64(full[:1]), acc[None]).max() <= TOL_BF16


def test_degenerate_cases(L):
    g = rng(190)
    # k = E (every expert), a single expert, an empty batch
    for T, E, k in ((33, 4, 4), (20, 1, 1)):
        logits = g.standard_normal((T, E)).astype(np.float32)
        ex, w = L.bi_moe_route(torch.from_numpy(logits).to(DEV), k)
        oex, ow = oracle.moe_route(logits, k)
        assert np.array_equal(ex.cpu().numpy(), oex)
        assert rowwise_normwise(w.cpu().numpy().astype(np.float64), ow).max() <= TOL_F32
        off, order, pos, tok = L.bi_moe_dispatch(ex, E)
        o_off, o_order, o_pos = oracle.moe_dispatch(oex, E)
        assert np.array_equal(order.cpu().numpy(), o_order)
        assert np.array_equal(off.cpu().numpy(), o_off)
    ex0, w0 = L.bi_moe_route(torch.empty((0, 8), device=DEV), 2)
    assert ex0.shape == (0, 2)
    off0, _, _, _ = L.bi_moe_dispatch(ex0, 8)
    assert off0.cpu().numpy().tolist() == [0] * 9


def test_bad_expert_id_is_flagged_not_faulted(L):
    L.bi_device_status()
    ex = torch.tensor([[0, 1], [9, 2]], dtype=torch.int32, device=DEV)  # 9 >= E = 4
    off, order, pos, tok = L.bi_moe_dispatch(ex, 4)
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX
    assert pos.cpu().numpy()[2] == -1
    y = torch.zeros((4, 16), dtype=torch.bfloat16, device=DEV)
    w = torch.full((2, 2), 0.5, dtype=torch.float32, device=DEV)
    L.bi_moe_combine(y, pos, w)  # the unplaced entry is skipped, not read
    assert L.bi_device_status() == bi.Status.DEVICE_INDEX


@pytest.mark.parametrize("sizes", [[0, 1, 255, 256, 257], [513, 0, 0, 2, 100, 700, 31, 1]])
def test_grouped_matmul_equals_per_group_matmul_bitwise(L, sizes):
    # every group's rows through one grouped launch give the bits bi_matmul
    # gives them alone (same tile, same K order), and match the oracle
    g = rng(200 + len(sizes))
    G, N, K = len(sizes), 640, 1024
    rows = int(sum(sizes))
    a = normal_bf16(g, (rows, K))
    w = normal_bf16(g, (G, N, K), std=0.02)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ad, wd = dev_bf16(a), dev_bf16(w)
    c = L.bi_matmul_grouped(ad, wd, torch.from_numpy(off).to(DEV))
    for gi in range(G):
        lo, hi = int(off[gi]), int(off[gi + 1])
        if hi == lo:
            continue
        alone = L.bi_matmul(ad[lo:hi].contiguous(), wd[gi])
        assert same_bytes(c[lo:hi], alone), gi
        want = oracle.matmul(a[lo:hi], w[gi])
        assert rowwise_normwise(to_f64(c[lo:hi]), want).max() <= TOL_BF16
    assert L.bi_device_status() == bi.Status.OK
