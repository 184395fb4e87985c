"""Pins for the fp64 oracle: closed forms, brute force on tiny inputs and
independent library routines.  No GPU; each pin is chosen so that a plausible
slip in the oracle (a dropped term, a wrong index, a transposed operand, a
misplaced eps, a wrong head mapping, a causal off-by-one) fails it."""
import math

import numpy as np
import pytest
import torch

import oracle as _oracle_mod
from synth import (bf16_bits_to_f32, f32_to_bf16_bits, normal_bf16, page_table, paged_kv, rng,
                   slot_mapping, uniform_bf16)


@pytest.fixture
def oracle():
    return _oracle_mod.default()


def bf(vals):
    return f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def widen(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- RMSNorm


@pytest.mark.parametrize("c", [1.0, -2.5, 0.001, 96.0])
def test_rmsnorm_constant_row_closed_form(oracle, c):
    # x = c * 1  =>  mean(x^2) = c^2  =>  y = c / sqrt(c^2 + eps) * w
    H, eps = 64, 1e-6
    g = rng(11)
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    x = np.tile(bf([c] * H), (2, 1))
    y = oracle.rmsnorm(x, w, eps)
    cc = float(widen(bf([c]))[0])
    want = cc / math.sqrt(cc * cc + eps) * widen(w)
    np.testing.assert_allclose(y[0], want, rtol=1e-14, atol=0)
    np.testing.assert_allclose(y[1], want, rtol=1e-14, atol=0)


def test_rmsnorm_alternating_sign_closed_form(oracle):
    H, eps, c = 32, 1e-6, 1.5
    x = bf([c if i % 2 == 0 else -c for i in range(H)])[None, :]
    w = bf(np.ones(H))
    y = oracle.rmsnorm(x, w, eps)[0]
    mag = c / math.sqrt(c * c + eps)
    want = np.array([mag if i % 2 == 0 else -mag for i in range(H)])
    np.testing.assert_allclose(y, want, rtol=1e-14)


def test_rmsnorm_hand_example(oracle):
    # x = [1, 2, 3, 4]: mean square (1+4+9+16)/4 = 7.5; eps = 0
    x = bf([1, 2, 3, 4])[None, :]
    w = bf([1, 0.5, 2, 1])
    y = oracle.rmsnorm(x, w, 0.0)[0]
    r = 1.0 / math.sqrt(7.5)
    np.testing.assert_allclose(y, [1 * r, 2 * r * 0.5, 3 * r * 2, 4 * r], rtol=1e-15)


def test_rmsnorm_eps_inside_the_root(oracle):
    # c = 1e-3: c^2 = 1e-6 = eps, so y = c / sqrt(2e-6) = 1/sqrt(2) (eps inside)
    # whereas eps outside the root would give c / (c + eps) ~ 0.999.
    c = float(widen(bf([1e-3]))[0])
    x = bf([1e-3] * 8)[None, :]
    y = oracle.rmsnorm(x, bf(np.ones(8)), 1e-6)[0]
    np.testing.assert_allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-14)
    assert abs(y[0] - 1 / math.sqrt(2)) < 0.01


def test_rmsnorm_matches_torch_fp64(oracle):
    g = rng(12)
    x = normal_bf16(g, (5, 96))
    w = uniform_bf16(g, (96,), 0.5, 1.5)
    y = oracle.rmsnorm(x, w, 1e-6)
    xt = torch.from_numpy(widen(x))
    want = torch.nn.functional.rms_norm(xt, (96,), weight=torch.from_numpy(widen(w)), eps=1e-6)
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-14)


def test_rmsnorm_scale_invariance_without_eps(oracle):
    g = rng(13)
    x = normal_bf16(g, (3, 40))
    x2 = bf(widen(x) * 4.0)  # exact: scaling by a power of two
    w = uniform_bf16(g, (40,), 0.5, 1.5)
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 0.0), oracle.rmsnorm(x2, w, 0.0), rtol=1e-14)


def test_rmsnorm_rows_independent(oracle):
    g = rng(14)
    x = normal_bf16(g, (6, 24))
    w = uniform_bf16(g, (24,), 0.5, 1.5)
    full = oracle.rmsnorm(x, w, 1e-6)
    for r in range(6):
        np.testing.assert_array_equal(oracle.rmsnorm(x[r:r + 1], w, 1e-6)[0], full[r])


# ---------------------------------------------------------------- matmul


def test_matmul_identity_weight(oracle):
    g = rng(20)
    a = normal_bf16(g, (7, 16))
    eye = bf(np.eye(16))
    np.testing.assert_array_equal(oracle.matmul(a, eye), widen(a))


def test_matmul_one_hot_rows_select_columns(oracle):
    g = rng(21)
    a = normal_bf16(g, (4, 12))
    pick = [3, 0, 11, 5, 5]
    w = np.zeros((5, 12), dtype=np.float32)
    for n, k in enumerate(pick):
        w[n, k] = 1.0
    c = oracle.matmul(a, bf(w))
    np.testing.assert_array_equal(c, widen(a)[:, pick])


def test_matmul_small_integers_brute_force(oracle):
    # M=3, N=5, K=7: distinct sizes so a transposed operand cannot pass.
    g = rng(22)
    A = g.integers(-8, 9, size=(3, 7))
    W = g.integers(-8, 9, size=(5, 7))
    c = oracle.matmul(bf(A), bf(W))
    for m in range(3):
        for n in range(5):
            assert c[m, n] == sum(int(A[m, k]) * int(W[n, k]) for k in range(7))


def test_matmul_hand_example(oracle):
    # [[1, 2, 3], [4, 5, 6]] times the transpose of [[1, 0, -1], [2, 1, 0]]
    c = oracle.matmul(bf([[1, 2, 3], [4, 5, 6]]), bf([[1, 0, -1], [2, 1, 0]]))
    np.testing.assert_array_equal(c, [[1 - 3, 2 + 2], [4 - 6, 8 + 5]])


def test_matmul_matches_torch_fp64(oracle):
    g = rng(23)
    a = normal_bf16(g, (9, 130))
    w = normal_bf16(g, (33, 130), std=0.02)
    want = torch.from_numpy(widen(a)) @ torch.from_numpy(widen(w)).T
    np.testing.assert_allclose(oracle.matmul(a, w), want.numpy(), rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- kv_write


def test_kv_write_matches_direct_scatter(oracle):
    g = rng(30)
    Hkv, d = 2, 8
    bt, num_pages = page_table(g, [37, 5], extra_pages=3)
    kc = normal_bf16(g, (num_pages, Hkv, 16, d))
    vc = normal_bf16(g, (num_pages, Hkv, 16, d))
    kn = normal_bf16(g, (6, Hkv, d))
    vn = normal_bf16(g, (6, Hkv, d))
    slots = np.concatenate([slot_mapping(bt, 0, [0, 17, 36]), [-1], slot_mapping(bt, 1, [2, 4])])
    k2, v2 = kc.copy(), vc.copy()
    oracle.kv_write(k2, v2, kn, vn, slots)
    kw, vw = kc.copy(), vc.copy()
    for t, s in enumerate(slots):
        if s >= 0:
            kw[s // 16, :, s % 16, :] = kn[t]
            vw[s // 16, :, s % 16, :] = vn[t]
    np.testing.assert_array_equal(k2, kw)
    np.testing.assert_array_equal(v2, vw)
    assert not np.array_equal(k2, kc)


# ---------------------------------------------------------------- attention


def _contig_cache(K, V):
    """Place logical K/V [L, Hkv, d] on pages 0, 1, 2, ... in order."""
    L, Hkv, d = K.shape
    n = (L + 15) // 16
    kc = np.zeros((n, Hkv, 16, d), dtype=np.uint16)
    vc = np.zeros_like(kc)
    for j in range(L):
        kc[j // 16, :, j % 16] = K[j]
        vc[j // 16, :, j % 16] = V[j]
    return kc, vc, np.arange(n, dtype=np.int32)[None, :]


def test_attention_identical_keys_give_prefix_mean(oracle):
    # Every key equal => uniform softmax over keys 0..t => o = mean(V[0..t]).
    g = rng(40)
    L, Hkv, d = 40, 1, 8
    k0 = normal_bf16(g, (d,))
    K = np.tile(k0, (L, Hkv, 1))
    V = normal_bf16(g, (L, Hkv, d))
    kc, vc, bt = _contig_cache(K, V)
    q = normal_bf16(g, (L, d))
    pos = np.arange(L)
    o, lse = oracle.attention(q, np.zeros(L), np.zeros(L), pos, 1, kc, vc, bt, want_lse=True)
    Vw = widen(V)[:, 0, :]
    for t in range(L):
        np.testing.assert_allclose(o[t], Vw[: t + 1].mean(axis=0), rtol=1e-12, atol=1e-14)
        s = float(widen(q[t]) @ widen(k0)) / math.sqrt(d)
        assert abs(lse[t] - (s + math.log(t + 1))) < 1e-12


def test_attention_single_key_returns_value_row(oracle):
    g = rng(41)
    kv = paged_kv(g, [1, 1, 1], num_kv_heads=2, head_dim=16)
    q = normal_bf16(g, (3, 4, 16))
    rows = _oracle_mod.decode_rows(q, kv.seq_lens)
    o = oracle.attention(*rows, 4, kv.k_cache, kv.v_cache, kv.block_table)
    for i, (b, h) in enumerate(zip(rows[1], rows[2])):
        page = kv.block_table[b, 0]
        np.testing.assert_array_equal(o[i], widen(kv.v_cache[page, h // 2, 0]))


def test_attention_dominant_logit_closed_form(oracle):
    # keys are scaled basis vectors; q = lam * e_j gives logit Delta on key j
    # and 0 elsewhere: o = (e^Delta v_j + sum_{i != j} v_i) / (e^Delta + L - 1)
    g = rng(42)
    L, d, j, lam = 12, 16, 7, 4.0
    K = np.zeros((L, 1, d), dtype=np.float32)
    for i in range(L):
        K[i, 0, i] = 1.0
    V = normal_bf16(g, (L, 1, d))
    kc, vc, bt = _contig_cache(bf(K), V)
    qv = np.zeros(d, dtype=np.float32)
    qv[j] = lam
    o = oracle.attention(bf(qv)[None], [0], [0], [L - 1], 1, kc, vc, bt, scale=1.0)[0]
    Vw = widen(V)[:, 0, :]
    e = math.exp(lam)
    want = (e * Vw[j] + Vw.sum(axis=0) - Vw[j]) / (e + L - 1)
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-14)


def test_attention_gqa_head_mapping(oracle):
    # V of kv head g is the constant g + 1, so head h must return h // (Hq/Hkv) + 1.
    g = rng(43)
    Hq, Hkv, d = 8, 2, 4
    kv = paged_kv(g, [20, 33], Hkv, d)
    for gg in range(Hkv):
        kv.v_cache[:, gg] = bf([gg + 1.0])[0]
    q = normal_bf16(g, (2, Hq, d))
    rows = _oracle_mod.decode_rows(q, kv.seq_lens)
    o = oracle.attention(*rows, Hq, kv.k_cache, kv.v_cache, kv.block_table)
    for i, h in enumerate(rows[2]):
        np.testing.assert_allclose(o[i], np.full(d, h // (Hq // Hkv) + 1.0), rtol=1e-14)


def test_attention_is_causal(oracle):
    g = rng(44)
    L, d = 30, 8
    K = normal_bf16(g, (L, 1, d))
    V = normal_bf16(g, (L, 1, d))
    q = normal_bf16(g, (1, d))
    t = 17
    kc, vc, bt = _contig_cache(K, V)
    base = oracle.attention(q, [0], [0], [t], 1, kc, vc, bt)
    K2, V2 = K.copy(), V.copy()
    K2[t + 1:] = normal_bf16(g, (L - t - 1, 1, d))
    V2[t + 1:] = normal_bf16(g, (L - t - 1, 1, d))
    kc2, vc2, _ = _contig_cache(K2, V2)
    np.testing.assert_array_equal(oracle.attention(q, [0], [0], [t], 1, kc2, vc2, bt), base)
    V3 = V.copy()
    V3[t] = normal_bf16(g, (1, d))
    kc3, vc3, _ = _contig_cache(K, V3)
    assert not np.array_equal(oracle.attention(q, [0], [0], [t], 1, kc3, vc3, bt), base)


def test_attention_paging_is_transparent(oracle):
    # Same logical K/V on shuffled pages vs on contiguous pages: equal in fp64.
    g = rng(45)
    lens = [50, 3, 129]
    Hq, Hkv, d = 4, 2, 16
    kv = paged_kv(g, lens, Hkv, d, extra_pages=5)
    q = normal_bf16(g, (3, Hq, d))
    rows = _oracle_mod.decode_rows(q, kv.seq_lens)
    got = oracle.attention(*rows, Hq, kv.k_cache, kv.v_cache, kv.block_table)
    for b, L in enumerate(lens):
        K = np.stack([kv.k_cache[kv.block_table[b, j // 16], :, j % 16] for j in range(L)])
        V = np.stack([kv.v_cache[kv.block_table[b, j // 16], :, j % 16] for j in range(L)])
        kc, vc, bt = _contig_cache(K, V)
        sel = rows[1] == b
        o = oracle.attention(rows[0][sel], np.zeros(sel.sum()), rows[2][sel], rows[3][sel], Hq, kc, vc, bt)
        np.testing.assert_array_equal(o, got[sel])


def test_attention_matches_torch_sdpa_fp64(oracle):
    g = rng(46)
    S, Hq, Hkv, d = 70, 4, 2, 16
    Q = normal_bf16(g, (S, Hq, d))
    K = normal_bf16(g, (S, Hkv, d))
    V = normal_bf16(g, (S, Hkv, d))
    kc, vc, bt = _contig_cache(K, V)
    rs = np.zeros(S * Hq)
    rh = np.tile(np.arange(Hq), S)
    rp = np.repeat(np.arange(S), Hq)
    o = oracle.attention(Q.reshape(S * Hq, d), rs, rh, rp, Hq, kc, vc, bt).reshape(S, Hq, d)
    qt = torch.from_numpy(widen(Q)).permute(1, 0, 2)
    kt = torch.from_numpy(widen(K)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    vt = torch.from_numpy(widen(V)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    mask = torch.ones(S, S, dtype=torch.bool).tril()
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    np.testing.assert_allclose(o, want.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_attention_brute_force_tiny(oracle):
    # d = 2, three keys, scale 1: written out by hand.
    K = bf([[1, 0], [0, 1], [1, 1]])[:, None, :]
    V = bf([[2, 0], [0, 4], [-2, 2]])[:, None, :]
    kc, vc, bt = _contig_cache(K, V)
    q = bf([[0.5, -1.0]])
    o, lse = oracle.attention(q, [0], [0], [2], 1, kc, vc, bt, scale=1.0, want_lse=True)
    s = [0.5, -1.0, -0.5]
    e = [math.exp(x - 0.5) for x in s]
    Z = sum(e)
    want = [(2 * e[0] - 2 * e[2]) / Z, (4 * e[1] + 2 * e[2]) / Z]
    np.testing.assert_allclose(o[0], want, rtol=1e-14)
    assert abs(lse[0] - (0.5 + math.log(Z))) < 1e-14


# ---------------------------------------------------------------- decoder glue
# Pins for the toy decoder's elementwise operations (embedding, rotary
# position embedding, SwiGLU, residual + RMSNorm, greedy argmax).


def test_embedding_rows_carry_their_ids(oracle):
    # Row v of the table holds the value v in every column: the gathered
    # rows must decode to the requested ids, in the requested order.
    V, H = 256, 16  # integers up to 256 are exact in bfloat16
    table = np.repeat(bf(np.arange(V, dtype=np.float32))[:, None], H, axis=1)
    ids = np.array([5, 0, 255, 5, 17], dtype=np.int32)
    out = oracle.embedding(table, ids)
    assert np.array_equal(widen(out), np.repeat(ids[:, None], H, axis=1).astype(np.float64))


def test_embedding_matches_fancy_indexing(oracle):
    g = rng(41)
    table = normal_bf16(g, (1000, 64))
    ids = g.integers(0, 1000, size=37).astype(np.int32)
    assert np.array_equal(oracle.embedding(table, ids), table[ids])


def test_rope_position_zero_is_identity(oracle):
    g = rng(42)
    x = normal_bf16(g, (3, 2, 8))
    out = oracle.rope(x, [0, 0, 0])
    assert np.array_equal(out, widen(x))


def test_rope_hand_example(oracle):
    # d = 4, theta = 10000: pair (x0, x2) turns by pos * 1, pair (x1, x3) by
    # pos * 10000^(-1/2) = pos / 100.
    x = bf([1.0, 2.0, 3.0, -1.0]).reshape(1, 1, 4)
    out = oracle.rope(x, [2])[0, 0]
    a0, a1 = 2.0, 0.02
    want = [1.0 * math.cos(a0) - 3.0 * math.sin(a0),
            2.0 * math.cos(a1) - (-1.0) * math.sin(a1),
            3.0 * math.cos(a0) + 1.0 * math.sin(a0),
            -1.0 * math.cos(a1) + 2.0 * math.sin(a1)]
    np.testing.assert_allclose(out, want, rtol=1e-14, atol=1e-15)


def test_rope_matches_complex_rotation(oracle):
    # The same rotation as multiplication by e^{i angle} of z = x_i + i x_{i+d/2}.
    g = rng(43)
    T, nh, d, theta = 5, 3, 128, 10000.0
    x = normal_bf16(g, (T, nh, d))
    pos = np.array([0, 1, 63, 300, 32767], dtype=np.int32)
    out = oracle.rope(x, pos, theta)
    xf = widen(x)
    z = xf[..., : d // 2] + 1j * xf[..., d // 2:]
    inv = theta ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    rot = np.exp(1j * pos[:, None].astype(np.float64) * inv[None, :])[:, None, :]
    zr = z * rot
    # angles up to 32767 rad: the two routes round the angle differently by
    # up to ~1e-11 rad
    np.testing.assert_allclose(out[..., : d // 2], zr.real, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(out[..., d // 2:], zr.imag, rtol=1e-10, atol=1e-10)


def test_rope_dot_products_depend_on_relative_position(oracle):
    # <rope(q, m), rope(k, n)> depends on m - n only, and pair norms are kept.
    g = rng(44)
    d = 64
    q = normal_bf16(g, (1, 1, d))
    k = normal_bf16(g, (1, 1, d))
    dots = []
    for m, n in [(10, 3), (107, 100), (7, 0)]:
        dots.append(float(np.dot(oracle.rope(q, [m])[0, 0], oracle.rope(k, [n])[0, 0])))
    np.testing.assert_allclose(dots, [dots[0]] * 3, rtol=1e-12)
    r = oracle.rope(q, [77])[0, 0]
    qf = widen(q)[0, 0]
    np.testing.assert_allclose(r[: d // 2] ** 2 + r[d // 2:] ** 2,
                               qf[: d // 2] ** 2 + qf[d // 2:] ** 2, rtol=1e-12)


def test_swiglu_closed_forms(oracle):
    # Gate first, up second.  silu(0) = 0; silu(1) = 1 / (1 + 1/e)
    # = 0.7310585786300049; silu(x) - silu(-x) = x.
    gu = bf([[0.0, 1.0, -3.0, 3.0, 5.0, 2.0, 1.0, 1.0]])
    out = oracle.swiglu(gu)[0]
    assert out[0] == 0.0
    assert abs(out[1] - 2.0 * 0.7310585786300049) < 1e-15
    assert abs((out[3] - out[2]) - 3.0) < 1e-14


def test_swiglu_matches_torch_fp64(oracle):
    g = rng(45)
    T, F = 4, 96
    gu = normal_bf16(g, (T, 2 * F), std=3.0)
    out = oracle.swiglu(gu)
    gt = torch.from_numpy(widen(gu))
    want = torch.nn.functional.silu(gt[:, :F]) * gt[:, F:]
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-13, atol=1e-15)


def test_add_rmsnorm_constant_sum_closed_form(oracle):
    # x + delta = c * 1  =>  y = c / sqrt(c^2 + eps) * w; s is the exact sum.
    H, eps = 32, 1e-6
    g = rng(46)
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    x = np.tile(bf([0.75] * H), (2, 1))
    delta = np.tile(bf([-2.0] * H), (2, 1))
    s, y = oracle.add_rmsnorm(x, delta, w, eps)
    c = -1.25
    np.testing.assert_array_equal(s, np.full((2, H), c))
    np.testing.assert_allclose(y[1], c / math.sqrt(c * c + eps) * widen(w), rtol=1e-14)


def test_add_rmsnorm_matches_torch_fp64(oracle):
    g = rng(47)
    M, H, eps = 5, 256, 1e-6
    x, delta = normal_bf16(g, (M, H)), normal_bf16(g, (M, H), std=0.3)
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    s, y = oracle.add_rmsnorm(x, delta, w, eps)
    st = torch.from_numpy(widen(x) + widen(delta))
    want = torch.nn.functional.rms_norm(st, (H,), torch.from_numpy(widen(w)), eps)
    np.testing.assert_allclose(s, st.numpy(), rtol=0, atol=0)
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-13)


def test_argmax_ties_take_the_lowest_index(oracle):
    logits = np.array([[1.0, 3.0, 3.0, 2.0],
                       [-np.inf, -5.0, -np.inf, -5.0],
                       [0.0, 0.0, 0.0, 0.0],
                       [1.0, 2.0, 3.0, 4.0]], dtype=np.float32)
    assert oracle.argmax(logits).tolist() == [1, 1, 0, 3]


def test_argmax_matches_numpy_first_occurrence(oracle):
    g = rng(48)
    logits = g.integers(-3, 4, size=(50, 1000)).astype(np.float32)  # many ties
    assert np.array_equal(oracle.argmax(logits), np.argmax(logits, axis=1))


# ---------------------------------------------------------------- sampling


def test_philox_known_answer_vectors(oracle):
    # Known-answer vectors published with the generator (Salmon et al., SC 2011;
    # the Random123 distribution's test vectors for philox4x32 with 10 rounds).
    kat = [((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
           ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
           ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
            (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1))]
    for ctr, key, want in kat:
        assert tuple(int(x) for x in oracle.philox4x32_10(ctr, key)) == want


def _u(oracle, seed, offset):
    w = oracle.philox4x32_10((offset & 0xFFFFFFFF, offset >> 32, 0, 0),
                             (seed & 0xFFFFFFFF, seed >> 32))
    return (int(w[0]) >> 8) / 16777216.0


def test_sample_temperature_zero_is_greedy(oracle):
    g = rng(140)
    logits = g.integers(-3, 4, size=(30, 500)).astype(np.float32)
    got = oracle.sample(logits, 0.0, 0.9, np.arange(30, dtype=np.uint64), 7)
    assert np.array_equal(got, oracle.argmax(logits))


def test_sample_uniform_logits_closed_form(oracle):
    # four equal weights, everything kept: token = floor(4 u)
    logits = np.zeros((1, 4), dtype=np.float32)
    for seed in range(200):
        tok = oracle.sample(logits, 1.0, 1.0, seed, 3 * seed + 1)[0]
        assert tok == int(4 * _u(oracle, seed, 3 * seed + 1)), seed


def test_sample_dominant_logit_and_tiny_top_p(oracle):
    g = rng(141)
    logits = g.standard_normal((50, 300)).astype(np.float32)
    logits[np.arange(50), g.integers(0, 300, size=50)] += 60.0
    seeds = np.arange(50, dtype=np.uint64) * 7919
    assert np.array_equal(oracle.sample(logits, 1.0, 1.0, seeds, 5), oracle.argmax(logits))
    mild = g.standard_normal((50, 300)).astype(np.float32)
    assert np.array_equal(oracle.sample(mild, 0.8, 1e-6, seeds, 5), oracle.argmax(mild))


def test_sample_nucleus_drops_the_tail(oracle):
    # weights 0.5, 0.3, 0.2 at top_p 0.6: keep {0, 1}; token 2 never drawn,
    # tokens 0 and 1 in proportion 5 : 3.
    logits = np.log(np.array([[0.5, 0.3, 0.2]], dtype=np.float64)).astype(np.float32)
    n = 4000
    toks = np.array([oracle.sample(logits, 1.0, 0.6, s, 11)[0] for s in range(n)])
    assert not (toks == 2).any()
    f0 = (toks == 0).mean()
    assert abs(f0 - 0.625) < 4 * np.sqrt(0.625 * 0.375 / n)


def test_sample_ties_at_the_threshold_are_all_kept(oracle):
    # weights 1, 1, 1, 0.5 at top_p 0.5: the threshold is 1 and all three
    # tied weights stay; 0.5 never drawn; the three equally often.
    logits = np.log(np.array([[1.0, 1.0, 1.0, 0.5]])).astype(np.float32)
    n = 3000
    toks = np.array([oracle.sample(logits, 1.0, 0.5, s, 0)[0] for s in range(n)])
    assert not (toks == 3).any()
    for k in range(3):
        assert abs((toks == k).mean() - 1 / 3) < 4 * np.sqrt(2 / 9 / n)


def test_sample_frequencies_follow_the_softmax(oracle):
    logits = np.array([[1.0, 0.0, -1.0, 2.0, 0.5]], dtype=np.float32)
    T = 0.7
    p = np.exp(logits[0].astype(np.float64) / T)
    p /= p.sum()
    n = 20000
    rows = np.repeat(logits, n, axis=0)
    toks = oracle.sample(rows, T, 1.0, np.arange(n, dtype=np.uint64), 99)
    for k in range(5):
        f = (toks == k).mean()
        assert abs(f - p[k]) < 4.5 * np.sqrt(p[k] * (1 - p[k]) / n), (k, f, p[k])


# ---------------------------------------------------------------- mixture of experts


def test_moe_route_hand_example(oracle):
    logits = np.array([[0.5, 2.0, -1.0, 2.0, 1.0]], dtype=np.float32)
    ex, w = oracle.moe_route(logits, 3)
    assert ex.tolist() == [[1, 3, 4]]          # tie 2.0: index 1 before 3
    e = np.exp([0.0, 0.0, -1.0])
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=1e-15)


def test_moe_route_matches_a_stable_sort(oracle):
    g = rng(160)
    logits = g.integers(-4, 5, size=(200, 16)).astype(np.float32)  # many ties
    ex, w = oracle.moe_route(logits, 4)
    want = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, :4]
    assert np.array_equal(ex, want)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
    sel = np.take_along_axis(logits, want, axis=1).astype(np.float64)
    t = torch.softmax(torch.from_numpy(sel), dim=1).numpy()
    np.testing.assert_allclose(w, t, rtol=1e-13)
    _, w1 = oracle.moe_route(logits, 1)
    assert np.all(w1 == 1.0)


def test_moe_dispatch_groups_by_expert_stably(oracle):
    g = rng(161)
    ex = g.integers(0, 8, size=(50, 3)).astype(np.int32)
    off, order, pos = oracle.moe_dispatch(ex, 8)
    flat = ex.ravel()
    want = np.argsort(flat, kind="stable")
    assert np.array_equal(order, want)
    assert np.array_equal(pos[order], np.arange(flat.size))
    assert np.array_equal(np.diff(off), np.bincount(flat, minlength=8))


def test_moe_combine_closed_forms(oracle):
    g = rng(162)
    y = normal_bf16(g, (6, 32))
    pos = np.array([3, 0, 5, 1, 2, 4])           # T = 3 tokens, k = 2
    w = np.array([[1.0, 0.0], [0.25, 0.75], [0.5, 0.5]])
    out = oracle.moe_combine(y, pos, w)
    yf = widen(y)
    np.testing.assert_array_equal(out[0], yf[3])
    np.testing.assert_allclose(out[1], 0.25 * yf[5] + 0.75 * yf[1], rtol=1e-15)
    np.testing.assert_allclose(out[2], 0.5 * (yf[2] + yf[4]), rtol=1e-15)


# ---------------------------------------------------------------- fused matmuls


def test_fold_norm_weight_closed_forms(oracle):
    g = rng(80)
    W = normal_bf16(g, (6, 20), std=0.02)
    # w = 1 leaves W; powers of two scale exactly; a one-hot w keeps one column
    np.testing.assert_array_equal(oracle.fold_norm_weight(W, bf(np.ones(20))), widen(W))
    p2 = 2.0 ** np.arange(-4, 16)
    np.testing.assert_array_equal(oracle.fold_norm_weight(W, bf(p2)), widen(W) * p2[None, :])
    one = np.zeros(20)
    one[13] = 1.0
    got = oracle.fold_norm_weight(W, bf(one))
    assert np.count_nonzero(got[:, np.arange(20) != 13]) == 0
    np.testing.assert_array_equal(got[:, 13], widen(W)[:, 13])


def test_fold_norm_weight_small_integers(oracle):
    # N=3, K=4: distinct sizes, so indexing w by the row fails
    W = np.array([[1, -2, 3, 4], [0, 5, -6, 7], [8, 1, 2, -3]])
    w = np.array([2, -1, 3, 5])
    got = oracle.fold_norm_weight(bf(W), bf(w))
    for n in range(3):
        for k in range(4):
            assert got[n, k] == W[n, k] * w[k]


def test_rmsnorm_matmul_hand_example(oracle):
    # x = [3, 4]: mean square 12.5; with eps = 0 each output is (w . x) / sqrt(12.5)
    c = oracle.rmsnorm_matmul(bf([[3, 4]]), bf([[1, 1], [1, -1], [2, 0]]), 0.0)
    np.testing.assert_allclose(c[0], np.array([7.0, -1.0, 6.0]) / math.sqrt(12.5), rtol=1e-15)


def test_rmsnorm_matmul_one_hot_rows_closed_form(oracle):
    # row m = v e_j: mean square v^2 / K, so C[m, n] = v / sqrt(v^2/K + eps) * wf[n, j].
    # v = 2^-10 makes eps (1e-6) dominate v^2 / K, so a dropped or misplaced eps shows.
    g = rng(81)
    K, N = 64, 9
    wf = normal_bf16(g, (N, K), std=0.5)
    cols = [0, 17, 63]
    vals = [2.0 ** -10, -3.0, 40.0]
    x = np.zeros((3, K))
    for m, (j, v) in enumerate(zip(cols, vals)):
        x[m, j] = v
    c = oracle.rmsnorm_matmul(bf(x), wf, 1e-6)
    for m, (j, v) in enumerate(zip(cols, vals)):
        np.testing.assert_allclose(c[m], v / math.sqrt(v * v / K + 1e-6) * widen(wf)[:, j],
                                   rtol=1e-13)


def test_rmsnorm_matmul_scale_invariance_without_eps(oracle):
    g = rng(82)
    x = normal_bf16(g, (4, 48))
    wf = normal_bf16(g, (5, 48), std=0.1)
    x2 = bf(widen(x) * 8.0)
    np.testing.assert_allclose(oracle.rmsnorm_matmul(x, wf, 0.0),
                               oracle.rmsnorm_matmul(x2, wf, 0.0), rtol=1e-13)


def test_rmsnorm_matmul_matches_torch_fp64(oracle):
    g = rng(83)
    x = normal_bf16(g, (6, 72))
    wf = normal_bf16(g, (11, 72), std=0.05)
    xt = torch.from_numpy(widen(x))
    y = torch.nn.functional.rms_norm(xt, (72,), eps=1e-6)
    want = y @ torch.from_numpy(widen(wf)).T
    np.testing.assert_allclose(oracle.rmsnorm_matmul(x, wf, 1e-6), want.numpy(), rtol=1e-11,
                               atol=1e-14)


def test_matmul_residual_small_integers_brute_force(oracle):
    # M=2, N=3, K=4, all distinct, so a transposed operand or residual fails
    g = rng(84)
    R = g.integers(-20, 21, size=(2, 3))
    A = g.integers(-5, 6, size=(2, 4))
    W = g.integers(-5, 6, size=(3, 4))
    c = oracle.matmul_residual(bf(R), bf(A), bf(W))
    for m in range(2):
        for n in range(3):
            assert c[m, n] == R[m, n] + sum(int(A[m, k]) * int(W[n, k]) for k in range(4))


def test_matmul_residual_degenerate_cases(oracle):
    g = rng(85)
    R = normal_bf16(g, (5, 24))
    A = normal_bf16(g, (5, 16))
    W = normal_bf16(g, (24, 16), std=0.1)
    np.testing.assert_array_equal(oracle.matmul_residual(R, A, bf(np.zeros((24, 16)))), widen(R))
    np.testing.assert_allclose(oracle.matmul_residual(bf(np.zeros((5, 24))), A, W),
                               oracle.matmul(A, W), rtol=1e-15)


def test_rope_angles_closed_forms(oracle):
    t = oracle.rope_angles(40, 8, 10000.0)
    np.testing.assert_array_equal(t[0, :, 0], 1.0)   # position 0: no rotation
    np.testing.assert_array_equal(t[0, :, 1], 0.0)
    p = np.arange(40)
    np.testing.assert_allclose(t[:, 0, 0], np.cos(p), rtol=0, atol=1e-15)  # i = 0: frequency 1
    np.testing.assert_allclose(t[:, 0, 1], np.sin(p), rtol=0, atol=1e-15)
    # d = 4, theta = 100: i = 1 has frequency 100^(-1/2) = 0.1; position 10 turns by 1 radian
    h = oracle.rope_angles(11, 4, 100.0)
    np.testing.assert_allclose(h[10, 1], [math.cos(1.0), math.sin(1.0)], rtol=1e-14)
    np.testing.assert_allclose(t[..., 0] ** 2 + t[..., 1] ** 2, 1.0, rtol=1e-15)


def test_rope_angles_rotate_like_rope(oracle):
    g = rng(90)
    x = normal_bf16(g, (6, 3, 16))
    pos = g.integers(0, 50, size=6).astype(np.int32)
    t = oracle.rope_angles(50, 16, 10000.0)
    xw = widen(x)
    c, s = t[pos, :, 0][:, None, :], t[pos, :, 1][:, None, :]
    want = np.concatenate([xw[..., :8] * c - xw[..., 8:] * s, xw[..., 8:] * c + xw[..., :8] * s], -1)
    np.testing.assert_allclose(oracle.rope(x, pos), want, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- backward


def _loss_grad_fd(oracle, x, w, dy, eps, h=1e-6):
    """Central differences of L = sum(dy * RMSNorm(x) * w) in x and w, taken
    on the oracle's forward in float64 (inputs perturbed off the bf16 grid
    through the exact forward formula restated with numpy)."""
    xw, ww, dyw = widen(x), widen(w), widen(dy)

    def loss(xv, wv):
        r = 1.0 / np.sqrt((xv * xv).mean(axis=1, keepdims=True) + eps)
        return float((dyw * xv * r * wv).sum())

    gx = np.zeros_like(xw)
    for idx in np.ndindex(*xw.shape):
        a, b = xw.copy(), xw.copy()
        a[idx] += h
        b[idx] -= h
        gx[idx] = (loss(a, ww) - loss(b, ww)) / (2 * h)
    gw = np.zeros_like(ww)
    for j in range(ww.shape[0]):
        a, b = ww.copy(), ww.copy()
        a[j] += h
        b[j] -= h
        gw[j] = (loss(xw, a) - loss(xw, b)) / (2 * h)
    return gx, gw


def test_rmsnorm_backward_matches_finite_differences(oracle):
    g = rng(95)
    x = normal_bf16(g, (3, 10))
    w = uniform_bf16(g, (10,), 0.5, 1.5)
    dy = normal_bf16(g, (3, 10))
    dx, dw = oracle.rmsnorm_backward(x, w, dy, 1e-6)
    gx, gw = _loss_grad_fd(oracle, x, w, dy, 1e-6)
    np.testing.assert_allclose(dx, gx, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(dw, gw, rtol=1e-6, atol=1e-7)
    # the forward the differences were taken on is the oracle's own
    xw, ww = widen(x), widen(w)
    r = 1.0 / np.sqrt((xw * xw).mean(axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 1e-6), xw * r * ww, rtol=1e-14)


def test_rmsnorm_backward_closed_forms(oracle):
    # dy parallel to y's direction: a row-scale-invariant map has dx orthogonal
    # to x when eps = 0 (sum_j x_j dx_j = 0); dw with dy = 1 is sum over rows of x r
    g = rng(96)
    x = normal_bf16(g, (4, 16))
    w = bf(np.ones(16))
    dy = normal_bf16(g, (4, 16))
    dx, _ = oracle.rmsnorm_backward(x, w, dy, 0.0)
    np.testing.assert_allclose((dx * widen(x)).sum(axis=1), 0.0, atol=1e-12)
    ones = bf(np.ones((4, 16)))
    _, dw = oracle.rmsnorm_backward(x, w, ones, 1e-6)
    xw = widen(x)
    r = 1.0 / np.sqrt((xw * xw).mean(axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(dw, (xw * r).sum(axis=0), rtol=1e-13)


def _attn_case(seed, L=7, Hq=4, Hkv=2, d=4):
    g = rng(seed)
    K, V = normal_bf16(g, (L, Hkv, d)), normal_bf16(g, (L, Hkv, d))
    kc, vc, bt = _contig_cache(K, V)
    rows = [(h, t) for h in range(Hq) for t in (2, L - 1)]
    q = normal_bf16(g, (len(rows), d))
    do = normal_bf16(g, (len(rows), d))
    heads = np.array([h for h, _ in rows])
    pos = np.array([t for _, t in rows])
    return q, do, heads, pos, kc, vc, bt


def _attn_forward_np(q, kc, vc, heads, pos, Hq, scale):
    """softmax(scale q.k) v over keys 0..t of the contiguous cache, float64."""
    Hkv, d = kc.shape[1], kc.shape[3]
    Kl = kc.transpose(0, 2, 1, 3).reshape(-1, Hkv, d)
    Vl = vc.transpose(0, 2, 1, 3).reshape(-1, Hkv, d)
    out = np.zeros_like(q)
    for r in range(q.shape[0]):
        g, t = heads[r] // (Hq // Hkv), pos[r]
        s = scale * (Kl[: t + 1, g] @ q[r])
        p = np.exp(s - s.max())
        out[r] = (p / p.sum()) @ Vl[: t + 1, g]
    return out


def test_attention_backward_matches_finite_differences(oracle):
    Hq, d = 4, 4
    q, do, heads, pos, kc, vc, bt = _attn_case(97, Hq=Hq, d=d)
    R, scale = q.shape[0], 0.7
    dq, dk, dv = oracle.attention_backward(q, do, np.zeros(R), heads, pos, Hq, kc, vc, bt, scale)
    qw, dow, kw, vw = widen(q), widen(do), widen(kc), widen(vc)
    # the numpy forward is the oracle's forward
    np.testing.assert_allclose(_attn_forward_np(qw, kw, vw, heads, pos, Hq, scale),
                               oracle.attention(q, np.zeros(R), heads, pos, Hq, kc, vc, bt,
                                                scale=scale), rtol=1e-13, atol=1e-15)

    def loss(qv, kv, vv):
        return float((dow * _attn_forward_np(qv, kv, vv, heads, pos, Hq, scale)).sum())

    h = 1e-6
    for arr, grad, which in ((qw, dq, 0), (kw, dk, 1), (vw, dv, 2)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(*arr.shape):
            a, b = arr.copy(), arr.copy()
            a[idx] += h
            b[idx] -= h
            args_a = [qw, kw, vw]
            args_b = [qw, kw, vw]
            args_a[which], args_b[which] = a, b
            fd[idx] = (loss(*args_a) - loss(*args_b)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


def test_attention_backward_closed_forms(oracle):
    # identical keys: uniform weights, so sum_j ds_j = 0 and dq = 0; and each
    # visible value row gets dO / (t + 1) from every row that sees it
    g = rng(98)
    L, d = 6, 4
    K = np.tile(normal_bf16(g, (d,)), (L, 1, 1))
    V = normal_bf16(g, (L, 1, d))
    kc, vc, bt = _contig_cache(K, V)
    q, do = normal_bf16(g, (2, d)), normal_bf16(g, (2, d))
    pos = np.array([1, 5])
    dq, dk, dv = oracle.attention_backward(q, do, np.zeros(2), np.zeros(2), pos, 1, kc, vc, bt)
    assert np.abs(dq).max() < 1e-12
    dow = widen(do)
    for j in range(L):
        want = dow[1] / 6 + (dow[0] / 2 if j <= 1 else 0.0)
        np.testing.assert_allclose(dv[0, 0, j], want, rtol=1e-13, atol=1e-15)
    # a single visible key: weight 1, no gradient to q or k, dv = dO
    dq1, dk1, dv1 = oracle.attention_backward(q[:1], do[:1], [0], [0], [0], 1, kc, vc, bt)
    assert np.all(dq1 == 0) and np.all(dk1 == 0)
    np.testing.assert_array_equal(dv1[0, 0, 0], dow[0])
    assert np.all(dv1[0, 0, 1:] == 0)


def test_swiglu_backward_matches_finite_differences(oracle):
    g = rng(99)
    gu = normal_bf16(g, (3, 10), std=2.0)
    dout = normal_bf16(g, (3, 5))
    grad = oracle.swiglu_backward(gu, dout)
    guw, dw = widen(gu), widen(dout)
    np.testing.assert_allclose(oracle.swiglu(gu), guw[:, :5] / (1 + np.exp(-guw[:, :5])) * guw[:, 5:],
                               rtol=1e-14)

    def loss(v):
        return float((dw * v[:, :5] / (1 + np.exp(-v[:, :5])) * v[:, 5:]).sum())

    h = 1e-6
    fd = np.zeros_like(guw)
    for idx in np.ndindex(*guw.shape):
        a, b = guw.copy(), guw.copy()
        a[idx] += h
        b[idx] -= h
        fd[idx] = (loss(a) - loss(b)) / (2 * h)
    np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-9)
    # closed forms at gate 0: dgate = dout * up / 2, dup = 0
    z = bf([[0.0, 0.0, 3.0, -1.0]])
    np.testing.assert_array_equal(oracle.swiglu_backward(z, bf([[2.0, 1.0]])), [[3.0, -0.5, 0.0, 0.0]])


def test_rope_backward_is_the_inverse_rotation(oracle):
    g = rng(100)
    dy = normal_bf16(g, (5, 2, 8))
    pos = g.integers(0, 500, size=5).astype(np.int32)
    dx = oracle.rope_backward(dy, pos)
    # the forward is linear with an orthogonal matrix per (t, pair): its
    # gradient is the transpose, so rotating dx forward gives dy back
    t = oracle.rope_angles(500, 8)
    c, s = t[pos, :, 0][:, None, :], t[pos, :, 1][:, None, :]
    fwd = np.concatenate([dx[..., :4] * c - dx[..., 4:] * s, dx[..., 4:] * c + dx[..., :4] * s], -1)
    np.testing.assert_allclose(fwd, widen(dy), rtol=1e-12, atol=1e-14)
    # position 0: identity
    np.testing.assert_array_equal(oracle.rope_backward(dy, np.zeros(5, np.int32)), widen(dy))
    # the adjoint identity <rope(x), dy> = <x, rope_backward(dy)> on bf16 inputs
    x = normal_bf16(g, (5, 2, 8))
    lhs = float((oracle.rope(x, pos) * widen(dy)).sum())
    rhs = float((widen(x) * dx).sum())
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))
