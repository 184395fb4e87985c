"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module draws the random tensors of the workloads and nothing else: it
holds none of the arithmetic of RMSNorm, matmul or attention.  Both sides of
every parity test receive the same bytes from here.

Floating-point tensors are drawn in float32 with numpy's PCG64 generator and
rounded to bfloat16 (round to nearest, ties to even); they are returned as
``uint16`` arrays of bfloat16 bit patterns, which is what the C-ABI and the
oracle both take.  Integer tensors (page tables, lengths, slot maps) are
drawn with the same generator.

Workloads (distributions and shapes of the serving workloads described in the
reports on "Defeating Nondeterminism in LLM Inference"):

* ``tiny_layer``      x[B,256]~N(0,1), w~U(0.5,1.5), W[512,256]~N(0,0.02),
                      1-head decode attention d=64, KV length U(1,300), page 16.
* ``norm_matmul``     x[2048,4096]~N(0,1), w~U(0.5,1.5), W[N,4096]~N(0,0.02).
* ``paged_decode``    GQA 64/4, d=128, q,K,V~N(0,1), lengths U(1,32768),
                      shuffled physical page ids.
* ``prefill``         32/8 heads, d=128, one 8192-token sequence, N(0,1).

Weights are stored output-feature-major, ``W[N, K]`` (the ``nn.Linear``
layout), so that the product is ``x @ W.T``.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

PAGE = 16


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); NaN stays NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x = x * np.float32(std)
    return f32_to_bf16_bits(x)


def uniform_bf16(g: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    x = g.uniform(lo, hi, size=shape).astype(np.float32)
    return f32_to_bf16_bits(x)


# ---------------------------------------------------------------------------
# paged KV cache
# ---------------------------------------------------------------------------

@dataclass
class PagedKV:
    """A paged KV cache: ``k_cache``/``v_cache`` are ``[num_pages, Hkv, 16, d]``
    bfloat16 bit arrays; ``block_table[b, i]`` is the physical page holding
    tokens ``16*i .. 16*i+15`` of sequence ``b`` (entries past a sequence's
    last page are -1)."""

    k_cache: np.ndarray
    v_cache: np.ndarray
    block_table: np.ndarray
    seq_lens: np.ndarray
    num_kv_heads: int
    head_dim: int

    @property
    def num_pages(self) -> int:
        return self.k_cache.shape[0]

    @property
    def max_pages(self) -> int:
        return self.block_table.shape[1]


def page_table(g: np.random.Generator, seq_lens, extra_pages: int = 0,
               max_pages: int | None = None):
    """Assign shuffled physical pages to sequences of the given lengths.

    Returns ``(block_table, num_pages)``.  The pool holds every page the
    sequences need plus ``extra_pages`` unused ones; physical ids are a random
    permutation of the pool, so neighbouring logical pages are scattered.
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    need = (seq_lens + PAGE - 1) // PAGE
    total = int(need.sum())
    num_pages = total + int(extra_pages)
    perm = g.permutation(num_pages).astype(np.int32)
    mp = int(need.max()) if len(need) else 0
    if max_pages is not None:
        mp = max(mp, int(max_pages))
    bt = np.full((len(seq_lens), max(mp, 1)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[off:off + n]
        off += int(n)
    return bt, num_pages


def paged_kv(g: np.random.Generator, seq_lens, num_kv_heads: int, head_dim: int,
             extra_pages: int = 0, fill_unused: str = "normal") -> PagedKV:
    """A filled paged cache.  ``fill_unused`` decides what the slots past each
    sequence's length hold: ``"normal"`` (random values), ``"nan"`` (bfloat16
    NaN, a stale pool) or ``"zero"``."""
    bt, num_pages = page_table(g, seq_lens, extra_pages)
    shape = (num_pages, num_kv_heads, PAGE, head_dim)
    k = normal_bf16(g, shape)
    v = normal_bf16(g, shape)
    if fill_unused != "normal":
        val = np.uint16(0x7FC0 if fill_unused == "nan" else 0)
        used = np.zeros((num_pages, PAGE), dtype=bool)
        for b, L in enumerate(np.asarray(seq_lens)):
            for j in range(int(L)):
                used[bt[b, j // PAGE], j % PAGE] = True
        mask = ~used
        k[mask[:, None, :, None].repeat(num_kv_heads, 1).repeat(head_dim, 3)] = val
        v[mask[:, None, :, None].repeat(num_kv_heads, 1).repeat(head_dim, 3)] = val
    return PagedKV(k, v, bt, np.asarray(seq_lens, dtype=np.int32), num_kv_heads, head_dim)


def kv_to_blocks(cache: np.ndarray) -> np.ndarray:
    """Logical cache [num_pages, Hkv, 16, d] -> the device layout: each
    (page, head) block of 16 x d values in core-matrix order
    [key group 2][value group d/8][8 keys][8 values].  A pure permutation."""
    P, H, T, d = cache.shape
    assert T == PAGE
    x = cache.reshape(P, H, 2, 8, d // 8, 8)          # page, head, kg, r, vg, c
    return np.ascontiguousarray(x.transpose(0, 1, 2, 4, 3, 5)).reshape(P, H, T, d)


def kv_from_blocks(blocks: np.ndarray) -> np.ndarray:
    """Inverse of kv_to_blocks."""
    P, H, T, d = blocks.shape
    x = blocks.reshape(P, H, 2, d // 8, 8, 8)         # page, head, kg, vg, r, c
    return np.ascontiguousarray(x.transpose(0, 1, 2, 4, 3, 5)).reshape(P, H, T, d)


def slot_mapping(block_table: np.ndarray, seq: int, positions) -> np.ndarray:
    """Physical slot (page * 16 + offset) of each absolute token position."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = block_table[seq, positions // PAGE].astype(np.int64)
    return pages * PAGE + positions % PAGE


# ---------------------------------------------------------------------------
# named workloads
# ---------------------------------------------------------------------------

def tiny_layer(seed: int = 0, batch_sizes=(1, 3, 8)):
    """The tiny layer: hidden 256, matmul to 512, one-head decode attention
    with head dim 64 over KV lengths U(1,300)."""
    g = rng(seed)
    B = max(batch_sizes)
    x = normal_bf16(g, (B, 256))
    w = uniform_bf16(g, (256,), 0.5, 1.5)
    W = normal_bf16(g, (512, 256), std=0.02)
    lens = g.integers(1, 301, size=B).astype(np.int32)
    kv = paged_kv(g, lens, num_kv_heads=1, head_dim=64)
    q = normal_bf16(g, (B, 1, 64))
    return dict(x=x, w=w, W=W, eps=1e-6, kv=kv, q=q, batch_sizes=tuple(batch_sizes))


def norm_matmul(seed: int = 1, M: int = 2048, H: int = 4096, N: int = 4096):
    """RMSNorm + matmul at hidden 4096: x[M,H]~N(0,1), w~U(0.5,1.5),
    W[N,H]~N(0,0.02)."""
    g = rng(seed)
    x = normal_bf16(g, (M, H))
    w = uniform_bf16(g, (H,), 0.5, 1.5)
    W = normal_bf16(g, (N, H), std=0.02)
    return dict(x=x, w=w, W=W, eps=1e-6)


def decode_lengths(seed: int, B: int, max_len: int = 32768) -> np.ndarray:
    return rng(seed).integers(1, max_len + 1, size=B).astype(np.int32)


def paged_decode(seed: int = 2, B: int = 8, Hq: int = 64, Hkv: int = 4, d: int = 128,
                 max_len: int = 32768, seq_lens=None, extra_pages: int = 0,
                 fill_unused: str = "normal"):
    """Paged decode: one new query token per request, GQA Hq/Hkv."""
    g = rng(seed)
    if seq_lens is None:
        seq_lens = g.integers(1, max_len + 1, size=B).astype(np.int32)
    kv = paged_kv(g, seq_lens, Hkv, d, extra_pages=extra_pages, fill_unused=fill_unused)
    q = normal_bf16(g, (len(seq_lens), Hq, d))
    return dict(kv=kv, q=q, Hq=Hq)


def prefill(seed: int = 3, S: int = 8192, Hq: int = 32, Hkv: int = 8, d: int = 128):
    """One causal sequence of S tokens: q[S,Hq,d], new K/V [S,Hkv,d], and an
    empty paged cache (shuffled pages) big enough to hold them."""
    g = rng(seed)
    q = normal_bf16(g, (S, Hq, d))
    k = normal_bf16(g, (S, Hkv, d))
    v = normal_bf16(g, (S, Hkv, d))
    bt, num_pages = page_table(g, [S])
    return dict(q=q, k=k, v=v, block_table=bt, num_pages=num_pages, Hq=Hq, Hkv=Hkv, d=d)


# ---------------------------------------------------------------------------
# device-side bulk generation (for workloads too large to draw on the host)
# ---------------------------------------------------------------------------

def torch_normal_bf16(shape, seed: int, device, std: float = 1.0):
    """N(0, std) bfloat16 drawn by torch's counter-based generator on
    ``device`` from ``seed``.  Used only where a host draw would take too long
    (the multi-GB decode cache); the bytes are copied back for the oracle."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    t.normal_(0.0, std, generator=gen)
    return t


# ---------------------------------------------------------------------------
# the toy decoder's weights and the unique-completion workload
# ---------------------------------------------------------------------------

def toy_decoder_weights(shapes: dict, seed: int, device, std: float = 0.02) -> dict:
    """Random-init weights for the toy decoder: every matrix N(0, std) drawn
    on ``device`` by torch's generator (one seed per tensor, in the order of
    ``shapes``), every norm weight 1."""
    import torch

    out = {}
    for k, (name, shape) in enumerate(shapes.items()):
        if len(shape) == 1:
            out[name] = torch.ones(shape, dtype=torch.bfloat16, device=device)
        else:
            out[name] = torch_normal_bf16(shape, seed * 1000 + k, device, std=std)
    return out


def unique_completion_workload(seed: int = 4, n_target: int = 1000, n_other: int = 1000,
                               prompt_len: int = 64, gen_len: int = 256, vocab: int = 32000,
                               other_prompt_max: int = 512, steps_span: int = 2000):
    """One fixed prompt (``prompt_len`` ids drawn from ``seed``) to be
    completed ``n_target`` times, amid ``n_other`` requests with random
    prompts of U(1, other_prompt_max) tokens and U(1, gen_len) new tokens.
    Arrival steps are drawn in bursts (each request's step is uniform inside
    one of several windows of random width over ``steps_span`` steps), so
    the number of running requests sweeps from 1 up to the scheduler's cap.

    Returns ``(prompt, requests)`` with requests a list of dicts
    ``{rid, prompt, max_new, arrival, tag, seed}`` in random order; every
    target copy carries the same sampling seed (the same request sent again),
    the others seeds of their own."""
    g = rng(seed)
    prompt = g.integers(0, vocab, size=prompt_len).astype(np.int32)
    n = n_target + n_other
    tags = np.array(["target"] * n_target + ["other"] * n_other)
    g.shuffle(tags)
    # bursts: 16 windows with random centres and widths
    centres = np.sort(g.uniform(0, steps_span, size=16))
    widths = g.uniform(1, steps_span / 8, size=16)
    which = g.integers(0, 16, size=n)
    arrival = np.clip(centres[which] + g.uniform(-0.5, 0.5, size=n) * widths[which], 0, None)
    target_seed = int(g.integers(0, 2 ** 62))
    reqs = []
    for i in range(n):
        if tags[i] == "target":
            p, m, sd = prompt, gen_len, target_seed
        else:
            p = g.integers(0, vocab, size=int(g.integers(1, other_prompt_max + 1))).astype(np.int32)
            m = int(g.integers(1, gen_len + 1))
            sd = int(g.integers(0, 2 ** 62))
        reqs.append(dict(rid=i, prompt=p, max_new=m, arrival=int(arrival[i]), tag=str(tags[i]),
                         seed=sd))
    return prompt, reqs
