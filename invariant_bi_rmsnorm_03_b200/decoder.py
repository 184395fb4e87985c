"""A pre-norm decoder built from the library's batch-invariant kernels, and
a small continuous-batching scheduler that feeds it.

The reports on "Defeating Nondeterminism in LLM Inference" show the effect
of batch invariance end to end: one prompt, completed greedily many times
while other requests come and go, gives one completion instead of many
(xitu-tech news, "显著成果与高昂成本"; liuwei.blog, "实验成果").  They name no
layer beyond RMSNorm, matmul and attention, so the model here is the plain
pre-norm transformer (token embedding; per layer RMSNorm -> stacked q/k/v
matmul -> rotary embedding + KV-cache write -> paged attention -> output
matmul -> residual + RMSNorm -> stacked gate/up matmul -> SwiGLU -> down
matmul -> residual, or a mixture of experts in place of the one feed-forward
(router matmul -> top-k route -> grouping by expert -> each expert's SwiGLU
feed-forward -> gate-weighted combine); final RMSNorm; lm_head matmul in
fp32; the next token by bi_sample: greedy at temperature 0, else nucleus
sampling from the request's own counter-based random stream).

Every arithmetic step runs in the library's CUDA kernels through the C ABI;
this module only plans the batch on the host (which request contributes
which tokens, where their keys and values go in the paged cache) and copies
that plan to the device.  Which requests share a step, how many tokens each
contributes and whether a token is decoded or prefilled (whole or in chunks)
changes nothing in any request's bits.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from .binding import PAGE_SIZE, Library, PagedKV


@dataclass(frozen=True)
class DecoderConfig:
    hidden: int = 4096
    layers: int = 8
    n_heads: int = 32
    n_kv_heads: int = 8
    head_dim: int = 128
    ffn: int = 14336
    vocab: int = 32000
    theta: float = 10000.0
    eps: float = 1e-6
    n_experts: int = 0            # > 0: a mixture-of-experts feed-forward
    top_k: int = 2
    expert_ffn: int = 1408
    fused: bool = False           # RMSNorm folded into the next matmul, RoPE and the
                                  # cache write in the QKV matmul's epilogue, residual
                                  # adds in the matmul epilogue (dense feed-forward only)
    max_pos: int = 8192           # fused form: positions covered by the rotary table

    @property
    def qkv_dim(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


def weight_shapes(cfg: DecoderConfig) -> dict:
    """Name -> shape of every weight (matmul weights are [out, in])."""
    s = {"embed": (cfg.vocab, cfg.hidden), "lm_head": (cfg.vocab, cfg.hidden),
         "final_norm": (cfg.hidden,)}
    for i in range(cfg.layers):
        s["l%d.attn_norm" % i] = (cfg.hidden,)
        s["l%d.wqkv" % i] = (cfg.qkv_dim, cfg.hidden)
        s["l%d.wo" % i] = (cfg.hidden, cfg.n_heads * cfg.head_dim)
        s["l%d.mlp_norm" % i] = (cfg.hidden,)
        if cfg.n_experts:  # the experts' weights stacked: [E, out, in]
            s["l%d.router" % i] = (cfg.n_experts, cfg.hidden)
            s["l%d.moe_wgu" % i] = (cfg.n_experts, 2 * cfg.expert_ffn, cfg.hidden)
            s["l%d.moe_wdown" % i] = (cfg.n_experts, cfg.hidden, cfg.expert_ffn)
        else:
            s["l%d.wgu" % i] = (2 * cfg.ffn, cfg.hidden)
            s["l%d.wdown" % i] = (cfg.hidden, cfg.ffn)
    return s


# ---------------------------------------------------------------- host plan


@dataclass
class Request:
    rid: int
    prompt: np.ndarray            # int32 token ids
    max_new: int                  # tokens to generate
    arrival: int = 0              # first step at which it may be admitted
    tag: str = ""
    temperature: float = 0.0      # 0: greedy
    top_p: float = 1.0
    seed: int = 0                 # the request's own random stream
    pages: list = field(default_factory=list)
    done_prompt: int = 0          # prompt tokens already in the cache
    out: list = field(default_factory=list)

    @property
    def cached(self) -> int:
        """Tokens whose keys and values are in the cache."""
        return self.done_prompt + max(0, len(self.out) - 1)

    @property
    def finished(self) -> bool:
        return len(self.out) >= self.max_new


@dataclass
class StepPlan:
    """One forward step: decode rows first, then the prefill chunks."""
    tokens: np.ndarray       # int32 [T]
    positions: np.ndarray    # int32 [T]
    slots: np.ndarray        # int64 [T]
    dec: list                # requests decoding one token
    dec_lens: np.ndarray     # int32 [B_dec], lengths including the new token
    pre: list                # (request, chunk length)
    cu_q: np.ndarray         # int32 [B_pre + 1]
    ctx: np.ndarray          # int32 [B_pre]
    sample_rows: np.ndarray  # int32 rows whose next token is taken
    sample_reqs: list        # the request of each sampled row
    temperature: np.ndarray  # float32 per sampled row
    top_p: np.ndarray        # float32 per sampled row
    seed: np.ndarray         # uint64 per sampled row
    offset: np.ndarray       # uint64 per sampled row: the position of the token drawn
    block_table: np.ndarray  # int32 [B_dec + B_pre, max_pages]


class PagePool:
    """Physical pages of the KV cache (the same page ids in every layer)."""

    def __init__(self, num_pages: int, seed: int = 0):
        # hand out pages in a shuffled order so neighbouring pages are scattered
        self.free = list(np.random.default_rng(seed).permutation(num_pages).astype(int))

    def take(self, n: int) -> list:
        if n > len(self.free):
            raise RuntimeError("KV cache pool exhausted")
        out, self.free = self.free[:n], self.free[n:]
        return out

    def give(self, pages: list) -> None:
        self.free.extend(pages)


class Scheduler:
    """Admits requests as they arrive (at most ``max_batch`` at once) and
    plans each step within a token budget: every running request in decode
    contributes its one token; prompts take what budget is left, in chunks if
    needed, oldest first."""

    def __init__(self, pool: PagePool, max_batch: int = 256, token_budget: int = 2048):
        self.pool, self.max_batch, self.budget = pool, max_batch, token_budget
        self.waiting: list = []
        self.running: list = []
        self.finished: list = []
        self.step_no = 0

    def add(self, reqs) -> None:
        self.waiting.extend(reqs)
        self.waiting.sort(key=lambda r: (r.arrival, r.rid))

    def idle(self) -> bool:
        return not self.waiting and not self.running

    def _ensure_pages(self, r: Request, upto: int) -> None:
        need = (upto + PAGE_SIZE - 1) // PAGE_SIZE - len(r.pages)
        if need > 0:
            r.pages.extend(self.pool.take(need))

    def plan(self) -> StepPlan | None:
        while (self.waiting and self.waiting[0].arrival <= self.step_no
               and len(self.running) < self.max_batch):
            self.running.append(self.waiting.pop(0))
        if not self.running:
            self.step_no += 1
            return None
        dec = [r for r in self.running if r.done_prompt == len(r.prompt)]
        budget = self.budget - len(dec)
        pre = []
        for r in self.running:
            if r.done_prompt < len(r.prompt) and budget > 0:
                n = min(len(r.prompt) - r.done_prompt, budget)
                pre.append((r, n))
                budget -= n
        tokens, pos, slots, rows = [], [], [], []
        dec_lens = []
        for r in dec:
            p = r.cached                       # the new token's position
            self._ensure_pages(r, p + 1)
            tokens.append(r.out[-1])
            pos.append(p)
            slots.append(r.pages[p // PAGE_SIZE] * PAGE_SIZE + p % PAGE_SIZE)
            dec_lens.append(p + 1)
            rows.append(r)
        cu, ctx = [0], []
        sample_rows, sample_reqs = list(range(len(dec))), list(dec)
        for r, n in pre:
            p0 = r.done_prompt
            self._ensure_pages(r, p0 + n)
            for j in range(n):
                p = p0 + j
                tokens.append(int(r.prompt[p]))
                pos.append(p)
                slots.append(r.pages[p // PAGE_SIZE] * PAGE_SIZE + p % PAGE_SIZE)
            ctx.append(p0)
            cu.append(cu[-1] + n)
            if p0 + n == len(r.prompt):       # prompt complete: sample its last row
                sample_rows.append(len(dec) + cu[-1] - 1)
                sample_reqs.append(r)
            rows.append(r)
        max_pages = max(len(r.pages) for r in rows)
        bt = np.full((len(rows), max_pages), -1, dtype=np.int32)
        for i, r in enumerate(rows):
            bt[i, :len(r.pages)] = r.pages
        # the token drawn for request r sits at position len(prompt) + len(out)
        return StepPlan(np.array(tokens, np.int32), np.array(pos, np.int32),
                        np.array(slots, np.int64), dec, np.array(dec_lens, np.int32), pre,
                        np.array(cu, np.int32), np.array(ctx, np.int32),
                        np.array(sample_rows, np.int32), sample_reqs,
                        np.array([r.temperature for r in sample_reqs], np.float32),
                        np.array([r.top_p for r in sample_reqs], np.float32),
                        np.array([r.seed for r in sample_reqs], np.uint64),
                        np.array([len(r.prompt) + len(r.out) for r in sample_reqs], np.uint64),
                        bt)

    def commit(self, plan: StepPlan, next_tokens: np.ndarray) -> None:
        """Record the step's sampled tokens and retire finished requests."""
        for r, n in plan.pre:
            r.done_prompt += n
        for r, t in zip(plan.sample_reqs, next_tokens):
            r.out.append(int(t))
        keep = []
        for r in self.running:
            if r.finished:
                self.pool.give(r.pages)
                r.pages = []
                self.finished.append(r)
            else:
                keep.append(r)
        self.running = keep
        self.step_no += 1


# ---------------------------------------------------------------- device model


class ToyDecoder:
    """The decoder's forward step on one GPU.  ``weights`` maps the names of
    :func:`weight_shapes` to bf16 device tensors (the caller owns them)."""

    def __init__(self, lib: Library, cfg: DecoderConfig, weights: dict, num_pages: int,
                 device):
        self.L, self.cfg, self.w, self.dev = lib, cfg, weights, torch.device(device)
        for name, shape in weight_shapes(cfg).items():
            t = weights[name]
            if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_cuda:
                raise ValueError("weight %s must be bf16 %s on the GPU" % (name, shape))
        shape = (num_pages, cfg.n_kv_heads, PAGE_SIZE, cfg.head_dim)
        self.k_cache = [torch.zeros(shape, dtype=torch.bfloat16, device=self.dev)
                        for _ in range(cfg.layers)]
        self.v_cache = [torch.zeros(shape, dtype=torch.bfloat16, device=self.dev)
                        for _ in range(cfg.layers)]
        self.num_pages = num_pages
        # fused form: each matmul that follows an RMSNorm takes its weight with
        # the norm weight folded in (once, here)
        self.wf = {}
        if cfg.fused:
            if cfg.n_experts:
                raise ValueError("the fused form covers the dense feed-forward only")
            for i in range(cfg.layers):
                self.wf["l%d.wqkv" % i] = lib.bi_fold_norm_weight(weights["l%d.wqkv" % i],
                                                                  weights["l%d.attn_norm" % i])
                self.wf["l%d.wgu" % i] = lib.bi_fold_norm_weight(weights["l%d.wgu" % i],
                                                                 weights["l%d.mlp_norm" % i])
            self.wf["lm_head"] = lib.bi_fold_norm_weight(weights["lm_head"],
                                                         weights["final_norm"])
            self.rope = lib.bi_rope_table(cfg.max_pos, cfg.head_dim, cfg.theta, device=self.dev)

    def _to_dev(self, a: np.ndarray) -> torch.Tensor:
        return torch.from_numpy(np.ascontiguousarray(a)).to(self.dev, non_blocking=False)

    def forward(self, plan: StepPlan) -> np.ndarray:
        """Runs one step and returns the greedy next token of each sampled row."""
        L, c, W = self.L, self.cfg, self.w
        T = len(plan.tokens)
        Bd = len(plan.dec)
        if c.fused and T and int(plan.positions.max()) >= c.max_pos:
            raise ValueError("position %d is past the rotary table (max_pos %d)"
                             % (int(plan.positions.max()), c.max_pos))
        tokens, pos, slots = self._to_dev(plan.tokens), self._to_dev(plan.positions), \
            self._to_dev(plan.slots)
        bt = self._to_dev(plan.block_table)
        dec_lens = self._to_dev(plan.dec_lens) if Bd else None
        cu, ctx = (self._to_dev(plan.cu_q), self._to_dev(plan.ctx)) if plan.pre else (None, None)
        rows = self._to_dev(plan.sample_rows)
        max_len = int(plan.dec_lens.max()) if Bd else 0
        max_chunk = int(np.diff(plan.cu_q).max()) if plan.pre else 0

        x = L.bi_embedding(W["embed"], tokens)
        o = torch.empty((T, c.n_heads, c.head_dim), dtype=torch.bfloat16, device=self.dev)
        # the fused norm forms' row statistics, one buffer for the whole step
        nws = L._norm_ws(T, self.dev) if c.fused else None
        h = None if c.fused else L.bi_rmsnorm(x, W["l0.attn_norm"], c.eps)
        for i in range(c.layers):
            kv_all = PagedKV(self.k_cache[i], self.v_cache[i], bt)
            if c.fused:
                # RMSNorm, the QKV matmul, RoPE and the cache write: the row
                # statistics, then one matmul launch
                q = L.bi_rmsnorm_matmul_rope_kv(x, self.wf["l%d.wqkv" % i], c.eps, kv_all,
                                                self.rope, pos, slots, c.n_heads, ws=nws)
            else:
                qkv = L.bi_matmul(h, W["l%d.wqkv" % i])
                q = L.bi_rope_kv_write(kv_all, qkv, pos, slots, c.n_heads, c.theta)
            if Bd:
                kv = PagedKV(self.k_cache[i], self.v_cache[i], bt[:Bd])
                L.bi_attention_decode(kv, q[:Bd], dec_lens, max_len, out=o[:Bd])
            if plan.pre:
                kv = PagedKV(self.k_cache[i], self.v_cache[i], bt[Bd:])
                L.bi_attention_prefill(kv, q[Bd:], cu, ctx, max_chunk, out=o[Bd:])
            if c.fused:
                # x += o Wo^T; x += swiglu(RMSNorm(x) Wgu^T) Wdown^T
                L.bi_matmul_residual(o.view(T, c.n_heads * c.head_dim), W["l%d.wo" % i], x,
                                     out=x)
                f = L.bi_swiglu(L.bi_rmsnorm_matmul(x, self.wf["l%d.wgu" % i], c.eps, ws=nws))
                L.bi_matmul_residual(f, W["l%d.wdown" % i], x, out=x)
                continue
            a = L.bi_matmul(o.view(T, c.n_heads * c.head_dim), W["l%d.wo" % i])
            h = L.bi_add_rmsnorm(x, a, W["l%d.mlp_norm" % i], c.eps)
            if c.n_experts:
                m = self._moe(h, i)
            else:
                f = L.bi_swiglu(L.bi_matmul(h, W["l%d.wgu" % i]))
                m = L.bi_matmul(f, W["l%d.wdown" % i])
            nxt = W["l%d.attn_norm" % (i + 1)] if i + 1 < c.layers else W["final_norm"]
            h = L.bi_add_rmsnorm(x, m, nxt, c.eps)
        if c.fused:
            last = L.bi_embedding(x, rows)
            logits = L.bi_rmsnorm_matmul(last, self.wf["lm_head"], c.eps, out_dtype=torch.float32,
                                         ws=nws)
        else:
            last = L.bi_embedding(h, rows)
            logits = L.bi_matmul(last, W["lm_head"], out_dtype=torch.float32)
        nt = L.bi_sample(logits, self._to_dev(plan.temperature), self._to_dev(plan.top_p),
                         self._to_dev(plan.seed.view(np.int64)),
                         self._to_dev(plan.offset.view(np.int64)))
        return nt.cpu().numpy()


    def _moe(self, h: torch.Tensor, i: int):
        """The mixture-of-experts feed-forward of layer i; returns its output.
        All experts' matmuls run in one grouped launch each, their
        tiles laid out on the device from the dispatch offsets (no host
        read-back)."""
        L, c, W = self.L, self.cfg, self.w
        logits = L.bi_matmul(h, W["l%d.router" % i], out_dtype=torch.float32)
        experts, gates = L.bi_moe_route(logits, c.top_k)
        off, _, pos, tok = L.bi_moe_dispatch(experts, c.n_experts)
        xs = L.bi_embedding(h, tok)                  # rows grouped by expert
        f = L.bi_swiglu(L.bi_matmul_grouped(xs, W["l%d.moe_wgu" % i], off))
        ys = L.bi_matmul_grouped(f, W["l%d.moe_wdown" % i], off)
        return L.bi_moe_combine(ys, pos, gates)


def run(sched: Scheduler, model: ToyDecoder, max_steps: int = 1_000_000) -> int:
    """Steps until every request has finished; returns the number of steps."""
    steps = 0
    while not sched.idle() and steps < max_steps:
        plan = sched.plan()
        if plan is None:
            continue
        sched.commit(plan, model.forward(plan))
        steps += 1
    return steps
