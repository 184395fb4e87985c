"""The toy decoder end to end on the GPU: one fixed prompt completed
greedily many times amid random other requests (random prompt lengths,
arrival steps, chunked prefill, decode/prefill mixes, batch sizes from 1 up
to the cap) gives exactly one completion, equal to the prompt's completion
when it runs alone."""
import dataclasses

import numpy as np
import pytest
import torch

import invariant_bi_rmsnorm_03_b200 as bi
import oracle
from gpu_util import TOL_BF16, host_bits, rowwise_normwise, to_f64
from invariant_bi_rmsnorm_03_b200.decoder import (DecoderConfig, PagePool, Request, Scheduler,
                                                  ToyDecoder, run, weight_shapes)
from synth import toy_decoder_weights, unique_completion_workload

pytestmark = pytest.mark.gpu

SMALL = DecoderConfig(hidden=512, layers=2, n_heads=8, n_kv_heads=2, head_dim=64, ffn=1024,
                      vocab=2000)


def completions(L, cfg, weights, reqs, max_batch, budget, num_pages=4096):
    model = ToyDecoder(L, cfg, weights, num_pages, "cuda")
    sched = Scheduler(PagePool(num_pages, seed=3), max_batch=max_batch, token_budget=budget)
    sched.add(reqs)
    run(sched, model)
    assert L.bi_device_status() == bi.Status.OK
    return sched


def test_unique_completion_small():
    L = bi.load()
    w = toy_decoder_weights(weight_shapes(SMALL), seed=4, device="cuda")
    prompt, spec = unique_completion_workload(seed=4, n_target=24, n_other=120, prompt_len=40,
                                              gen_len=24, vocab=SMALL.vocab,
                                              other_prompt_max=300, steps_span=60)
    solo = Request(-1, prompt, 24)
    completions(L, SMALL, w, [solo], max_batch=1, budget=16)  # alone, prompt in chunks of 16
    reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"]) for d in spec]
    completions(L, SMALL, w, reqs, max_batch=48, budget=256)
    outs = {tuple(r.out) for r in reqs if r.tag == "target"}
    assert len(solo.out) == 24
    assert outs == {tuple(solo.out)}


def test_unique_completion_small_fused():
    # RMSNorm folded into the following matmul and the residual adds into
    # the matmul epilogue: other bits than the unfused decoder, but again
    # one completion, the prompt's own.
    cfg = dataclasses.replace(SMALL, fused=True)
    L = bi.load()
    w = toy_decoder_weights(weight_shapes(cfg), seed=4, device="cuda")
    prompt, spec = unique_completion_workload(seed=5, n_target=24, n_other=120, prompt_len=40,
                                              gen_len=24, vocab=cfg.vocab,
                                              other_prompt_max=300, steps_span=60)
    solo = Request(-1, prompt, 24)
    completions(L, cfg, w, [solo], max_batch=1, budget=16)
    reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"]) for d in spec]
    completions(L, cfg, w, reqs, max_batch=48, budget=256)
    outs = {tuple(r.out) for r in reqs if r.tag == "target"}
    assert outs == {tuple(solo.out)}


def test_fused_decoder_pieces_match_the_oracle():
    # The fused model's feed-forward pieces on its own folded weights against
    # the oracle, each fed the GPU's bf16 inputs: RMSNorm folded into the
    # gate/up matmul, and the down matmul added to the residual in place.
    cfg = dataclasses.replace(SMALL, fused=True, layers=1)
    L = bi.load()
    w = toy_decoder_weights(weight_shapes(cfg), seed=6, device="cuda")
    model = ToyDecoder(L, cfg, w, 64, "cuda")
    # the model's norm weights are ones, so the folded weights are the weights
    assert torch.equal(model.wf["l0.wqkv"].view(torch.int16), w["l0.wqkv"].view(torch.int16))
    x = torch.from_numpy(np.random.default_rng(7).standard_normal((37, cfg.hidden))
                         .astype(np.float32)).to("cuda").to(torch.bfloat16)
    gu = L.bi_rmsnorm_matmul(x, model.wf["l0.wgu"], cfg.eps)
    ref = oracle.rmsnorm_matmul(host_bits(x), host_bits(model.wf["l0.wgu"]), cfg.eps)
    assert rowwise_normwise(to_f64(gu), ref).max() <= TOL_BF16
    f = L.bi_swiglu(gu)
    x2 = x.clone()
    L.bi_matmul_residual(f, w["l0.wdown"], x2, out=x2)
    ref2 = oracle.matmul_residual(host_bits(x), host_bits(f), host_bits(w["l0.wdown"]))
    assert rowwise_normwise(to_f64(x2), ref2).max() <= TOL_BF16


def test_full_size_decoder_step_runs():
    # The 8-layer, hidden-4096 model: one mixed step (decode + chunked
    # prefill) and its greedy tokens are the same when the rows run alone.
    cfg = DecoderConfig()
    L = bi.load()
    w = toy_decoder_weights(weight_shapes(cfg), seed=4, device="cuda")
    g = np.random.default_rng(9)
    reqs = [Request(i, g.integers(0, cfg.vocab, size=n).astype(np.int32), 3)
            for i, n in enumerate([64, 300, 5, 64])]
    together = completions(L, cfg, w, reqs, max_batch=4, budget=200, num_pages=256)
    for r in reqs:
        alone = Request(r.rid, r.prompt, 3)
        completions(L, cfg, w, [alone], max_batch=1, budget=64, num_pages=256)
        assert alone.out == r.out, r.rid
    torch.cuda.synchronize()
    assert len(together.finished) == 4


def test_unique_completion_small_with_sampling():
    # temperature 0.8, nucleus 0.95: every target copy carries the same seed,
    # so every copy draws the same tokens however the batch around it looks
    L = bi.load()
    w = toy_decoder_weights(weight_shapes(SMALL), seed=4, device="cuda")
    prompt, spec = unique_completion_workload(seed=5, n_target=24, n_other=120, prompt_len=40,
                                              gen_len=24, vocab=SMALL.vocab,
                                              other_prompt_max=300, steps_span=60)
    tseed = next(d["seed"] for d in spec if d["tag"] == "target")
    solo = Request(-1, prompt, 24, temperature=0.8, top_p=0.95, seed=tseed)
    completions(L, SMALL, w, [solo], max_batch=1, budget=16)
    reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"], temperature=0.8,
                    top_p=0.95, seed=d["seed"]) for d in spec]
    completions(L, SMALL, w, reqs, max_batch=48, budget=256)
    outs = {tuple(r.out) for r in reqs if r.tag == "target"}
    assert outs == {tuple(solo.out)}
    # and sampling did not collapse to the greedy completion
    greedy = Request(-1, prompt, 24)
    completions(L, SMALL, w, [greedy], max_batch=1, budget=64)
    assert tuple(greedy.out) != tuple(solo.out)


def test_unique_completion_small_moe():
    # the same experiment on a mixture-of-experts decoder (16 experts, top 4)
    L = bi.load()
    cfg = DecoderConfig(hidden=512, layers=2, n_heads=8, n_kv_heads=2, head_dim=64, vocab=2000,
                        n_experts=16, top_k=4, expert_ffn=256)
    w = toy_decoder_weights(weight_shapes(cfg), seed=6, device="cuda")
    prompt, spec = unique_completion_workload(seed=7, n_target=16, n_other=80, prompt_len=32,
                                              gen_len=16, vocab=cfg.vocab, other_prompt_max=200,
                                              steps_span=40)
    solo = Request(-1, prompt, 16)
    completions(L, cfg, w, [solo], max_batch=1, budget=16)
    reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"]) for d in spec]
    completions(L, cfg, w, reqs, max_batch=40, budget=256)
    assert {tuple(r.out) for r in reqs if r.tag == "target"} == {tuple(solo.out)}
