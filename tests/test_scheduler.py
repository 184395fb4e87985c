"""Host-side planning of the toy decoder's steps (no GPU): every request's
tokens reach the model once, in order, at consecutive positions, in slots of
its own pages; prompts are chunked to the token budget; decode rows come
first; finished requests return their pages."""
import numpy as np

from invariant_bi_rmsnorm_03_b200.decoder import PagePool, Request, Scheduler, StepPlan
from synth import unique_completion_workload

PAGE = 16


class FakeModel:
    """Checks each plan against the requests' state and returns a token that
    depends only on the request's own history."""

    def __init__(self):
        self.seen = {}      # rid -> list of (position, token)
        self.batch_sizes = []
        self.chunked = 0

    def forward(self, plan: StepPlan) -> np.ndarray:
        T = len(plan.tokens)
        Bd = len(plan.dec)
        assert len(plan.positions) == len(plan.slots) == T
        assert plan.cu_q[-1] == T - Bd and len(plan.cu_q) == len(plan.pre) + 1
        live = set()
        rows = list(plan.dec) + [r for r, _ in plan.pre]
        assert plan.block_table.shape[0] == len(rows)
        for i, r in enumerate(rows):
            assert list(plan.block_table[i, :len(r.pages)]) == r.pages
            live.update(r.pages)
        # decode rows: one token each, the last sampled token, at the next position
        for i, r in enumerate(plan.dec):
            assert plan.tokens[i] == r.out[-1]
            assert plan.positions[i] == len(r.prompt) + len(r.out) - 1
            assert plan.dec_lens[i] == plan.positions[i] + 1
            self._record(r, plan.positions[i], plan.tokens[i], plan.slots[i])
        for k, (r, n) in enumerate(plan.pre):
            lo = Bd + plan.cu_q[k]
            assert plan.cu_q[k + 1] - plan.cu_q[k] == n
            assert plan.ctx[k] == r.done_prompt
            if n < len(r.prompt):
                self.chunked += 1
            for j in range(n):
                assert plan.positions[lo + j] == r.done_prompt + j
                assert plan.tokens[lo + j] == r.prompt[r.done_prompt + j]
                self._record(r, plan.positions[lo + j], plan.tokens[lo + j], plan.slots[lo + j])
        assert len(set(plan.slots.tolist())) == T
        self.batch_sizes.append(len(rows))
        return np.array([(r.rid * 7919 + len(r.out) * 104729) % 32000 for r in plan.sample_reqs])

    def _record(self, r, pos, tok, slot):
        page, off = divmod(int(slot), PAGE)
        assert page == r.pages[pos // PAGE] and off == pos % PAGE
        self.seen.setdefault(r.rid, []).append((int(pos), int(tok)))


def drive(reqs, max_batch=256, budget=2048, num_pages=20000):
    sched = Scheduler(PagePool(num_pages, seed=1), max_batch=max_batch, token_budget=budget)
    sched.add(reqs)
    model = FakeModel()
    steps = 0
    while not sched.idle():
        plan = sched.plan()
        if plan is None:
            continue
        sched.commit(plan, model.forward(plan))
        steps += 1
        assert len(sched.pool.free) + sum(len(r.pages) for r in sched.running) == num_pages
    return sched, model, steps


def test_every_token_once_in_order():
    g = np.random.default_rng(5)
    reqs = [Request(i, g.integers(0, 32000, size=int(g.integers(1, 200))).astype(np.int32),
                    int(g.integers(1, 40)), arrival=int(g.integers(0, 30))) for i in range(60)]
    sched, model, _ = drive(reqs, max_batch=16, budget=96)
    assert len(sched.finished) == 60
    for r in reqs:
        assert len(r.out) == r.max_new and r.pages == []
        seen = model.seen[r.rid]
        assert [p for p, _ in seen] == list(range(len(r.prompt) + r.max_new - 1))
        assert [t for _, t in seen[:len(r.prompt)]] == list(r.prompt)
        assert [t for _, t in seen[len(r.prompt):]] == r.out[:-1]
    assert model.chunked > 0
    assert max(model.batch_sizes) == 16 and min(model.batch_sizes) == 1


def test_unique_completion_workload_sweeps_batch_sizes():
    _, spec = unique_completion_workload(seed=4, n_target=40, n_other=300, gen_len=32,
                                         other_prompt_max=128, steps_span=300)
    reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"]) for d in spec]
    sched, model, steps = drive(reqs, max_batch=64, budget=512)
    assert len(sched.finished) == 340
    assert min(model.batch_sizes) <= 4 and max(model.batch_sizes) >= 48
    outs = {tuple(r.out) for r in reqs if r.tag == "target"}
    assert len(outs) == 40  # the fake token depends on rid: all distinct, all complete
    assert all(len(r.out) == 32 for r in reqs if r.tag == "target")
