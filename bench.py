"""Benchmark of the batch-invariant forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input,
shaped like the serving workloads the reports describe:
  * bi_kv_write   the step's new tokens into the paged caches (256 decode
                  tokens; the 8192 prompt tokens of the prefill sequence)
  * bi_rmsnorm    x[2048, 4096] (hidden 4096)
  * bi_matmul     x[2048, 4096] @ W[12288, 4096]^T
  * bi_attention_decode   256 requests, GQA 64/4, d=128, KV lengths
                          U(1, 32768), shuffled 16-token pages, 256-key splits
  * bi_attention_prefill  one causal 8192-token prompt, 32/8 heads, d=128
The L2 cache (126 MB) is flushed between steps with a 512 MB write; each
step is timed with CUDA events on the launching stream.

``value`` is the batch-invariant GEMM throughput (TFLOP/s, all ranks'
matmul FLOPs over the slowest rank's matmul time); ``split_kv_attn`` carries
the decode attention's HBM throughput.  ``roofline`` is for the kernel that
takes most of the step.  ``e2e`` repeats the measurement through the same
public calls with the step's activations copied from pinned host memory and
its results copied back inside the timed region.  ``cpu_baseline`` is the
fp64 oracle timed on a bounded sample on this host's cores.
``--impl reference`` times that oracle alone (the only other implementation
of the method here) and prints its own line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-invariant GEMM TFLOP/s + split-KV attn GB/s (% of peak); bitwise match"
WORKLOAD = ("hidden-4096 RMSNorm + matmul (M=2048, N=12288) + paged decode attention "
            "(B=256, GQA 64/4, d=128, KV U(1,32768)) + causal prefill (8192 tokens, 32/8 heads)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}

# Workload sizes.
H, M_ROWS, N_COLS = 4096, 2048, 12288
DEC_B, DEC_HQ, DEC_HKV, D = 256, 64, 4, 128
DEC_MAXLEN = 32768
PRE_S, PRE_HQ, PRE_HKV = 8192, 32, 8


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- workload

class Workload:
    """Device-resident inputs of one step (seeded, synthetic)."""

    def __init__(self, torch, bi, dev, seed_base=0):
        from synth import (decode_lengths, norm_matmul, normal_bf16, page_table, rng,
                           slot_mapping, torch_normal_bf16)

        self.torch = torch
        T = torch
        nm = norm_matmul(seed=1 + seed_base, M=M_ROWS, H=H, N=N_COLS)
        self.x = T.from_numpy(nm["x"].view(np.int16)).to(dev).view(T.bfloat16)
        self.w = T.from_numpy(nm["w"].view(np.int16)).to(dev).view(T.bfloat16)
        self.W = T.from_numpy(nm["W"].view(np.int16)).to(dev).view(T.bfloat16)
        self.eps = nm["eps"]
        self.y = T.empty_like(self.x)
        self.c = T.empty((M_ROWS, N_COLS), dtype=T.bfloat16, device=dev)
        self.x_np, self.W_np, self.w_np = nm["x"], nm["W"], nm["w"]

        # decode: lengths include the step's new token
        g = rng(2 + seed_base)
        lens = decode_lengths(2 + seed_base, DEC_B, DEC_MAXLEN)
        bt, num_pages = page_table(g, lens, max_pages=DEC_MAXLEN // 16)
        self.dec_lens_np, self.dec_bt_np = lens, bt
        shape = (num_pages, DEC_HKV, 16, D)
        self.dec_kv = bi.PagedKV(torch_normal_bf16(shape, 1000 + seed_base, dev),
                                 torch_normal_bf16(shape, 2000 + seed_base, dev),
                                 T.from_numpy(bt).to(dev))
        self.dec_q = T.from_numpy(normal_bf16(g, (DEC_B, DEC_HQ, D)).view(np.int16)).to(dev).view(T.bfloat16)
        self.dec_knew = T.from_numpy(normal_bf16(g, (DEC_B, DEC_HKV, D)).view(np.int16)).to(dev).view(T.bfloat16)
        self.dec_vnew = T.from_numpy(normal_bf16(g, (DEC_B, DEC_HKV, D)).view(np.int16)).to(dev).view(T.bfloat16)
        slots = np.array([slot_mapping(bt, b, [int(lens[b]) - 1])[0] for b in range(DEC_B)])
        self.dec_slots = T.from_numpy(slots).to(dev)
        self.dec_lens = T.from_numpy(lens).to(dev)
        self.dec_o = T.empty_like(self.dec_q)
        self.dec_ws_bytes = bi.load().bi_attention_decode_workspace_bytes(
            self.dec_kv, DEC_B, DEC_HQ, DEC_MAXLEN)
        self.dec_ws = T.empty(max(self.dec_ws_bytes, 16), dtype=T.uint8, device=dev)

        # prefill: one prompt of PRE_S tokens into an empty (NaN) cache
        gp = rng(3 + seed_base)
        self.pre_q_np = normal_bf16(gp, (PRE_S, PRE_HQ, D))
        self.pre_q = T.from_numpy(self.pre_q_np.view(np.int16)).to(dev).view(T.bfloat16)
        self.pre_k = T.from_numpy(normal_bf16(gp, (PRE_S, PRE_HKV, D)).view(np.int16)).to(dev).view(T.bfloat16)
        self.pre_v = T.from_numpy(normal_bf16(gp, (PRE_S, PRE_HKV, D)).view(np.int16)).to(dev).view(T.bfloat16)
        pbt, pnp = page_table(gp, [PRE_S])
        self.pre_bt_np = pbt
        self.pre_kv = bi.PagedKV(T.full((pnp, PRE_HKV, 16, D), float("nan"), dtype=T.bfloat16, device=dev),
                                 T.full((pnp, PRE_HKV, 16, D), float("nan"), dtype=T.bfloat16, device=dev),
                                 T.from_numpy(pbt).to(dev))
        self.pre_slots = T.from_numpy(slot_mapping(pbt, 0, np.arange(PRE_S))).to(dev)
        self.pre_cu = T.tensor([0, PRE_S], dtype=T.int32, device=dev)
        self.pre_ctx = T.tensor([0], dtype=T.int32, device=dev)
        self.pre_o = T.empty_like(self.pre_q)

        self.flush = T.empty(512 * 1024 * 1024, dtype=T.uint8, device=dev)

        # algorithmic work per step
        self.gemm_flops = 2.0 * M_ROWS * N_COLS * H
        self.norm_bytes = 2.0 * M_ROWS * H * 2 + 2 * H
        Lsum = float(lens.astype(np.int64).sum())
        self.dec_bytes = (Lsum * DEC_HKV * D * 2 * 2            # K and V rows read once
                          + 2.0 * DEC_B * DEC_HQ * D * 2          # q in, o out
                          + 4.0 * float(((lens + 15) // 16).sum())  # block-table entries
                          + 4.0 * DEC_B)                          # lengths
        self.pre_flops = 4.0 * PRE_HQ * D * (PRE_S * (PRE_S + 1) / 2.0)
        # new K and V rows read once and written once
        self.kvw_bytes = 4.0 * D * 2 * (DEC_B * DEC_HKV + PRE_S * PRE_HKV)

    def step(self, L, ev=None):
        """One pass of the hot path.  ev: 7 CUDA events recorded between kernels."""
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        rec(0)
        L.bi_kv_write(self.dec_kv, self.dec_knew, self.dec_vnew, self.dec_slots)
        L.bi_kv_write(self.pre_kv, self.pre_k, self.pre_v, self.pre_slots)
        rec(1)
        L.bi_rmsnorm(self.x, self.w, self.eps, out=self.y)
        rec(2)
        L.bi_matmul(self.y, self.W, out=self.c)
        rec(3)
        L.bi_attention_decode(self.dec_kv, self.dec_q, self.dec_lens, DEC_MAXLEN, out=self.dec_o,
                              ws=self.dec_ws)
        rec(4)
        L.bi_attention_prefill(self.pre_kv, self.pre_q, self.pre_cu, self.pre_ctx, PRE_S,
                               out=self.pre_o)
        rec(5)

    def launches_per_step(self, L) -> int:
        # two cache writes, RMSNorm, matmul, the decode launch order (the
        # bench's batch has more blocks than SMs), decode attention, its
        # combine when a sequence is split over blocks (the workspace then
        # holds split records beyond the order array), prefill
        ws = L.bi_attention_decode_workspace_bytes(self.dec_kv, DEC_B, DEC_HQ, DEC_MAXLEN)
        order = (4 * DEC_B + 255) // 256 * 256
        return 2 + 1 + 1 + 1 + 1 + (1 if ws > order else 0) + 1


# ---------------------------------------------------------------- clocks

def pci_bus_id(props) -> bytes | None:
    """NVML's bus-id string ("DDDDDDDD:BB:DD.0") for a torch device, built
    from the integer PCI domain, bus and device numbers torch reports."""
    try:
        dom, bus, dv = (int(getattr(props, k)) for k in ("pci_domain_id", "pci_bus_id",
                                                          "pci_device_id"))
    except (AttributeError, TypeError, ValueError):
        return None
    return ("%08X:%02X:%02X.0" % (dom, bus, dv)).encode()


class Clocks:
    """SM clock and clock-event reasons of this process's GPU, read through
    NVML by a background thread every few milliseconds.  ``mark()`` brackets
    the timed region; ``stop()`` summarises the samples taken inside it (or
    the nearest ones when the region is shorter than the sampling period).
    Read-only: no clock or other GPU setting is changed."""

    NAMES = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
             ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
             ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
             ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, bus_id: bytes | None, index: int, period_s: float = 0.005):
        import threading

        self.samples, self.window, self.err = [], [None, None], None
        try:
            import pynvml as nv

            nv.nvmlInit()
            self.h = None
            if isinstance(bus_id, bytes):  # never an int: NVML takes it as a char*
                try:
                    self.h = nv.nvmlDeviceGetHandleByPciBusId(bus_id)
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = nv.nvmlDeviceGetHandleByIndex(index)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it, do not guess
            self.nv, self.err = None, "nvml unavailable: %s" % e
            return
        self.stop_flag = threading.Event()
        self.period = period_s
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception as e:
                self.err = str(e)
            self.stop_flag.wait(self.period)

    def mark(self, which: int):
        self.window[which] = time.perf_counter()

    def stop(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err]}
        self.stop_flag.set()
        self.t.join(timeout=2)
        t0, t1 = self.window
        inside = [s for s in self.samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
        if not inside and self.samples and t0 is not None:
            mid = 0.5 * (t0 + (t1 or t0))
            inside = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:2]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = sorted({n for _, _, rs in inside for n, attr in self.NAMES
                          if rs & getattr(self.nv, attr, 0)})
        return {"sm_mhz": statistics.median([s[1] for s in inside]), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "source": "nvml, 5 ms period",
                "window_ms": (t1 - t0) * 1e3 if t1 and t0 else None}


# ---------------------------------------------------------------- ours

HOST_AHEAD_CYCLES = 2_000_000  # ~1 ms of GPU clock


def host_ahead(torch):
    """A GPU spin of ~1 ms queued after the L2 flush and before the timed
    region, so that the host has queued every launch of the timed region
    before it starts: the device times then never include a wait for the
    host (the ctypes calls take tens of microseconds each, longer than the
    shortest kernels)."""
    torch.cuda._sleep(HOST_AHEAD_CYCLES)


def timed_steps(torch, L, wl, steps, warmup, dist=None, clocks=None):
    for _ in range(warmup):
        wl.flush.zero_()
        wl.step(L)
    torch.cuda.synchronize()
    per = np.zeros((steps, 5))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    if clocks is not None:
        clocks.mark(0)
    for i in range(steps):
        wl.flush.zero_()
        host_ahead(torch)
        wl.step(L, evs[i])
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.mark(1)
    wall = time.perf_counter() - t0
    if dist is not None:
        dist.barrier()
    for i in range(steps):
        e = evs[i]
        per[i] = [e[j].elapsed_time(e[j + 1]) for j in range(5)]
    return per, wall  # ms: kv_write, rmsnorm, matmul, decode, prefill


def e2e_steps(torch, L, wl, steps, warmup):
    """The same step through the public calls with host buffers: pinned host
    activations copied in and results copied out inside the timed region."""
    T = torch
    hx = wl.x.cpu().pin_memory()
    hq = wl.dec_q.cpu().pin_memory()
    hkn, hvn = wl.dec_knew.cpu().pin_memory(), wl.dec_vnew.cpu().pin_memory()
    hpq = wl.pre_q.cpu().pin_memory()
    hpk, hpv = wl.pre_k.cpu().pin_memory(), wl.pre_v.cpu().pin_memory()
    hc = T.empty(wl.c.shape, dtype=wl.c.dtype).pin_memory()
    ho = T.empty(wl.dec_o.shape, dtype=wl.dec_o.dtype).pin_memory()
    hpo = T.empty(wl.pre_o.shape, dtype=wl.pre_o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hx, hq, hkn, hvn, hpq, hpk, hpv))
    d2h = sum(t.numel() * t.element_size() for t in (hc, ho, hpo))

    def one(ev=None):
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        rec(0)
        wl.x.copy_(hx, non_blocking=True)
        L.bi_rmsnorm(wl.x, wl.w, wl.eps, out=wl.y)
        L.bi_matmul(wl.y, wl.W, out=wl.c)
        hc.copy_(wl.c, non_blocking=True)
        rec(1)
        wl.dec_q.copy_(hq, non_blocking=True)
        wl.dec_knew.copy_(hkn, non_blocking=True)
        wl.dec_vnew.copy_(hvn, non_blocking=True)
        L.bi_kv_write(wl.dec_kv, wl.dec_knew, wl.dec_vnew, wl.dec_slots)
        L.bi_attention_decode(wl.dec_kv, wl.dec_q, wl.dec_lens, DEC_MAXLEN, out=wl.dec_o,
                              ws=wl.dec_ws)
        ho.copy_(wl.dec_o, non_blocking=True)
        rec(2)
        wl.pre_q.copy_(hpq, non_blocking=True)
        wl.pre_k.copy_(hpk, non_blocking=True)
        wl.pre_v.copy_(hpv, non_blocking=True)
        L.bi_kv_write(wl.pre_kv, wl.pre_k, wl.pre_v, wl.pre_slots)
        L.bi_attention_prefill(wl.pre_kv, wl.pre_q, wl.pre_cu, wl.pre_ctx, PRE_S, out=wl.pre_o)
        hpo.copy_(wl.pre_o, non_blocking=True)
        rec(3)

    for _ in range(warmup):
        wl.flush.zero_()
        one()
    torch.cuda.synchronize()
    evs = [[T.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        wl.flush.zero_()
        one(evs[i])
    torch.cuda.synchronize()
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(3)] for e in evs])
    return per, h2d, d2h


def e2e_pipelined(torch, L, wl, steps, legs=("gemm", "decode", "prefill")):
    """The step (or some of its legs) through the public calls as a serving
    loop runs it: step k's inputs are copied in from pinned host memory on
    one stream while step k-1 computes on a second and step k-2's results
    are copied out on a third.  Device inputs and outputs are double
    buffered; every copy and every launch of the K steps is inside the timed
    region (first copy-in to last copy-out), each step starts with the L2
    flush.  Returns the mean time of a step in ms and whether the last
    step's results, copied out, equal the step computed plainly bit for bit."""
    T = torch
    dev = wl.x.device
    host_in = {"x": wl.x, "dec_q": wl.dec_q, "dec_knew": wl.dec_knew, "dec_vnew": wl.dec_vnew,
               "pre_q": wl.pre_q, "pre_k": wl.pre_k, "pre_v": wl.pre_v}
    hin = {k: v.cpu().pin_memory() for k, v in host_in.items()}
    outs = {"c": wl.c, "dec_o": wl.dec_o, "pre_o": wl.pre_o}
    hout = {k: T.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in outs.items()}
    bufs = [dict(host_in, y=wl.y, **outs),
            {**{k: T.empty_like(v) for k, v in host_in.items()}, "y": T.empty_like(wl.y),
             **{k: T.empty_like(v) for k, v in outs.items()}}]
    ins_of = {"gemm": ["x"], "decode": ["dec_q", "dec_knew", "dec_vnew"],
              "prefill": ["pre_q", "pre_k", "pre_v"]}
    outs_of = {"gemm": ["c"], "decode": ["dec_o"], "prefill": ["pre_o"]}

    def compute(bf):
        if "gemm" in legs:
            L.bi_rmsnorm(bf["x"], wl.w, wl.eps, out=bf["y"])
            L.bi_matmul(bf["y"], wl.W, out=bf["c"])
        if "decode" in legs:
            L.bi_kv_write(wl.dec_kv, bf["dec_knew"], bf["dec_vnew"], wl.dec_slots)
            L.bi_attention_decode(wl.dec_kv, bf["dec_q"], wl.dec_lens, DEC_MAXLEN, out=bf["dec_o"],
                                  ws=wl.dec_ws)
        if "prefill" in legs:
            L.bi_kv_write(wl.pre_kv, bf["pre_k"], bf["pre_v"], wl.pre_slots)
            L.bi_attention_prefill(wl.pre_kv, bf["pre_q"], wl.pre_cu, wl.pre_ctx, PRE_S,
                                   out=bf["pre_o"])

    s_in, s_c, s_out = T.cuda.Stream(dev), T.cuda.Stream(dev), T.cuda.Stream(dev)
    names_in = [n for lg in legs for n in ins_of[lg]]
    names_out = [n for lg in legs for n in outs_of[lg]]

    def run(k_steps, timed):
        ev = lambda: T.cuda.Event(enable_timing=timed)  # noqa: E731
        comp_done, out_done = [], []
        T.cuda.synchronize()
        t0, t1 = ev(), ev()
        t0.record(s_in)
        for k in range(k_steps):
            bf = bufs[k % 2]
            with T.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp_done[k - 2])
                for n in names_in:
                    bf[n].copy_(hin[n], non_blocking=True)
                in_ready = ev()
                in_ready.record(s_in)
            with T.cuda.stream(s_c):
                s_c.wait_event(in_ready)
                if k >= 2:
                    s_c.wait_event(out_done[k - 2])
                wl.flush.zero_()
                compute(bf)
                done = ev()
                done.record(s_c)
                comp_done.append(done)
            with T.cuda.stream(s_out):
                s_out.wait_event(done)
                for n in names_out:
                    hout[n].copy_(bf[n], non_blocking=True)
                od = ev()
                od.record(s_out)
                out_done.append(od)
        s_out.wait_event(out_done[-1])
        t1.record(s_out)
        T.cuda.synchronize()
        return t0.elapsed_time(t1) / k_steps if timed else None

    run(3, False)
    ms = run(steps, True)
    # the pipeline's last results against the same step run plainly
    ref = {n: T.empty_like(outs[n]) for n in names_out}
    with T.cuda.stream(s_c):
        bf = dict(bufs[0])
        for n in names_in:
            bf[n].copy_(hin[n])
        bf.update(ref)
        compute(bf)
    T.cuda.synchronize()
    same = all(T.equal(hout[n].view(T.int16), ref[n].cpu().view(T.int16)) for n in names_out)
    del bufs, ref
    return ms, same


def invariance_checks(torch, L, wl) -> dict:
    """Bitwise checks on the bench's own data: rows against smaller batches,
    a request alone against the batch, the last prompt token in decode
    against prefill."""
    T = torch
    eq = lambda a, b: bool(T.equal(a.contiguous().view(T.int16), b.contiguous().view(T.int16)))  # noqa: E731
    out = {}
    wl.step(L)
    T.cuda.synchronize()
    ok = True
    for M in (1, 7, 128, 1000):
        ok &= eq(L.bi_rmsnorm(wl.x[:M], wl.w, wl.eps), wl.y[:M])
        ok &= eq(L.bi_matmul(wl.y[:M], wl.W), wl.c[:M])
    out["gemm_rows_vs_batch"] = ok
    ok = True
    for b in (0, 17, 255):
        kv1 = type(wl.dec_kv)(wl.dec_kv.k_cache, wl.dec_kv.v_cache,
                              wl.dec_kv.block_table[b:b + 1].contiguous())
        o1 = L.bi_attention_decode(kv1, wl.dec_q[b:b + 1].contiguous(), wl.dec_lens[b:b + 1],
                                   int(wl.dec_lens_np[b]))
        ok &= eq(o1[0], wl.dec_o[b])
    out["decode_request_vs_batch"] = ok
    t = PRE_S - 1
    od = L.bi_attention_decode(wl.pre_kv, wl.pre_q[t:t + 1].contiguous(),
                               T.tensor([PRE_S], dtype=T.int32, device=wl.x.device), PRE_S)
    out["decode_vs_prefill"] = eq(od[0], wl.pre_o[t])
    out["all"] = all(out.values())
    return out


def rmsnorm_context(torch, L, wl) -> dict:
    """What bounds RMSNorm at the step's size: a plain device copy of the same
    bytes timed the same way, and RMSNorm on 65536 rows (1 GiB moved)."""
    T = torch

    def timed(fn, reps=20):
        for _ in range(3):
            wl.flush.zero_()
            fn()
        ev = [(T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            wl.flush.zero_()
            host_ahead(T)
            a.record()
            fn()
            b.record()
        T.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in ev]))

    y = T.empty_like(wl.x)
    copy_ms = timed(lambda: y.copy_(wl.x))
    big = T.empty((65536, H), dtype=T.bfloat16, device=wl.x.device)
    big.copy_(wl.x.repeat(32, 1))
    big_out = T.empty_like(big)
    big_ms = timed(lambda: L.bi_rmsnorm(big, wl.w, wl.eps, out=big_out), reps=10)
    # The step's size launched back to back over the 32 distinct 2048-row
    # slices of the same 1 GiB (more than L2, so every slice comes from HBM):
    # the kernel's rate when launches follow each other, without the fixed
    # cost of one isolated launch (an empty kernel timed like the step's
    # launches is reported beside it).
    slices = [(big[i * M_ROWS:(i + 1) * M_ROWS], big_out[i * M_ROWS:(i + 1) * M_ROWS])
              for i in range(65536 // M_ROWS)]

    def stream():
        for xs, ys in slices:
            L.bi_rmsnorm(xs, wl.w, wl.eps, out=ys)
    stream_ms = timed(stream, reps=10) / len(slices)
    # the same 32 launches captured once in a CUDA graph and replayed (the
    # launches of a captured serving loop)
    graph_ms = None
    try:
        side = T.cuda.Stream(wl.x.device)
        side.wait_stream(T.cuda.current_stream())
        with T.cuda.stream(side):
            stream()  # warm-up on the capture stream
        T.cuda.current_stream().wait_stream(side)
        T.cuda.synchronize()
        graph = T.cuda.CUDAGraph()
        with T.cuda.graph(graph):
            stream()
        graph_ms = timed(graph.replay, reps=10) / len(slices)
        del graph
    except RuntimeError:
        graph_ms = None
    e = T.empty(1, device=wl.x.device)
    empty_ms = timed(lambda: e.zero_())
    nbytes = 2.0 * 2 * M_ROWS * H
    big_bytes = 2.0 * 2 * 65536 * H
    del big, big_out, slices
    return {"copy_same_bytes_ms": copy_ms, "copy_same_bytes_GB/s": nbytes / (copy_ms * 1e-3) / 1e9,
            "rmsnorm_M65536_ms": big_ms, "rmsnorm_M65536_GB/s": big_bytes / (big_ms * 1e-3) / 1e9,
            "back_to_back_M2048_ms": stream_ms,
            "back_to_back_M2048_GB/s": nbytes / (stream_ms * 1e-3) / 1e9,
            "graph_M2048_ms": graph_ms,
            "graph_M2048_GB/s": nbytes / (graph_ms * 1e-3) / 1e9 if graph_ms else None,
            "empty_kernel_ms": empty_ms}


def _median_ms(torch, fn, flush, reps=15, warm=3):
    """Median CUDA-event time of fn() on the current stream, L2 flushed
    (a 512 MB write) before every launch and the launch queued before its
    start event runs (host_ahead)."""
    T = torch
    for _ in range(warm):
        flush.zero_()
        fn()
    ev = [(T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        host_ahead(T)
        a.record()
        fn()
        b.record()
    T.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


def cost_of_invariance(torch, L, Lv, wl) -> dict:
    """Each kernel of the step at several sizes in both builds (the
    invariant build and the variant-off build, whose matmul splits K when the
    tiles cannot fill the GPU and whose decode blocks pre-merge their own
    range), the cuBLAS product (torch.matmul) at the same shapes as context,
    and the weight bandwidth of the small-M products.  Medians of CUDA-event
    times, L2 flushed before each launch."""
    T = torch
    dev = wl.x.device
    pk, _ = peaks()
    out = {"matmul": [], "rmsnorm": [], "attention_decode": [], "attention_prefill": []}
    # matmul: M rows of the step's normalised x times W [N, 4096]
    Ws = {N_COLS: wl.W}
    for N in (4096, 28672):
        Ws[N] = T.randn((N, H), device=dev, dtype=T.float32).mul_(0.02).to(T.bfloat16)
    for M in (64, 256, 2048):
        for N in (4096, N_COLS, 28672):
            if M == 2048 and N != N_COLS:
                continue
            a, W = wl.y[:M], Ws[N]
            c = T.empty((M, N), dtype=T.bfloat16, device=dev)
            need = max(Lv.bi_matmul_workspace_bytes(M, N, H), 16)
            ws = T.empty(need, dtype=T.uint8, device=dev)
            ms_i = _median_ms(T, lambda: L.bi_matmul(a, W, out=c), wl.flush)
            ms_v = _median_ms(T, lambda: Lv.bi_matmul(a, W, out=c, ws=ws), wl.flush)
            ms_cb = _median_ms(T, lambda: T.matmul(a, W.t()), wl.flush)
            flops = 2.0 * M * N * H
            wbytes = 2.0 * N * H
            out["matmul"].append({
                "M": M, "N": N, "K": H, "invariant_ms": ms_i, "variant_off_ms": ms_v,
                "overhead": ms_i / ms_v - 1.0, "k_splits_variant_off":
                    (need // (4 * M * N)) if need > 16 else 1,
                "cublas_ms": ms_cb, "vs_cublas": ms_i / ms_cb - 1.0,
                "TFLOP/s": flops / (ms_i * 1e-3) / 1e12,
                "frac_bf16": flops / (ms_i * 1e-3) / 1e12 / pk["bf16_tflops"],
                "weight_GB/s": wbytes / (ms_i * 1e-3) / 1e9,
                "weight_frac_hbm": wbytes / (ms_i * 1e-3) / 1e9 / pk["hbm_gbs"]})
    del Ws
    for M in (64, 256, 2048):
        x = wl.x[:M]
        y = T.empty_like(x)
        ms_i = _median_ms(T, lambda: L.bi_rmsnorm(x, wl.w, wl.eps, out=y), wl.flush)
        ms_v = _median_ms(T, lambda: Lv.bi_rmsnorm(x, wl.w, wl.eps, out=y), wl.flush)
        out["rmsnorm"].append({"M": M, "H": H, "invariant_ms": ms_i, "variant_off_ms": ms_v,
                               "overhead": ms_i / ms_v - 1.0})
    # decode: the first B requests of the step's batch
    for B in (1, 16, DEC_B):
        kv = type(wl.dec_kv)(wl.dec_kv.k_cache, wl.dec_kv.v_cache,
                             wl.dec_kv.block_table[:B].contiguous())
        q, sl = wl.dec_q[:B].contiguous(), wl.dec_lens[:B].contiguous()
        o = T.empty_like(q)
        mx = int(wl.dec_lens_np[:B].max())
        need = max(L.bi_attention_decode_workspace_bytes(kv, B, DEC_HQ, mx),
                   Lv.bi_attention_decode_workspace_bytes(kv, B, DEC_HQ, mx), 16)
        ws = T.empty(need, dtype=T.uint8, device=dev)
        ms_i = _median_ms(T, lambda: L.bi_attention_decode(kv, q, sl, mx, out=o, ws=ws), wl.flush)
        ms_v = _median_ms(T, lambda: Lv.bi_attention_decode(kv, q, sl, mx, out=o, ws=ws), wl.flush)
        nbytes = float(wl.dec_lens_np[:B].astype(np.int64).sum()) * DEC_HKV * D * 4
        out["attention_decode"].append({
            "B": B, "kv_tokens": int(wl.dec_lens_np[:B].sum()), "invariant_ms": ms_i,
            "variant_off_ms": ms_v, "overhead": ms_i / ms_v - 1.0,
            "GB/s": nbytes / (ms_i * 1e-3) / 1e9})
    ms_i = _median_ms(T, lambda: L.bi_attention_prefill(wl.pre_kv, wl.pre_q, wl.pre_cu, wl.pre_ctx,
                                                         PRE_S, out=wl.pre_o), wl.flush, reps=7)
    ms_v = _median_ms(T, lambda: Lv.bi_attention_prefill(wl.pre_kv, wl.pre_q, wl.pre_cu, wl.pre_ctx,
                                                          PRE_S, out=wl.pre_o), wl.flush, reps=7)
    out["attention_prefill"].append({"S": PRE_S, "invariant_ms": ms_i, "variant_off_ms": ms_v,
                                     "overhead": ms_i / ms_v - 1.0,
                                     "note": "one prefill kernel in both builds"})
    return out


def cpu_baseline(wl, budget_s: float = 20.0) -> dict:
    """The oracle (fp64, OpenMP) on a bounded sample of the same workload."""
    import oracle
    from synth import kv_from_blocks

    cores = oracle.num_threads()
    # matmul: rows of the step's x (after RMSNorm, which the oracle recomputes)
    t0 = time.perf_counter()
    rows = 0
    while time.perf_counter() - t0 < budget_s / 2 and rows < M_ROWS:
        xs = wl.x_np[rows:rows + 8]
        oracle.matmul(xs, wl.W_np)
        rows += xs.shape[0]
    tg = time.perf_counter() - t0
    gemm_tflops = 2.0 * rows * N_COLS * H / tg / 1e12
    # decode attention: whole requests of the batch (device-to-host copies untimed)
    import torch

    kc, vc = wl.dec_kv.k_cache, wl.dec_kv.v_cache
    tstart = time.perf_counter()
    ta, done, nbytes = 0.0, 0, 0.0
    order = np.argsort(wl.dec_lens_np)
    while time.perf_counter() - tstart < budget_s / 2 and done < 16:
        b = int(order[(done * 16) % DEC_B])
        Lb = int(wl.dec_lens_np[b])
        pages = wl.dec_bt_np[b, :(Lb + 15) // 16].tolist()
        k = kv_from_blocks(kc[pages].view(torch.int16).cpu().numpy().view(np.uint16))
        v = kv_from_blocks(vc[pages].view(torch.int16).cpu().numpy().view(np.uint16))
        bt = np.arange(len(pages), dtype=np.int32)[None, :]
        q = wl.dec_q[b].view(torch.int16).cpu().numpy().view(np.uint16)
        ts = time.perf_counter()
        oracle.attention(q, np.zeros(DEC_HQ), np.arange(DEC_HQ), np.full(DEC_HQ, Lb - 1), DEC_HQ,
                         k, v, bt)
        ta += time.perf_counter() - ts
        nbytes += Lb * DEC_HKV * D * 4.0 + 2 * DEC_HQ * D * 2
        done += 1
    return {"value": gemm_tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": "matmul: %d of %d rows of x[2048,4096] times W[12288,4096]^T; decode: %d "
                      "whole requests of the batch" % (rows, M_ROWS, done),
            "split_kv_attn_gbs": nbytes / ta / 1e9 if ta > 0 else None}


def traffic_record(kernel_src: str, name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(name)
    if not rec:
        return None
    with open(os.path.join(ROOT, "invariant_bi_rmsnorm_03_b200", "csrc", kernel_src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if rec.get("source_sha") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The largest value of ``v`` over all ranks (every rank gets it)."""
    if dist is None:
        return v
    import torch

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank processes
    ``units_per_rank`` (replicas, weak scaling), over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


def run_ours(args):
    import torch

    import invariant_bi_rmsnorm_03_b200 as bi

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td

        torch.cuda.set_device(local)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L = bi.load()
    wl = Workload(torch, bi, dev, seed_base=0)
    launches = wl.launches_per_step(L)

    clocks = Clocks(pci_bus_id(torch.cuda.get_device_properties(dev)), local)
    per, wall = timed_steps(torch, L, wl, args.steps, args.warmup, dist, clocks)
    clk = clocks.stop()
    mean = per.mean(axis=0)  # ms per kernel group
    step_ms = float(per.sum(axis=1).mean())

    # whole-job figures: all ranks' work over the slowest rank's time
    def maxall(v):
        return max_over_ranks(v, dist, dev)

    gemm_ms = maxall(float(mean[2]))
    dec_ms = maxall(float(mean[3]))
    pre_ms = maxall(float(mean[4]))
    norm_ms = maxall(float(mean[1]))
    kvw_ms = maxall(float(mean[0]))
    step_ms = maxall(step_ms)
    gemm_tf = whole_job(wl.gemm_flops, world, gemm_ms) / 1e12
    dec_gbs = whole_job(wl.dec_bytes, world, dec_ms) / 1e9

    # e2e through host buffers
    e2e_per, h2d, d2h = e2e_steps(torch, L, wl, max(2, args.steps // 2), 1)
    pipe_steps = max(4, args.steps // 2)
    pipe = [e2e_pipelined(torch, L, wl, pipe_steps, legs)
            for legs in (("gemm",), ("decode",), ("gemm", "decode", "prefill"))]
    pipe_gemm_ms, pipe_dec_ms, pipe_step_ms = (maxall(ms) for ms, _ in pipe)
    pipe_same = all(same for _, same in pipe)
    e2e_gemm_ms = maxall(float(e2e_per[:, 0].mean()))
    e2e_dec_ms = maxall(float(e2e_per[:, 1].mean()))
    e2e_step_ms = maxall(float(e2e_per.sum(axis=1).mean()))
    e2e_pre_ms = maxall(float(e2e_per[:, 2].mean()))

    # variant-off build on the same step (the cost of invariance)
    Lv = bi.load(variant=True)
    wl_v_ws = Lv.bi_attention_decode_workspace_bytes(wl.dec_kv, DEC_B, DEC_HQ, DEC_MAXLEN)
    if wl_v_ws > wl.dec_ws.numel():
        wl.dec_ws = torch.empty(wl_v_ws, dtype=torch.uint8, device=dev)
    per_v, _ = timed_steps(torch, Lv, wl, max(3, args.steps // 2), 2, dist)
    mean_v = per_v.mean(axis=0)
    names = ["kv_write", "rmsnorm", "matmul", "attention_decode", "attention_prefill"]
    overhead = {n: float(mean[i] / mean_v[i] - 1.0) for i, n in enumerate(names)}
    overhead["step"] = float(per.sum(axis=1).mean() / per_v.sum(axis=1).mean() - 1.0)

    coi = cost_of_invariance(torch, L, Lv, wl) if rank == 0 else None
    checks = invariance_checks(torch, L, wl)
    rms_ctx = rmsnorm_context(torch, L, wl)
    uc = None
    if rank == 0 and args.uc_targets > 0:
        # the end-to-end check on the toy decoder: one prompt completed by
        # --uc-targets copies amid as many other requests, in both builds
        uc = unique_completions(args.uc_targets, args.uc_targets,
                                span=min(2000, 2 * args.uc_targets))
        checks["unique_completions"] = uc["invariant"]["unique_completions"]
        checks["all"] = bool(checks["all"] and checks["unique_completions"] == 1)

    if rank != 0:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return None

    pk, src = peaks()
    dec_traffic = traffic_record("attention.cu", "attn_split_kernel<128>/decode")
    nom_hbm, nom_tf = NOMINAL["hbm_gbs"], NOMINAL["bf16_tflops"]
    kernels = {
        "bi_kv_write": {"ms": float(mean[0]), "GB/s": wl.kvw_bytes / (mean[0] * 1e-3) / 1e9},
        "bi_rmsnorm": {"ms": float(mean[1]), "GB/s": wl.norm_bytes / (mean[1] * 1e-3) / 1e9,
                       "frac_hbm": wl.norm_bytes / (mean[1] * 1e-3) / 1e9 / pk["hbm_gbs"],
                       "context": rms_ctx,
                       "frac_hbm_M65536": rms_ctx["rmsnorm_M65536_GB/s"] / pk["hbm_gbs"],
                       "frac_hbm_back_to_back": rms_ctx["back_to_back_M2048_GB/s"] / pk["hbm_gbs"],
                       "frac_hbm_graph": (rms_ctx["graph_M2048_GB/s"] / pk["hbm_gbs"]
                                          if rms_ctx["graph_M2048_GB/s"] else None)},
        "bi_matmul": {"ms": float(mean[2]), "TFLOP/s": wl.gemm_flops / (mean[2] * 1e-3) / 1e12,
                      "frac_bf16": wl.gemm_flops / (mean[2] * 1e-3) / 1e12 / pk["bf16_tflops"]},
        "bi_attention_decode": {"ms": float(mean[3]), "GB/s": wl.dec_bytes / (mean[3] * 1e-3) / 1e9,
                                "frac_hbm": wl.dec_bytes / (mean[3] * 1e-3) / 1e9 / pk["hbm_gbs"]},
        "bi_attention_prefill": {"ms": float(mean[4]),
                                 "TFLOP/s": wl.pre_flops / (mean[4] * 1e-3) / 1e12,
                                 "frac_bf16": wl.pre_flops / (mean[4] * 1e-3) / 1e12 / pk["bf16_tflops"]},
    }
    # the same fractions against NVIDIA's datasheet figures (labelled as such)
    for name, k in kernels.items():
        if "GB/s" in k and name != "bi_kv_write":
            k["frac_datasheet_hbm"] = k["GB/s"] / nom_hbm
        if "TFLOP/s" in k:
            k["frac_datasheet_bf16_dense"] = k["TFLOP/s"] / nom_tf
    # dominant kernel of the step
    dom = int(np.argmax(mean))
    if dom == 3:
        ach = wl.dec_bytes / (mean[3] * 1e-3) / 1e9
        roof = {"kernel": "bi_attention_decode", "bound": "hbm", "achieved": ach,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                "traffic": dec_traffic, "algorithmic_bytes": wl.dec_bytes,
                "peak_source": src + " (copy bandwidth)"}
    elif dom == 4:
        ach = wl.pre_flops / (mean[4] * 1e-3) / 1e12
        roof = {"kernel": "bi_attention_prefill", "bound": "tensor", "achieved": ach,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                "traffic": None, "algorithmic_flops": wl.pre_flops,
                "peak_source": src + " (cuBLAS bf16, burst)"}
    else:
        ach = wl.gemm_flops / (mean[2] * 1e-3) / 1e12
        roof = {"kernel": "bi_matmul", "bound": "tensor", "achieved": ach,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"],
                "traffic": None, "algorithmic_flops": wl.gemm_flops,
                "peak_source": src + " (cuBLAS bf16, burst)"}
    cpu = cpu_baseline(wl, budget_s=args.cpu_budget)
    line = {
        "metric": METRIC,
        "value": gemm_tf,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "hidden": H, "M": M_ROWS, "N": N_COLS,
                   "decode": {"B": DEC_B, "Hq": DEC_HQ, "Hkv": DEC_HKV, "d": D,
                              "kv_len": "U(1,32768)", "page": 16, "split": 256},
                   "prefill": {"S": PRE_S, "Hq": PRE_HQ, "Hkv": PRE_HKV, "d": D},
                   "l2": "flushed between steps (512 MB write)", "parallelism": "replicas"},
        "split_kv_attn": {"value": dec_gbs, "unit": "GB/s", "frac": dec_gbs / world / pk["hbm_gbs"],
                          "peak": pk["hbm_gbs"]},
        "bitwise_match": checks,
        "roofline": roof,
        "kernels": kernels,
        "overhead_vs_variant_off": overhead,
        "cost_of_invariance": coi,
        "unique_completions": uc,
        "e2e": {"value": world * wl.gemm_flops / (pipe_gemm_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "split_kv_attn_gbs": world * wl.dec_bytes / (pipe_dec_ms * 1e-3) / 1e9,
                "step_ms": pipe_step_ms,
                "legs_ms": {"rmsnorm_matmul": pipe_gemm_ms, "kv_write_decode": pipe_dec_ms},
                "results_equal_serial": pipe_same,
                "serial": {"step_ms": e2e_step_ms,
                           "legs_ms": {"rmsnorm_matmul": e2e_gemm_ms, "kv_write_decode": e2e_dec_ms,
                                       "kv_write_prefill": e2e_pre_ms},
                           "TFLOP/s": world * wl.gemm_flops / (e2e_gemm_ms * 1e-3) / 1e12},
                "note": "through the public calls with pinned host buffers: every step copies its "
                        "inputs in and its results out inside the timed region. value, "
                        "split_kv_attn_gbs, step_ms: copies of the next and the previous step "
                        "overlapped with the current step's compute on three streams (double-"
                        "buffered device tensors, L2 flushed each step); serial: copy in, "
                        "compute, copy out one after the other"},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
        "peaks": {"source": src, **pk, "nominal_hbm_gbs": NOMINAL["hbm_gbs"],
                  "nominal_bf16_tflops": NOMINAL["bf16_tflops"]},
        "wall_s_timed_region": wall,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return line


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The fp64 oracle, as it stands, on this host's cores: each step is a
    bounded sample of the same workload (8 rows of the matmul)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    from synth import norm_matmul

    nm = norm_matmul(seed=1, M=M_ROWS, H=H, N=N_COLS)
    x, W = nm["x"], nm["W"]
    rows_per_step = 8

    def step(i):
        r0 = (i * rows_per_step) % M_ROWS
        oracle.matmul(x[r0:r0 + rows_per_step], W)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows_per_step * N_COLS * H * args.steps
    val = flops / dt / 1e12
    sample = "%d rows of x[2048,4096] times W[12288,4096]^T per step" % rows_per_step
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": val,
        "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "hidden": H, "M": M_ROWS, "N": N_COLS},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


# ---------------------------------------------------------------- profiling cases

def run_profile_case(args):
    """Runs one kernel alone on a reduced case (inputs above L2, a few GB at
    most) for ncu captures: --profile {rmsnorm,matmul,decode,prefill}."""
    import torch

    import invariant_bi_rmsnorm_03_b200 as bi
    from synth import (decode_lengths, norm_matmul, normal_bf16, page_table, rng,
                       slot_mapping, torch_normal_bf16)

    dev = torch.device("cuda", 0)
    L = bi.load(variant=args.variant)
    T = torch
    d16 = lambda a: T.from_numpy(a.view(np.int16)).to(dev).view(T.bfloat16)  # noqa: E731
    if args.profile == "copy":
        # size-matched reference for RMSNorm: a device copy of x[2048,4096]
        xs = [d16(norm_matmul(seed=10 + i, M=M_ROWS, H=H, N=8)["x"]) for i in range(16)]
        ys = [torch.empty_like(x) for x in xs]
        fn = lambda i: ys[i % 16].copy_(xs[i % 16])  # noqa: E731
    elif args.profile in ("rmsnorm", "matmul"):
        nm = norm_matmul(seed=1, M=M_ROWS, H=H, N=N_COLS)
        x, w, W = d16(nm["x"]), d16(nm["w"]), d16(nm["W"])
        if args.profile == "rmsnorm":
            # 16 row-blocks of 2048 x 4096 rotate through 268 MB (> L2)
            xs = [d16(norm_matmul(seed=10 + i, M=M_ROWS, H=H, N=8)["x"]) for i in range(16)]
            fn = lambda i: L.bi_rmsnorm(xs[i % 16], w, 1e-6)  # noqa: E731
        else:
            fn = lambda i: L.bi_matmul(x, W)  # noqa: E731
    elif args.profile in ("rmsnorm_matmul", "rmsnorm_then_matmul", "matmul_residual",
                          "matmul_rows"):
        # fused forms against their unfused launches, M = --profile-rows rows
        # of hidden 4096 times N = --profile-cols (12288); two weight copies
        # rotate (201 MB > L2 at N = 12288)
        M, NC = args.profile_rows, args.profile_cols
        nm = norm_matmul(seed=1, M=M, H=H, N=NC)
        x, w = d16(nm["x"]), d16(nm["w"])
        Ws = [d16(nm["W"]), d16(norm_matmul(seed=11, M=1, H=H, N=NC)["W"])]
        c = T.empty((M, NC), dtype=T.bfloat16, device=dev)
        if args.profile == "rmsnorm_matmul":
            wfs = [L.bi_fold_norm_weight(W, w) for W in Ws]
            fn = lambda i: L.bi_rmsnorm_matmul(x, wfs[i % 2], 1e-6, out=c)  # noqa: E731
        elif args.profile == "rmsnorm_then_matmul":
            y = T.empty_like(x)
            fn = lambda i: L.bi_matmul(L.bi_rmsnorm(x, w, 1e-6, out=y), Ws[i % 2],  # noqa: E731
                                       out=c)
        elif args.profile == "matmul_residual":
            r = d16(normal_bf16(rng(12), (M, NC)))
            fn = lambda i: L.bi_matmul_residual(x, Ws[i % 2], r, out=c)  # noqa: E731
        else:
            fn = lambda i: L.bi_matmul(x, Ws[i % 2], out=c)  # noqa: E731
    elif args.profile in ("qkv_fused", "qkv_unfused"):
        # the attention input of one layer of the toy decoder (hidden 4096, 32 q and
        # 8 kv heads of 128), M = --profile-rows tokens: RMSNorm, QKV matmul, RoPE and
        # the cache write, in one launch or as RMSNorm + matmul + RoPE/cache write
        M, Hq, Hkv, d = args.profile_rows, 32, 8, D
        g = rng(13)
        nm = norm_matmul(seed=1, M=M, H=H, N=8)
        x, w = d16(nm["x"]), d16(nm["w"])
        Wq = d16(normal_bf16(g, ((Hq + 2 * Hkv) * d, H), std=0.02))
        npages = M // 16 + 16
        kv = bi.PagedKV(T.zeros((npages, Hkv, 16, d), dtype=T.bfloat16, device=dev),
                        T.zeros((npages, Hkv, 16, d), dtype=T.bfloat16, device=dev),
                        T.zeros((1, 1), dtype=T.int32, device=dev))
        pos = T.from_numpy(g.integers(0, 4096, size=M).astype(np.int32)).to(dev)
        slots = T.from_numpy(g.permutation(npages * 16)[:M].astype(np.int64)).to(dev)
        q = T.empty((M, Hq, d), dtype=T.bfloat16, device=dev)
        if args.profile == "qkv_fused":
            wf = L.bi_fold_norm_weight(Wq, w)
            table = L.bi_rope_table(4096, d)
            fn = lambda i: L.bi_rmsnorm_matmul_rope_kv(x, wf, 1e-6, kv, table, pos,  # noqa: E731
                                                       slots, Hq, q_out=q)
        else:
            y = T.empty_like(x)
            qkv = T.empty((M, (Hq + 2 * Hkv) * d), dtype=T.bfloat16, device=dev)
            fn = lambda i: L.bi_rope_kv_write(  # noqa: E731
                kv, L.bi_matmul(L.bi_rmsnorm(x, w, 1e-6, out=y), Wq, out=qkv), pos, slots, Hq,
                q_out=q)
    elif args.profile in ("rmsnorm_backward", "matmul_backward"):
        # the backward passes at the hidden-4096 sizes: RMSNorm of x[M, 4096];
        # the matmul C = x W^T with W [12288, 4096] (dA and dW, 2 x 2MNK flop)
        M = args.profile_rows
        g = rng(14)
        nm = norm_matmul(seed=1, M=M, H=H, N=N_COLS)
        x, w, W = d16(nm["x"]), d16(nm["w"]), d16(nm["W"])
        if args.profile == "rmsnorm_backward":
            dy = d16(normal_bf16(g, (M, H)))
            fn = lambda i: L.bi_rmsnorm_backward(x, w, dy, 1e-6)  # noqa: E731
        else:
            dc = d16(normal_bf16(g, (M, N_COLS)))
            fn = lambda i: L.bi_matmul_backward(dc, x, W)  # noqa: E731
    elif args.profile in ("attention_backward", "swiglu_backward", "rope_backward"):
        # the toy decoder's shapes: 32 query / 8 kv heads of 128 over one
        # causal prompt of --profile-seq tokens; SwiGLU 14336 and RoPE of the
        # q heads over the same tokens
        g = rng(15)
        S = args.profile_seq
        if args.profile == "attention_backward":
            Hq, Hkv = 32, 8
            q = d16(normal_bf16(g, (S, Hq, D)))
            k = d16(normal_bf16(g, (S, Hkv, D)))
            v = d16(normal_bf16(g, (S, Hkv, D)))
            dout = d16(normal_bf16(g, (S, Hq, D)))
            pbt, pnp = page_table(g, [S])
            kv = bi.PagedKV(T.zeros((pnp, Hkv, 16, D), dtype=T.bfloat16, device=dev),
                            T.zeros((pnp, Hkv, 16, D), dtype=T.bfloat16, device=dev),
                            T.from_numpy(pbt).to(dev))
            L.bi_kv_write(kv, k, v, T.from_numpy(slot_mapping(pbt, 0, np.arange(S))).to(dev))
            cu = T.tensor([0, S], dtype=T.int32, device=dev)
            ctx = T.tensor([0], dtype=T.int32, device=dev)
            o, lse = L.bi_attention_prefill(kv, q, cu, ctx, S, want_lse=True)
            dk, dv = T.zeros_like(kv.k_cache), T.zeros_like(kv.v_cache)
            fn = lambda i: L.bi_attention_backward(kv, q, o, dout, lse, cu, ctx, S, S,  # noqa: E731
                                                   dk=dk, dv=dv)
        elif args.profile == "swiglu_backward":
            gu = d16(normal_bf16(g, (S, 2 * 14336)))
            dout = d16(normal_bf16(g, (S, 14336)))
            out = T.empty_like(gu)
            fn = lambda i: L.bi_swiglu_backward(gu, dout, out=out)  # noqa: E731
        else:
            dy = d16(normal_bf16(g, (S, 32, D)))
            pos = T.from_numpy(np.arange(S, dtype=np.int32)).to(dev)
            out = T.empty_like(dy)
            fn = lambda i: L.bi_rope_backward(dy, pos, out=out)  # noqa: E731
    elif args.profile == "sample":
        # 256 rows of lm_head logits (vocab 32000), temperature 0.8, nucleus 0.95
        g = rng(5)
        lg = T.from_numpy((g.standard_normal((256, 32000)) * 2.0).astype(np.float32)).to(dev)
        seeds = T.from_numpy(g.integers(0, 2 ** 62, size=256)).to(dev)
        offs = T.from_numpy(g.integers(0, 2 ** 20, size=256)).to(dev)
        fn = lambda i: L.bi_sample(lg, 0.8, 0.95, seeds, offs)  # noqa: E731
    elif args.profile == "decode":
        B = args.profile_batch
        g = rng(2)
        lens = decode_lengths(2, B, DEC_MAXLEN)
        bt, num_pages = page_table(g, lens, max_pages=DEC_MAXLEN // 16)
        shape = (num_pages, DEC_HKV, 16, D)
        kv = bi.PagedKV(torch_normal_bf16(shape, 1000, dev), torch_normal_bf16(shape, 2000, dev),
                        T.from_numpy(bt).to(dev))
        q = d16(normal_bf16(g, (B, DEC_HQ, D)))
        sl = T.from_numpy(lens).to(dev)
        fn = lambda i: L.bi_attention_decode(kv, q, sl, DEC_MAXLEN)  # noqa: E731
    else:
        gp = rng(3)
        S = args.profile_seq
        q = d16(normal_bf16(gp, (S, PRE_HQ, D)))
        k = d16(normal_bf16(gp, (S, PRE_HKV, D)))
        v = d16(normal_bf16(gp, (S, PRE_HKV, D)))
        pbt, pnp = page_table(gp, [S])
        kv = bi.PagedKV(T.zeros((pnp, PRE_HKV, 16, D), dtype=T.bfloat16, device=dev),
                        T.zeros((pnp, PRE_HKV, 16, D), dtype=T.bfloat16, device=dev),
                        T.from_numpy(pbt).to(dev))
        L.bi_kv_write(kv, k, v, T.from_numpy(slot_mapping(pbt, 0, np.arange(S))).to(dev))
        cu = T.tensor([0, S], dtype=T.int32, device=dev)
        ctx = T.tensor([0], dtype=T.int32, device=dev)
        fn = lambda i: L.bi_attention_prefill(kv, q, cu, ctx, S)  # noqa: E731
    for i in range(args.warmup):
        fn(i)
    torch.cuda.synchronize()
    ev = [T.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    # launches back to back: ~1 ms of GPU spin per 10 of them queued first
    T.cuda._sleep(HOST_AHEAD_CYCLES * max(1, (args.steps + 9) // 10))
    for i in range(args.steps):
        ev[i].record()
        fn(i)
    ev[-1].record()
    torch.cuda.synchronize()
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    print(json.dumps({"profile": args.profile, "ms": ms, "status": int(L.bi_device_status())}))


def run_unique_completions(args):
    print(json.dumps(unique_completions(args.targets, args.others, args.max_batch,
                                        args.token_budget, args.span, args.temperature,
                                        args.top_p, args.moe, args.fused)), flush=True)


def unique_completions(targets, others, max_batch=256, token_budget=2048, span=2000,
                       temperature=0.0, top_p=1.0, moe=False, fused=False) -> dict:
    """One fixed 64-token prompt completed greedily (256 tokens) many times
    amid random other requests, on the 8-layer hidden-4096 random-init
    decoder: the number of distinct completions for the invariant and the
    variant-off build, and where the completions first differ from the
    prompt's completion when it runs alone."""
    import torch

    import invariant_bi_rmsnorm_03_b200 as bi
    from invariant_bi_rmsnorm_03_b200.decoder import (DecoderConfig, PagePool, Request, Scheduler,
                                                      ToyDecoder, run, weight_shapes)
    from synth import toy_decoder_weights, unique_completion_workload

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    # dense: SwiGLU 14336; mixture of experts: 16 experts of SwiGLU 1408, top 4
    cfg = DecoderConfig(n_experts=16, top_k=4, expert_ffn=1408) if moe else DecoderConfig(fused=fused)
    weights = toy_decoder_weights(weight_shapes(cfg), seed=4, device=dev)
    prompt, spec = unique_completion_workload(seed=4, n_target=targets, n_other=others,
                                              vocab=cfg.vocab, steps_span=span)
    pages_per_req = (512 + 256 + 15) // 16
    num_pages = max_batch * pages_per_req + 64
    ffn = ("mixture of 16 experts (SwiGLU 1408, top 4)" if moe else "SwiGLU 14336")
    result = {"experiment": "unique completions", "model": "8-layer decoder, hidden 4096, GQA 32/8, "
              "d 128, %s, vocab 32000, W~N(0,0.02) seed 4" % ffn,
              "prompt_tokens": 64, "new_tokens": 256, "targets": targets,
              "others": others, "max_batch": max_batch,
              "token_budget": token_budget, "data": "synthetic",
              "fused": ("RMSNorm folded into the next matmul, RoPE and the cache write in "
                        "the QKV matmul's epilogue, residual adds in the matmul epilogue"
                        if cfg.fused else False),
              "sampling": ("greedy" if temperature <= 0 else
                           {"temperature": temperature, "top_p": top_p,
                            "seed": "one per request; every target copy the same"})}
    for variant in (False, True):
        L = bi.load(variant=variant)
        model = ToyDecoder(L, cfg, weights, num_pages, dev)
        tseed = next(d["seed"] for d in spec if d["tag"] == "target")
        solo = Request(-1, prompt, 256, temperature=temperature, top_p=top_p, seed=tseed)
        s1 = Scheduler(PagePool(num_pages, seed=1), max_batch=1, token_budget=token_budget)
        s1.add([solo])
        run(s1, model)
        reqs = [Request(d["rid"], d["prompt"], d["max_new"], d["arrival"], d["tag"],
                        temperature=temperature, top_p=top_p, seed=d["seed"]) for d in spec]
        sched = Scheduler(PagePool(num_pages, seed=2), max_batch=max_batch,
                          token_budget=token_budget)
        sched.add(reqs)
        sizes = []
        orig_plan = sched.plan

        def plan_and_count():
            p = orig_plan()
            if p is not None:
                sizes.append(len(p.dec) + len(p.pre))
            return p

        sched.plan = plan_and_count
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        steps = run(sched, model)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        outs = [tuple(r.out) for r in reqs if r.tag == "target"]
        ref = tuple(solo.out)
        first_div = [next((i for i, (a, b) in enumerate(zip(o, ref)) if a != b), None) for o in outs]
        div = [f for f in first_div if f is not None]
        tokens = sum(len(r.prompt) + r.max_new for r in reqs)
        result["variant_off" if variant else "invariant"] = {
            "unique_completions": len(set(outs)),
            "equal_to_solo_run": sum(o == ref for o in outs),
            "first_divergent_token": {"min": min(div), "median": float(np.median(div))} if div else None,
            "steps": steps, "batch_rows_min": int(min(sizes)), "batch_rows_max": int(max(sizes)),
            "wall_s": wall, "tokens_per_s": tokens / wall,
            "device_status": int(L.bi_device_status())}
        del model
        torch.cuda.empty_cache()
    del weights
    torch.cuda.empty_cache()
    return result


def main(argv=None):
    import faulthandler

    faulthandler.enable()  # a host-side crash prints every thread's stack
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--profile", choices=["rmsnorm", "matmul", "decode", "prefill", "copy",
                                          "sample", "rmsnorm_matmul", "rmsnorm_then_matmul",
                                          "matmul_residual", "matmul_rows", "qkv_fused",
                                          "qkv_unfused", "rmsnorm_backward", "matmul_backward",
                                          "attention_backward", "swiglu_backward",
                                          "rope_backward"],
                    help="run one kernel alone on a reduced case (for ncu)")
    ap.add_argument("--profile-batch", type=int, default=32)
    ap.add_argument("--profile-seq", type=int, default=4096)
    ap.add_argument("--profile-rows", type=int, default=M_ROWS,
                    help="rows of the fused-matmul --profile cases")
    ap.add_argument("--profile-cols", type=int, default=N_COLS,
                    help="output columns of the fused-matmul --profile cases")
    ap.add_argument("--variant", action="store_true", help="--profile the variant-off build")
    ap.add_argument("--unique-completions", action="store_true",
                    help="run the toy-decoder unique-completion experiment instead")
    ap.add_argument("--targets", type=int, default=1000)
    ap.add_argument("--others", type=int, default=1000)
    ap.add_argument("--max-batch", type=int, default=256)
    ap.add_argument("--token-budget", type=int, default=2048)
    ap.add_argument("--span", type=int, default=2000, help="arrival steps are spread over this")
    ap.add_argument("--temperature", type=float, default=0.0,
                    help="unique-completion run: 0 = greedy, else sampling at this temperature")
    ap.add_argument("--top-p", type=float, default=1.0)
    ap.add_argument("--moe", action="store_true",
                    help="unique-completion run on the mixture-of-experts decoder")
    ap.add_argument("--fused", action="store_true",
                    help="unique-completion run with the fused matmul forms")
    ap.add_argument("--uc-targets", type=int, default=1000,
                    help="target copies (and as many others) of the in-bench unique-completion "
                         "check; 0 skips it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile:
        run_profile_case(args)
    elif args.unique_completions:
        run_unique_completions(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
