"""Benchmark of the Orthrus dual-view decode step's hot path on B200.

One step = one full decode step of the hot path on Qwen3-8B-shaped synthetic
data (36 layers, 32 query / 8 KV heads, head_dim 128, hidden 4096, vocab
151936), batch 1, block K = 32, context 40960:
    diffusion pass: 36 x block attention (diffusion mask) + LM head argmax -> drafts
    AR pass:        36 x block attention (AR mask)        + LM head argmax
    consensus:      verify + KV commit (one launch)
Metric: verified draft tokens per second = B*K / step time.  The step is
captured once into a CUDA graph of K unrolled steps with event nodes at the
phase boundaries, so the attention launches' average duration is measured on
the launching stream inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]
                    [--ctx L] [--block K] [--layers N] [--no-extras]

On one GPU the line also carries, unless --no-extras: the ragged-batch step (8
sequences, lengths U[1024, 32768], K 32, planted accept lengths U{0..32}; its
LM head has R = 256 rows, timed in the step and alone) and the verify-step
sweep over K in {1,4,8,16,32} x context in {1024, 8192, 40960, 131072} (K = 1
is plain decoding).

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (the reference arm of this benchmark).  Under torchrun (N > 1) every
rank runs an independent replica (weak scaling: the path has no exchange
step); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "verified draft tokens/sec per step at 40K ctx; attn HBM GB/s vs peak"
UNIT = "tokens/s"
QWEN = dict(Hq=32, Hkv=8, d=128, H=4096, V=151936, layers=36)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ctx", type=int, default=40960)
    ap.add_argument("--block", type=int, default=32)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--layers", type=int, default=QWEN["layers"])
    ap.add_argument("--accept", type=int, default=4,
                    help="planted accepted length per step (drafts agree with the AR "
                         "argmax on this many leading rows)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the ragged-batch step and the K x context sweep that a "
                         "single-GPU run reports beside the headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--json-out", default=None)
    return ap.parse_args(argv)


# ----------------------------------------------------------------- plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


ATTN_SOURCES = ("lossless_block_drafting_b200/csrc/block_attn.cu",
                "lossless_block_drafting_b200/csrc/common.cuh",
                "lossless_block_drafting_b200/csrc/ptx.cuh")


def attn_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(wl):
    """DRAM bytes (read + write) per attention launch from the committed ncu
    capture, scaled to this workload's KV bytes; None once the kernel's sources
    differ from the ones the counters were taken on, or for another workload."""
    path = os.path.join(ROOT, "profiles", "block_attn_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != attn_source_hash():
        return None
    if (rec.get("ctx"), rec.get("block_K"), rec.get("batch")) != (wl.L0, wl.K, wl.B):
        return None
    return int(rec["dram_bytes_read"] + rec["dram_bytes_write"])


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (identity without a process group).

    Timings are reduced this way so the slowest replica sets the step time.
    """
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sync_ranks():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def weak_scaling_value(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job verified tokens/s: every replica verifies tokens_per_rank per step."""
    return world * tokens_per_rank / (max_ms * 1e-3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(
            p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        """Host time stamp; samples between two marks form the timed window."""
        return time.time()

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        window = [(ts, ln) for ts, ln in self.lines
                  if (t0 is None or ts >= t0) and (t1 is None or ts <= t1 + 0.05)]
        if not window:  # window shorter than the sampling period: nearest samples
            window = self.lines[-3:]
        for _, ln in window:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                smax.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- workload
class Workload:
    """Resident synthetic inputs for one replica of the decode step.

    lens: committed context length per sequence (an int gives every sequence
    the same); accepts: planted accept length per sequence (the diffusion view's
    final hidden states equal the AR view's on that many leading rows of the
    block, so the drafts match the AR argmax there and nowhere else).  kv:
    optional (k, v) lists of per-layer caches to share with another workload.
    """

    def __init__(self, B, K, lens, layers, accepts, steps_total, device, seed=0, kv=None,
                 with_append=False):
        import torch
        from lossless_block_drafting_b200 import orthrus as ob
        self.ob = ob
        lens = [int(lens)] * B if isinstance(lens, int) else [int(x) for x in lens]
        accepts = [int(accepts)] * B if isinstance(accepts, int) else [int(x) for x in accepts]
        self.B, self.K, self.lens, self.layers = B, K, lens, layers
        self.L0 = lens[0]
        Hq, Hkv, d, H, V = QWEN["Hq"], QWEN["Hkv"], QWEN["d"], QWEN["H"], QWEN["V"]
        self.Hq, self.Hkv, self.d, self.H, self.V = Hq, Hkv, d, H, V
        g = torch.Generator(device=device).manual_seed(seed)
        bf = torch.bfloat16

        def randn(*shape, std=1.0):
            x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
            return (x * std).to(bf) if std != 1.0 else x.to(bf)

        if kv is None:
            # room for the committed length to grow by up to K per step
            cap = max(lens) + K * (steps_total + 2)
            self.k = [randn(B, Hkv, cap, d) for _ in range(layers)]
            self.v = [randn(B, Hkv, cap, d) for _ in range(layers)]
        else:
            self.k, self.v = kv
        self.cap = self.k[0].shape[2]
        # A step's inputs (both views' queries for every layer, both views' final
        # hidden states) live in one flat buffer, so one host->device copy
        # delivers them all in the end-to-end measurement.
        n_q, n_h = B * K * Hq * d, B * K * H
        self.inputs = torch.empty(2 * layers * n_q + 2 * n_h, dtype=bf, device=device)
        off = [0]

        def place(x):
            v = self.inputs[off[0]:off[0] + x.numel()].view(x.shape)
            v.copy_(x)
            off[0] += x.numel()
            return v

        self.q_diff = [place(randn(B, K, Hq, d)) for _ in range(layers)]
        self.q_ar = [place(randn(B, K, Hq, d)) for _ in range(layers)]
        self.W = randn(V, H, std=0.02)
        self.h_ar = place(randn(B * K, H))
        self.h_diff = place(randn(B * K, H))
        hv, ha = self.h_diff.view(B, K, H), self.h_ar.view(B, K, H)
        self.accepts = [max(0, min(a, K)) for a in accepts]
        for b_, a in enumerate(self.accepts):
            hv[b_, :a] = ha[b_, :a]
        self.accept = self.accepts[0]
        self.ctx_lens = torch.tensor(lens, dtype=torch.int32, device=device)
        self.ctx_init = self.ctx_lens.clone()
        self.attn_out = torch.empty(B, K, Hq, d, dtype=bf, device=device)
        self.ws_attn = torch.zeros(ob.block_attn_workspace_size(B, Hq, Hkv, d, K),
                                   dtype=torch.uint8, device=device)
        self.ws_lm = torch.empty(ob.lmhead_workspace_size(B * K, V), dtype=torch.uint8,
                                 device=device)
        self.draft = torch.empty(B * K, dtype=torch.int32, device=device)
        self.argmax = torch.empty(B * K, dtype=torch.int32, device=device)
        self.accept_len = torch.empty(B, dtype=torch.int32, device=device)
        self.next_tok = torch.empty(B, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.views = [ob.kv_cache_view(self.k[i], self.v[i], self.ctx_lens) for i in range(layers)]
        # With the block Q/K/V append in the step, every layer call first turns
        # that view's packed projections into rotated queries (written over
        # q_diff / q_ar) and the block's K/V in cache slots [L_b, L_b + K).
        self.with_append = with_append
        if with_append:
            W = Hq + 2 * Hkv
            self.qkv_diff = [randn(B * K, W * d) for _ in range(layers)]
            self.qkv_ar = [randn(B * K, W * d) for _ in range(layers)]
            self.qk_w = (1.0 + 0.1 * torch.randn(2, d, generator=g, device=device)).to(bf)

    # kernels launched per step (one per attention call; main + reduce per LM
    # head; one verify+commit)
    @property
    def launches_per_step(self):
        return (4 if self.with_append else 2) * self.layers + 2 * 2 + 1

    def emitted_per_step(self):
        """Tokens a step emits: the accepted drafts plus the correction (or the
        last draft when all K are accepted), per sequence."""
        return sum(min(a + 1, self.K) for a in self.accepts)

    def attn_bytes(self):
        """Algorithmic bytes of one attention call at the starting contexts:
        K and V of every key each (sequence, KV head) reads, plus Q and O."""
        kv = 2 * self.Hkv * self.d * 2 * sum(L + self.K for L in self.lens)
        qo = 2 * self.B * self.K * self.Hq * self.d * 2
        return kv + qo

    def lm_bytes(self):
        return self.V * self.H * 2 + self.B * self.K * self.H * 2

    def lm_flops(self):
        return 2.0 * self.B * self.K * self.H * self.V

    def append(self, qkv, q_out, i, stream):
        self.ob.block_qkv_append(qkv, None, None, None, self.Hq, self.K, q_norm_w=self.qk_w[0],
                                 k_norm_w=self.qk_w[1], q_out=q_out, cache_view=self.views[i],
                                 dev_status=self.status, stream=stream)

    def step(self, stream, events=None, verify_only=False):
        """Issue one decode step on `stream`; events (if given) mark phase
        boundaries.  verify_only: the AR pass, LM head and verify + commit only."""
        ob = self.ob
        ev = events or {}
        if "t0" in ev:
            ev["t0"].record(stream)
        if not verify_only:
            for i in range(self.layers):
                if self.with_append:
                    self.append(self.qkv_diff[i], self.q_diff[i], i, stream)
                ob.block_attn(self.q_diff[i], None, None, None, ob.MASK_DIFF, out=self.attn_out,
                              workspace=self.ws_attn, dev_status=self.status, stream=stream,
                              cache_view=self.views[i])
        if "t1" in ev:
            ev["t1"].record(stream)
        if not verify_only:
            ob.lmhead_argmax(self.h_diff, self.W, argmax=self.draft, workspace=self.ws_lm,
                             stream=stream, dev_status=self.status)
        if "t2" in ev:
            ev["t2"].record(stream)
        for i in range(self.layers):
            if self.with_append:
                self.append(self.qkv_ar[i], self.q_ar[i], i, stream)
            ob.block_attn(self.q_ar[i], None, None, None, ob.MASK_AR, out=self.attn_out,
                          workspace=self.ws_attn, dev_status=self.status, stream=stream,
                          cache_view=self.views[i])
        if "t3" in ev:
            ev["t3"].record(stream)
        ob.lmhead_argmax(self.h_ar, self.W, argmax=self.argmax, workspace=self.ws_lm,
                         stream=stream, dev_status=self.status)
        if "t4" in ev:
            ev["t4"].record(stream)
        ob.verify_commit(self.argmax.view(self.B, self.K), self.draft.view(self.B, self.K),
                         self.ctx_lens, self.cap, accept_len=self.accept_len,
                         next_tok=self.next_tok, dev_status=self.status, stream=stream)
        if "t5" in ev:
            ev["t5"].record(stream)


def capture(wl: Workload, n_steps: int, stream, with_events: bool, verify_only=False):
    """CUDA graph of n_steps unrolled steps (+ external timing events per phase)."""
    import torch
    evs = []
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(n_steps):
            e = None
            if with_events:
                e = {k: torch.cuda.Event(enable_timing=True, external=True)
                     for k in ("t0", "t1", "t2", "t3", "t4", "t5")}
                evs.append(e)
            wl.step(stream, e, verify_only=verify_only)
    return g, evs


def run_ours(args):
    import torch
    import torch.distributed as dist

    from lossless_block_drafting_b200 import build as libbuild
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=300))
    libbuild.build()
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sus, peak_kind = peaks()
    K_steps, W_steps = args.steps, args.warmup
    wl = Workload(args.batch, args.block, args.ctx, args.layers, args.accept,
                  K_steps + W_steps + 4, dev, seed=1234 + rank)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        # eager warm-up (also loads the library and sets kernel attributes)
        for _ in range(2):
            wl.step(stream)
        stream.synchronize()
        g_warm, _ = capture(wl, 1, stream, with_events=False)
        g_timed, evs = capture(wl, K_steps, stream, with_events=True)
    wl.ctx_lens.copy_(wl.ctx_init)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(W_steps):
            g_warm.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index)
    if rank == 0:
        sampler.start()
    sync_ranks()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t_win0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        g_timed.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t_win1 = time.time()
    sync_ranks()
    clocks = sampler.stop(t_win0, t_win1) if rank == 0 else None
    ms_total = max_over_ranks(start.elapsed_time(end), dev)
    ms_step = ms_total / K_steps

    # per-phase times from the event nodes of every timed step
    ph = {"diff_attn": 0.0, "diff_lm": 0.0, "ar_attn": 0.0, "ar_lm": 0.0, "verify": 0.0}
    for e in evs:
        ph["diff_attn"] += e["t0"].elapsed_time(e["t1"])
        ph["diff_lm"] += e["t1"].elapsed_time(e["t2"])
        ph["ar_attn"] += e["t2"].elapsed_time(e["t3"])
        ph["ar_lm"] += e["t3"].elapsed_time(e["t4"])
        ph["verify"] += e["t4"].elapsed_time(e["t5"])
    ph = {k: v / K_steps for k, v in ph.items()}
    attn_us = (ph["diff_attn"] + ph["ar_attn"]) * 1e3 / (2 * wl.layers)
    lm_us = (ph["diff_lm"] + ph["ar_lm"]) * 1e3 / 2
    status = int(wl.status.item())

    tokens = wl.B * wl.K
    value = weak_scaling_value(tokens, world, ms_step)
    attn_gbs = wl.attn_bytes() / (attn_us * 1e-6) / 1e9
    lm_gbs = wl.lm_bytes() / (lm_us * 1e-6) / 1e9
    lm_tflops = 2.0 * wl.B * wl.K * wl.H * wl.V / (lm_us * 1e-6) / 1e12
    verify_pass_ms = ph["ar_attn"] + ph["ar_lm"] + ph["verify"]

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, g_warm, stream, K_steps, W_steps, world, dev)
    try:  # an auxiliary measurement: its failure is reported, not fatal to the step's line
        qkv_append = time_qkv_append(wl, stream)
    except Exception as exc:  # noqa: BLE001
        qkv_append = {"error": f"{type(exc).__name__}: {exc}"}

    del g_timed, g_warm
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": round(ms_step, 4),
        "value_counts": "verified draft positions: B*K per step, every block position scored "
                        "by the AR pass and compared with its draft",
        "emitted_tokens_per_s": round(weak_scaling_value(wl.emitted_per_step(), world, ms_step),
                                      2),
        "emitted_per_step": wl.emitted_per_step(),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/KV/hidden, N(0,0.02) LM head; "
                "Qwen3-8B shapes, random weights)",
        "config": {
            "workload": f"qwen3-8b-shaped dual-view decode step: {wl.layers} layers, "
                        f"batch {wl.B}, K {wl.K}, context {wl.L0}",
            "step": "diffusion pass (36x block_attn DIFF + lmhead_argmax) + AR pass "
                    "(36x block_attn AR + lmhead_argmax) + verify_commit",
            "batch": wl.B, "block_K": wl.K, "ctx": wl.L0, "layers": wl.layers,
            "heads": "32q/8kv d128", "hidden": wl.H, "vocab": wl.V,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (per step: "
                  f"{(2 * wl.layers * wl.attn_bytes() + 2 * wl.lm_bytes()) / 1e9:.1f} GB read)",
            "graph": "K steps unrolled in one CUDA graph",
            "planted_accept_len": wl.accept,
        },
        "breakdown_ms_per_step": {k: round(v, 4) for k, v in ph.items()},
        "verify_pass_only": {
            "ms": round(verify_pass_ms, 4),
            "tokens_per_s": round(weak_scaling_value(tokens, world, verify_pass_ms), 2),
        },
        "attn": {"us_per_call": round(attn_us, 2), "GB_per_s": round(attn_gbs, 1),
                 "frac_of_hbm_peak": round(attn_gbs / hbm_peak, 4)},
        "lmhead": {"us_per_call": round(lm_us, 2), "GB_per_s": round(lm_gbs, 1),
                   "TFLOP_per_s": round(lm_tflops, 1),
                   "frac_of_hbm_peak": round(lm_gbs / hbm_peak, 4),
                   "frac_of_bf16_peak": round(lm_tflops / tc_sus, 4),
                   "frac_of_bf16_peak_burst": round(lm_tflops / tc_peak, 4)},
        "roofline": {
            "kernel": "orthrus_block_attn (persistent split-KV kernel with in-kernel LSE merge), "
                      "AR and DIFF masks",
            "bound": "hbm",
            "achieved": round(attn_gbs, 1),
            "peak": hbm_peak,
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"
                           if peak_kind == "measured" else "fallback 6650 GB/s",
            "unit": "GB/s",
            "frac": round(attn_gbs / hbm_peak, 4),
            "traffic": measured_traffic(wl),
            "algorithmic_bytes_per_launch": wl.attn_bytes(),
        },
        "qkv_append": qkv_append,
        "gpu_launches": wl.launches_per_step * K_steps,
        "device_status": status,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl.L0, wl.K, wl.layers)
    if world == 1 and not args.no_extras:
        del wl
        torch.cuda.empty_cache()
        result["step_with_append"] = run_step_with_append(dev, stream, args.ctx, args.block,
                                                          args.layers, args.accept)
        result["ragged_batch"] = run_ragged(dev, stream, hbm_peak, tc_peak, tc_sus)
        result["sweep"] = run_sweep(dev, stream, hbm_peak)
        try:  # a separate kernel; its failure is reported, not fatal to the step's line
            result["prefill"] = run_prefill(dev, stream, tc_peak)
        except Exception as exc:  # noqa: BLE001
            result["prefill"] = {"error": f"{type(exc).__name__}: {exc}"}
    if world > 1:
        sync_ranks()
        dist.destroy_process_group()
    return result if rank == 0 else None


def time_qkv_append(wl: "Workload", stream, launches: int = 100):
    """The block Q/K/V append (per-head RMS norm, rotary embedding, block K/V into
    the cache) for one layer at this workload's shapes: device time per launch
    from a CUDA graph of back-to-back launches.  Reported beside the step, not
    inside it (the step is the path from the block's queries onwards)."""
    import torch
    from lossless_block_drafting_b200 import orthrus as ob
    Hq, Hkv, d = QWEN["Hq"], QWEN["Hkv"], QWEN["d"]
    g = torch.Generator(device=wl.k[0].device).manual_seed(99)
    qkv = torch.randn(wl.B * wl.K, (Hq + 2 * Hkv) * d, generator=g, device=wl.k[0].device,
                      dtype=torch.float32).to(torch.bfloat16)
    w = (1 + 0.1 * torch.randn(2, d, generator=g, device=wl.k[0].device)).to(torch.bfloat16)
    ctx = wl.ctx_init.clone()
    view = ob.kv_cache_view(wl.k[0], wl.v[0], ctx)
    q_out = torch.empty(wl.B, wl.K, Hq, d, dtype=torch.bfloat16, device=qkv.device)

    def one():
        ob.block_qkv_append(qkv, None, None, None, Hq, wl.K, q_norm_w=w[0], k_norm_w=w[1],
                            q_out=q_out, cache_view=view, stream=stream, dev_status=wl.status)

    with torch.cuda.stream(stream):
        for _ in range(3):
            one()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(launches):
                one()
        graph.replay()
        stream.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / launches
    nbytes = 2 * (2 * wl.B * wl.K * (Hq + 2 * Hkv) * d + 2 * d)  # read qkv + weights, write q/k/v
    del graph
    return {"us_per_call": round(us, 2), "bytes_per_call": nbytes,
            "GB_per_s": round(nbytes / (us * 1e-6) / 1e9, 1),
            "bound": "launch latency (0.8 MB per call)", "in_step": False}


def run_e2e(wl: Workload, g_step, stream, K_steps, W_steps, world, dev):
    """Same metric end to end: per step, H2D of the step's inputs from pinned host
    memory, the captured step (public C-ABI calls), and a D2H read of the results."""
    import torch
    # every input of the step (queries of both views for all layers, both views'
    # hidden states) in one pinned buffer -> one copy into the flat device buffer
    host_in = [(wl.inputs.cpu().pin_memory(), wl.inputs)]
    outs = [wl.accept_len, wl.next_tok, wl.ctx_lens]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(h.numel() * h.element_size() for h, _ in host_in)
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def one():
        with torch.cuda.stream(stream):
            for h, d in host_in:
                d.copy_(h, non_blocking=True)
            g_step.replay()
            for h, d in zip(host_out, outs):
                h.copy_(d, non_blocking=True)
        stream.synchronize()

    wl.ctx_lens.copy_(wl.ctx_init)
    for _ in range(W_steps):
        one()
    torch.cuda.synchronize()
    sync_ranks()
    t0 = time.perf_counter()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(K_steps):
        one()
    end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end) / K_steps, dev)
    wall_ms = (time.perf_counter() - t0) * 1e3 / K_steps
    return {"value": round(weak_scaling_value(wl.B * wl.K, world, ms), 2), "unit": UNIT,
            "ms_per_step": round(ms, 4), "host_wall_ms_per_step": round(wall_ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "how": "per step: one pinned host->device copy of every input of the step (both "
                   "views' queries for all 72 layer calls and both views' final hidden states), "
                   "a replay of the CUDA graph in which the step's C-ABI calls were recorded "
                   "once, and a device->host read of accept lengths, next tokens and lengths; "
                   "each step synchronised"}


def time_graph_steps(wl: Workload, stream, n_steps: int, verify_only=False, replays=3):
    """Per-phase device times (ms, averaged over steps) of n_steps unrolled steps
    in one CUDA graph, after an eager step and a warm replay; the committed
    lengths are reset before every replay."""
    import torch
    with torch.cuda.stream(stream):
        wl.step(stream, verify_only=verify_only)
        stream.synchronize()
        g, evs = capture(wl, n_steps, stream, with_events=True, verify_only=verify_only)
    ph = None
    for _ in range(replays):
        with torch.cuda.stream(stream):
            wl.ctx_lens.copy_(wl.ctx_init)
            g.replay()
        torch.cuda.synchronize()
        cur = {"diff_attn": 0.0, "diff_lm": 0.0, "ar_attn": 0.0, "ar_lm": 0.0, "verify": 0.0,
               "step": 0.0}
        for e in evs:
            cur["diff_attn"] += e["t0"].elapsed_time(e["t1"])
            cur["diff_lm"] += e["t1"].elapsed_time(e["t2"])
            cur["ar_attn"] += e["t2"].elapsed_time(e["t3"])
            cur["ar_lm"] += e["t3"].elapsed_time(e["t4"])
            cur["verify"] += e["t4"].elapsed_time(e["t5"])
            cur["step"] += e["t0"].elapsed_time(e["t5"])
        cur = {k: v / len(evs) for k, v in cur.items()}
        ph = cur  # the last replay is reported (the earlier ones are warm-up)
    del g, evs
    return ph


def run_ragged(dev, stream, hbm_peak, tc_peak, tc_sus, n_steps=8):
    """The ragged-batch configuration: 8 sequences with committed lengths uniform
    in [1024, 32768], K = 32, per-sequence planted accept lengths uniform in
    0..32, the full dual-view step over 36 layers (the LM head then has
    R = 256 rows); the commit advances each sequence by min(accept + 1, 32)."""
    import torch
    from lossless_block_drafting_b200 import synth
    B, K = 8, 32
    lens = [int(x) for x in synth.ctx_lens_uniform(B, 1024, 32768, seed=4)]
    accepts = [int(x) for x in synth.accept_uniform(B, K, seed=5)]
    wl = Workload(B, K, lens, QWEN["layers"], accepts, n_steps + 4, dev, seed=77)
    ph = time_graph_steps(wl, stream, n_steps)
    got_accept = wl.accept_len.cpu().tolist()
    attn_us = (ph["diff_attn"] + ph["ar_attn"]) * 1e3 / (2 * wl.layers)
    lm_us = (ph["diff_lm"] + ph["ar_lm"]) * 1e3 / 2
    attn_gbs = wl.attn_bytes() / (attn_us * 1e-6) / 1e9
    lm_tf = wl.lm_flops() / (lm_us * 1e-6) / 1e12
    out = {
        "config": "8 sequences, committed lengths U[1024, 32768] (seed 4), K 32, 36 layers, "
                  "32q/8kv d128, vocab 151936; planted accept lengths U{0..32} (seed 5)",
        "ctx_lens": lens, "accept_planted": accepts, "accept_device": got_accept,
        "ms_per_step": round(ph["step"], 4),
        "verified_tokens_per_s": round(B * K / (ph["step"] * 1e-3), 1),
        "emitted_tokens_per_s": round(wl.emitted_per_step() / (ph["step"] * 1e-3), 1),
        "breakdown_ms_per_step": {k: round(v, 4) for k, v in ph.items() if k != "step"},
        "attn": {"us_per_call": round(attn_us, 2), "GB_per_s": round(attn_gbs, 1),
                 "frac_of_hbm_peak": round(attn_gbs / hbm_peak, 4)},
        "lmhead_r256": {"us_per_call": round(lm_us, 2), "TFLOP_per_s": round(lm_tf, 1),
                        "frac_of_bf16_peak_burst": round(lm_tf / tc_peak, 4),
                        "frac_of_bf16_peak_sustained": round(lm_tf / tc_sus, 4),
                        "GB_per_s": round(wl.lm_bytes() / (lm_us * 1e-6) / 1e9, 1)},
        "device_status": int(wl.status.item()),
    }
    out["lmhead_r256_alone"] = time_lmhead_alone(wl, stream, tc_peak)
    del wl
    torch.cuda.empty_cache()
    return out


def time_lmhead_alone(wl, stream, tc_peak, launches=10):
    """The step's AR-pass LM head (same h, W and workspace) timed alone: a CUDA
    graph of back-to-back launches, timed after one warm replay.  W (1.2 GB) is
    larger than L2, so every launch streams it from HBM; a kernel timed alone
    takes the burst bf16 peak."""
    import torch
    from lossless_block_drafting_b200 import orthrus as ob
    with torch.cuda.stream(stream):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for _ in range(launches):
                ob.lmhead_argmax(wl.h_ar, wl.W, argmax=wl.argmax, workspace=wl.ws_lm,
                                 stream=stream, dev_status=wl.status)
        gr.replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        gr.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / launches
    tf = wl.lm_flops() / (us * 1e-6) / 1e12
    del gr
    return {"us_per_call": round(us, 2), "TFLOP_per_s": round(tf, 1),
            "frac_of_bf16_peak_burst": round(tf / tc_peak, 4), "launches": launches,
            "device_status": int(wl.status.item())}


def run_step_with_append(dev, stream, L, K, layers, accept, n_steps=8):
    """The headline step with the block Q/K/V append (per-head RMS norm of q and
    k, rotary embedding at L_b + i, block K/V into the cache) before each of its
    72 attention calls, against the same workload's step without it (both from
    the same graph timing): the append's cost inside the step."""
    import torch
    wl = Workload(1, K, L, layers, accept, n_steps + 4, dev, seed=1234, with_append=True)
    with_app = time_graph_steps(wl, stream, n_steps)
    wl.with_append = False
    without = time_graph_steps(wl, stream, n_steps)
    wl.with_append = True
    out = {"ms_per_step": round(with_app["step"], 4),
           "ms_per_step_without_append": round(without["step"], 4),
           "verified_tokens_per_s": round(K / (with_app["step"] * 1e-3), 1),
           "append_us_per_call_in_step": round(
               (with_app["step"] - without["step"]) * 1e3 / (2 * layers), 2),
           "launches_per_step": wl.launches_per_step,
           "device_status": int(wl.status.item())}
    del wl
    torch.cuda.empty_cache()
    return out


def run_prefill(dev, stream, tc_peak, launches=4):
    """The AR view's pre-filling pass: causal attention over a whole prompt of P
    tokens (batch 1, 32 query / 8 KV heads, head_dim 128), one layer, timed
    alone in a CUDA graph of back-to-back launches.  Flops = 4 * Hq * d * sum
    over rows of the keys each row attends (i + 1 for row i): the masked-out
    upper triangle is not counted."""
    import torch
    from lossless_block_drafting_b200 import orthrus as ob
    out = []
    Hq, Hkv, d = QWEN["Hq"], QWEN["Hkv"], QWEN["d"]
    for P in (4096, 32768):
        g = torch.Generator(device=dev).manual_seed(P)
        q = torch.randn(1, P, Hq, d, generator=g, device=dev).to(torch.bfloat16)
        kc = torch.randn(1, Hkv, P, d, generator=g, device=dev).to(torch.bfloat16)
        vc = torch.randn(1, Hkv, P, d, generator=g, device=dev).to(torch.bfloat16)
        cl = torch.zeros(1, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        view = ob.kv_cache_view(kc, vc, cl)
        with torch.cuda.stream(stream):
            ob.prefill_attn(q, None, None, None, out=o, dev_status=st, stream=stream,
                            cache_view=view)
            stream.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for _ in range(launches):
                    ob.prefill_attn(q, None, None, None, out=o, dev_status=st, stream=stream,
                                    cache_view=view)
            gr.replay()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            gr.replay()
            t1.record(stream)
        torch.cuda.synchronize()
        us = t0.elapsed_time(t1) * 1e3 / launches
        flops = 4.0 * Hq * d * P * (P + 1) / 2
        tf = flops / (us * 1e-6) / 1e12
        out.append({"P": P, "us_per_call": round(us, 1), "TFLOP_per_s": round(tf, 1),
                    "frac_of_bf16_peak_burst": round(tf / tc_peak, 4),
                    "device_status": int(st.item())})
        del gr, q, kc, vc, o
        torch.cuda.empty_cache()
    return {"workload": "whole-prompt causal attention, batch 1, 32q/8kv d128, one layer",
            "points": out, "bound": "tensor"}


def run_sweep(dev, stream, hbm_peak, n_steps=4):
    """The verify-step sweep: K in {1, 4, 8, 16, 32} x context in {1024, 8192,
    40960, 131072}, batch 1, 36 layers: per point the AR pass (36 block
    attentions), the LM head + argmax and verify + commit, from a CUDA graph of
    n_steps steps.  One set of caches per context serves every K."""
    import torch
    out = []
    for L in (1024, 8192, 40960, 131072):
        base = Workload(1, 32, L, QWEN["layers"], 0, n_steps + 4, dev, seed=7)
        kv = (base.k, base.v)
        for K in (1, 4, 8, 16, 32):
            wl = base if K == 32 else Workload(1, K, L, QWEN["layers"], 0, n_steps + 4, dev,
                                               seed=7 + K, kv=kv)
            ph = time_graph_steps(wl, stream, n_steps, verify_only=True)
            verify_ms = ph["ar_attn"] + ph["ar_lm"] + ph["verify"]
            attn_us = ph["ar_attn"] * 1e3 / wl.layers
            gbs = wl.attn_bytes() / (attn_us * 1e-6) / 1e9
            out.append({"ctx": L, "K": K, "verify_step_ms": round(verify_ms, 4),
                        "attn_us": round(attn_us, 2), "attn_GB_per_s": round(gbs, 1),
                        "attn_frac_of_hbm_peak": round(gbs / hbm_peak, 4),
                        "lmhead_us": round(ph["ar_lm"] * 1e3, 2),
                        "verified_tokens_per_s": round(K / (verify_ms * 1e-3), 1)})
            if wl is not base:
                del wl
        del base, kv
        torch.cuda.empty_cache()
    return out


# -------------------------------------------------------------- CPU oracle
class OracleSample:
    """The fp64 oracle timed on a bounded sample of one step, scaled to a step.

    Sample: AR-mask attention of ONE KV head (its 4 query heads x K rows) of one
    layer at context L, and the LM head for `lm_rows` of the K hidden rows.
    Scaled: attention x (8 KV heads x layers x 2 passes), LM head x (K/lm_rows x 2).
    """

    def __init__(self, L, K, layers, lm_rows=8, seed=0):
        from lossless_block_drafting_b200 import synth
        self.L, self.K, self.layers, self.lm_rows = L, K, layers, lm_rows
        self.case = synth.attn_case(1, K, 4, 1, 128, [L], seed=seed, poison=None)
        self.h, self.W = synth.lmhead_case(lm_rows, QWEN["H"], QWEN["V"], seed=seed)

    def run(self):
        import numpy as np

        import oracle
        c = self.case
        t0 = time.perf_counter()
        oracle.block_attn(c.q, c.k_cache, c.v_cache, c.ctx_lens, oracle.MASK_AR)
        t_attn = time.perf_counter() - t0
        t0 = time.perf_counter()
        am, _, _ = oracle.lmhead_argmax(self.h, self.W)
        t_lm = time.perf_counter() - t0
        blk = np.asarray([np.resize(am, self.K)])
        t0 = time.perf_counter()
        oracle.verify(blk, blk)
        t_v = time.perf_counter() - t0
        t_step = (t_attn * QWEN["Hkv"] * self.layers * 2 + t_lm * (self.K / self.lm_rows) * 2
                  + t_v)
        return {"t_attn_sample_s": t_attn, "t_lm_sample_s": t_lm, "t_step_s": t_step,
                "threads": oracle.num_threads()}

    def describe(self, r):
        return (f"fp64 C oracle: AR attention of 1 of 8 KV heads of 1 layer at ctx {self.L} "
                f"({r['t_attn_sample_s']:.2f} s) + LM head for {self.lm_rows} of {self.K} rows "
                f"({r['t_lm_sample_s']:.2f} s), scaled to 2 passes x {self.layers} layers x 8 "
                f"KV heads and 2 x {self.K} LM-head rows (step {r['t_step_s']:.1f} s)")


def cpu_baseline(L, K, layers):
    s = OracleSample(L, K, layers)
    r = s.run()
    return {"value": round(K / r["t_step_s"], 4), "unit": UNIT, "cores": r["threads"],
            "kind": "oracle", "sample": s.describe(r)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    L, K, layers = args.ctx, args.block, args.layers
    s = OracleSample(L, K, layers)
    for _ in range(args.warmup):
        s.run()
    rs = [s.run() for _ in range(args.steps)]
    t_step = statistics.mean(r["t_step_s"] for r in rs)
    value = args.batch * K / t_step
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_step * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"qwen3-8b-shaped dual-view decode step: {layers} layers, "
                               f"batch {args.batch}, K {K}, context {L}",
                   "reference": "fp64 CPU oracle (the pages publish no code to run)"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "kind": "oracle",
                         "cores": oracle.num_threads(), "sample": s.describe(rs[-1])},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        line = json.dumps(res)
        print(line, flush=True)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(line + "\n")
    return 0


if __name__ == "__main__":
    sys.exit(main())
