"""Benchmark of one TiDAR decode step on B200: L x tidar_attn_step + tidar_verify_commit (the verify and the
commit in one launch).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

Prints one JSON line (rank 0).  The default workload is the Qwen3-8B-shaped
step (36 layers, 32 query / 8 KV heads, head dim 128, cached prefix 4096,
draft length 8 -> 80 query rows per layer, vocabulary 151936, batch 1).
Inputs are synthetic and seeded: Q/K/V and the KV caches are drawn on the
device, the logits, drafts and uniforms by the numpy recipe the parity tests
use.  Every layer has its own KV cache, so a step reads ~0.6 GB, far more
than the 126 MB L2.

Timing: the step is captured in a CUDA graph (layers stay separate launches);
W warm-up replays, then K timed replays between CUDA events on the launching
stream, with a barrier and device synchronise on both sides; the max over
ranks is reported.  `e2e` runs the same step through the C ABI without a
graph, every step copying its inputs from pinned host memory and reading its
results back on the host (host wall clock).  With --gpus N > 1 the script
starts N replicas itself (torchrun, one process per GPU) unless a launcher
already did; every rank runs an independent replica (the path has no
cross-GPU exchange), so scaling is weak.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TiDAR decode steps/s (attn+verify+commit) at 1 B200; % of HBM roofline"
UNIT = "steps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(cfg, B):
    return (f"{cfg.name}: {cfg.L} layers, Hq {cfg.Hq} / Hkv {cfg.Hkv}, D {cfg.D}, prefix {cfg.P}"
            + (f" (ragged {cfg.ragged[0]}..{cfg.ragged[1]})" if cfg.ragged else "")
            + f", k {cfg.k} ({cfg.R} query rows), vocab {cfg.V}, batch {B}")


def algorithmic_bytes(cfg, prefix_sum):
    """Compulsory HBM bytes of one step: every cached K/V row of every layer read once, the step's own
    Q/K_new/V_new read and O/LSE written once per layer, and the vocabulary rows the verify and the draft
    selection must read (p, q and the k slot rows of group j*)."""
    B, L, R = cfg.B, cfg.L, cfg.R
    es = 2 if cfg.logits_dtype == "bf16" else 4
    kv = 4 * L * cfg.Hkv * cfg.D * prefix_sum                    # K and V cache rows, bf16
    qkvo = L * B * R * (4 * cfg.Hq * cfg.D + 4 * cfg.Hkv * cfg.D + 4 * cfg.Hq)  # Q, K_new, V_new, O (bf16), LSE (f32)
    logits = 3 * B * cfg.k * cfg.V * es                          # p, q and the k rows of group j*
    commit = 0  # accepted rows copied: counted below from the measured accept lengths
    return dict(kv=kv, qkvo=qkvo, logits=logits, commit=commit)


def attn_flops(cfg, prefix_sum):
    return 4 * cfg.L * cfg.Hq * cfg.R * cfg.D * prefix_sum


# ---------------------------------------------------------------------------
# clocks


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            text = f.read()
        os.unlink(self.file.name)
        return parse_clock_samples(text)


def parse_clock_samples(text):
    """Median SM clock, max SM clock and the throttle reasons seen in nvidia-smi CSV samples of
    ClockSampler.QUERY (no header, no units)."""
    rows = [r.split(",") for r in text.strip().splitlines() if r.strip()]
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        r = [x.strip() for x in r]
        if len(r) < 9:
            continue
        try:
            sm.append(float(r[1]))
            mx.append(float(r[2]))
        except ValueError:
            continue
        for n, v in zip(names, r[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
    sm_sorted = sorted(sm)
    return {"sm_mhz": sm_sorted[len(sm) // 2], "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


# ---------------------------------------------------------------------------
# the GPU arm


class Step:
    """Device-resident inputs and outputs of one decode step, and its launches."""

    def __init__(self, cfg, device, seed=0):
        import numpy as np
        import torch
        from ar_lm_decoding_b200 import abi
        self.abi = abi
        self.cfg = cfg
        self.dev = device
        B, L, R, Hq, Hkv, D, k, V, Pm = cfg.B, cfg.L, cfg.R, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, cfg.V, cfg.P_max
        g = torch.Generator(device=device).manual_seed(seed)
        bf = torch.bfloat16

        def randn(*shape, std=1.0, dtype=bf):
            return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)

        from ar_lm_decoding_b200 import synth
        self.prefix0 = torch.from_numpy(synth.prefix_lengths(cfg, seed)).to(device)
        self.prefix = self.prefix0.clone()
        self.prefix_sum = int(self.prefix0.sum().item())
        # per-step inputs that a model forward would produce, packed in one buffer (for the e2e copy)
        shapes = []
        for _ in range(L):
            shapes += [(B, R, Hq, D), (B, R, Hkv, D), (B, R, Hkv, D)]
        ldt = bf if cfg.logits_dtype == "bf16" else torch.float32
        self.ldt = abi.TIDAR_DT_BF16 if cfg.logits_dtype == "bf16" else abi.TIDAR_DT_F32
        n_carves = len(shapes) + 9
        nbytes = sum(math.prod(s) * 2 for s in shapes) + 2 * B * k * V * (2 if ldt == bf else 4) \
            + B * (k + 1) * k * V * (2 if ldt == bf else 4) + 4 * B * k * 3 + 4 * B + B + 256 * (n_carves + 1)
        self.in_bytes = nbytes
        self.inbuf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        off = [0]

        def carve(shape, dtype):
            n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
            t = self.inbuf[off[0]:off[0] + n].view(dtype).view(*shape)
            off[0] = (off[0] + n + 255) // 256 * 256
            return t

        self.q, self.kn, self.vn = [], [], []
        self.layer_bytes = []  # [start, end) of each layer's inputs in inbuf, then of the verify/commit inputs
        for _ in range(L):
            a = off[0]
            self.q.append(carve((B, R, Hq, D), bf))
            self.kn.append(carve((B, R, Hkv, D), bf))
            self.vn.append(carve((B, R, Hkv, D), bf))
            self.layer_bytes.append((a, off[0]))
        tail0 = off[0]
        self.p_logits = carve((B, k, V), ldt)
        self.q_logits = carve((B, k, V), ldt)
        self.g_logits = carve((B, k + 1, k, V), ldt)
        self.drafts = carve((B, k), torch.int32)
        self.u_acc = carve((B, k), torch.float32)
        self.u_draft = carve((B, k), torch.float32)
        self.u_res = carve((B,), torch.float32)
        self.pre = carve((B,), torch.uint8)
        self.in_bytes = off[0]
        self.layer_bytes.append((tail0, off[0]))
        for t in self.q + self.kn + self.vn:
            t.copy_(randn(*t.shape))
        # logits, drafts, pre-accepted flags and uniforms: the seeded recipe the parity tests use (planted peaks
        # where the workload has them, so that the accept length and the commit's copies vary)
        vin = synth.make_verify_inputs(cfg, seed=seed)

        def put(dst, a):
            a = np.ascontiguousarray(a)
            src = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
            dst.view(src.dtype).copy_(src.reshape(dst.shape))

        put(self.p_logits, vin["p_logits"])
        put(self.q_logits, vin["q_logits"])
        put(self.g_logits, vin["group_logits"])
        put(self.drafts, vin["drafts"])
        put(self.u_acc, vin["u_acc"])
        put(self.u_draft, vin["u_draft"])
        put(self.u_res, vin["u_res"])
        put(self.pre, vin["preaccepted"])
        self.pre_u8 = self.pre
        # KV caches: one per layer (distinct memory)
        self.kc = [randn(B, Hkv, Pm, D) for _ in range(L)]
        self.vc = [randn(B, Hkv, Pm, D) for _ in range(L)]
        self.kc_ptrs = abi.pointer_array(self.kc, device)
        self.vc_ptrs = abi.pointer_array(self.vc, device)
        self.kn_ptrs = abi.pointer_array(self.kn, device)
        self.vn_ptrs = abi.pointer_array(self.vn, device)
        # outputs
        self.out = [torch.empty(B, R, Hq, D, dtype=bf, device=device) for _ in range(L)]
        self.lse = [torch.empty(B, R, Hq, dtype=torch.float32, device=device) for _ in range(L)]
        self.outbuf = torch.zeros(4 * B * (4 + 3 * k) + 256, dtype=torch.uint8, device=device)
        o = [0]

        def ocarve(n, dtype):
            t = self.outbuf[o[0]:o[0] + 4 * n].view(dtype)
            o[0] += 4 * n
            return t

        self.accept_len = ocarve(B, torch.int32)
        self.resampled = ocarve(B, torch.int32)
        self.n_emitted = ocarve(B, torch.int32)
        self.tokens = ocarve(B * k, torch.int32)
        self.next_drafts = ocarve(B * k, torch.int32)
        self.next_q_group = ocarve(B, torch.int32)
        self.next_pre = ocarve(B, torch.int32).view(torch.uint8)[:B]
        self.out_bytes = o[0]
        self.logp = torch.empty(B, k, dtype=torch.float32, device=device)
        self.logq = torch.empty(B, k, dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws_attn_n = abi.tidar_attn_workspace_size(B, Hq, Hkv, D, k, Pm)
        self.ws_ver_n = abi.tidar_verify_workspace_size(B, k, V)
        self.ws_com_n = abi.tidar_kv_commit_workspace_size(B, k, V)
        self.ws_vc_n = abi.tidar_verify_commit_workspace_size(B, k, V)
        self.ws = torch.empty(max(self.ws_attn_n, self.ws_ver_n, self.ws_com_n, self.ws_vc_n), dtype=torch.uint8,
                              device=device)
        self.scale = 1.0 / math.sqrt(D)
        self.launches_per_step = None

    def attn(self, l, stream):
        c = self.cfg
        self.abi.tidar_attn_step(self.q[l], self.kn[l], self.vn[l], self.kc[l], self.vc[l], self.prefix, c.B, c.Hq,
                                 c.Hkv, c.D, c.k, c.P_max, self.scale, self.abi.TIDAR_MASK_HYBRID, self.out[l],
                                 self.lse[l], self.ws, self.ws.numel(), self.status, stream)

    def verify(self, stream):
        c = self.cfg
        self.abi.tidar_verify(self.p_logits, self.q_logits, self.ldt, self.drafts, self.pre_u8, self.u_acc,
                              self.u_res, c.B, c.k, c.V, self.accept_len, self.resampled, self.tokens,
                              self.n_emitted, self.logp, self.logq, self.ws, self.ws.numel(), self.status, stream)

    def commit(self, stream):
        c = self.cfg
        self.abi.tidar_kv_commit(self.kc_ptrs, self.vc_ptrs, self.kn_ptrs, self.vn_ptrs, c.L, c.B, c.Hkv, c.D, c.k,
                                 c.P_max, self.prefix, self.accept_len, self.resampled, self.g_logits, self.ldt, c.V,
                                 self.u_draft, self.next_drafts, self.next_pre, self.next_q_group, self.ws,
                                 self.ws.numel(), self.status, stream)

    def verify_commit(self, stream):
        c = self.cfg
        self.abi.tidar_verify_commit(self.p_logits, self.q_logits, self.ldt, self.drafts, self.pre_u8, self.u_acc,
                                     self.u_res, 1.0, self.kc_ptrs, self.vc_ptrs, self.kn_ptrs, self.vn_ptrs, None, 0,
                                     0, c.L, c.B, c.Hkv, c.D, c.k, c.P_max, c.V, self.prefix, self.g_logits,
                                     self.u_draft, self.accept_len, self.resampled, self.tokens, self.n_emitted,
                                     self.logp, self.logq, self.next_drafts, self.next_pre, self.next_q_group,
                                     self.ws, self.ws.numel(), self.status, stream)

    def run(self, stream):
        """One decode step (prefix length restored first so every step sees the same prefix)."""
        self.prefix.copy_(self.prefix0)
        for l in range(self.cfg.L):
            self.attn(l, stream)
        self.verify_commit(stream)


def gpu_smi_id(device):
    """nvidia-smi --id for a torch device (its UUID, so CUDA_VISIBLE_DEVICES remapping does not matter)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # noqa: BLE001 - fall back to the ordinal
        return str(device.index or 0)


class Ranks:
    """The replicas of a multi-GPU run (one process per GPU, torch.distributed initialised by the caller):
    a barrier and the maximum of a per-rank time, so that every figure is the slowest rank's."""

    def __init__(self, world, device=None):
        self.world, self.device = world, device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x):
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def job_throughput(world, step_s):
    """Whole-job steps/s: each of the `world` replicas completes one step every `step_s` seconds (the slowest
    rank's step time)."""
    return world / step_s


def kernels_per_step(cfg):
    # per layer: one attention kernel (split-KV merged in-kernel); verify + commit: one cooperative kernel (its
    # counters are zeroed by a memset node, not a kernel)
    return cfg.L + 1


def init_ranks(backend):
    """(world, rank, local rank) from the launcher's environment; joins the process group when world > 1
    (NCCL for the GPU arm: only the barrier and the max-over-ranks reduction use it)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120), **kw)
    return world, rank, local


def replica_dry_run(args, cfg):
    """The replica bookkeeping alone, on CPU over gloo: every rank joins, passes the barriers, contributes a
    per-rank time to the max-over-ranks reduction, and rank 0 prints the line's replica fields.  No GPU work:
    it checks the launcher and the rank plumbing the GPU arm uses."""
    import torch
    import torch.distributed as dist
    world, rank, _ = init_ranks("gloo")
    ranks = Ranks(world, torch.device("cpu"))
    ranks.barrier()
    step_s = ranks.max(1e-3 * (1 + rank))  # rank r pretends a step takes (r+1) ms: the slowest rank counts
    ranks.barrier()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {"mode": "replica_dry_run", "metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 5),
            "value": round(job_throughput(world, step_s), 3), "scaling": "weak",
            "config": {"workload": workload_desc(cfg, cfg.B),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}}


def gpu_arm(args, cfg):
    import torch
    import torch.distributed as dist

    world, rank, local = init_ranks("nccl")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    ranks = Ranks(world, device)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    step = Step(cfg, device, seed=rank)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()
    # warm the library and check the device status once
    with torch.cuda.stream(stream):
        step.run(stream.cuda_stream)
    torch.cuda.synchronize()
    assert step.status.item() == 0, f"device status {step.status.item()}"

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step.run(stream.cuda_stream)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_smi_id(device))
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ck = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms)
    ms_step = ms / args.steps
    assert step.status.item() == 0
    accept = step.accept_len.cpu().numpy()

    # dominant-kernel timing: the step's L tidar_attn_step launches captured alone in a graph on the same
    # stream, replayed and timed with events on that stream (average launch duration as it runs in the step)
    attn_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(attn_graph, stream=stream):
        for l in range(cfg.L):
            step.attn(l, stream.cuda_stream)
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 200))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            attn_graph.replay()
        a0.record(stream)
        for _ in range(reps):
            attn_graph.replay()
        a1.record(stream)
    torch.cuda.synchronize()
    attn_ms_launch = max_over_ranks(a0.elapsed_time(a1) / (reps * cfg.L))
    del attn_graph
    # the step's verify + commit launch, and (for comparison) the two separate calls it replaces; each graph
    # restores the prefix length first (a 4-byte copy node)
    breakdown = {"attn_us_per_launch": round(attn_ms_launch * 1e3, 3),
                 "verify_commit_us": round(graph_us(stream, reps, lambda: (step.prefix.copy_(step.prefix0),
                                                                           step.verify_commit(stream.cuda_stream))),
                                           3),
                 "separate_verify_us": round(graph_us(stream, reps, lambda: step.verify(stream.cuda_stream)), 3),
                 "separate_commit_us": round(graph_us(stream, reps, lambda: (step.prefix.copy_(step.prefix0),
                                                                             step.commit(stream.cuda_stream))), 3)}

    e2e = e2e_leg(step, stream, args, barrier, max_over_ranks, world)

    del graph
    torch.cuda.synchronize()

    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    byts = algorithmic_bytes(cfg, step.prefix_sum)
    commit_bytes = 4 * cfg.L * cfg.Hkv * cfg.D * int(accept.sum()) * 1  # read new rows + write cache rows (K and V)
    total_bytes = byts["kv"] + byts["qkvo"] + byts["logits"] + commit_bytes
    kvlog = byts["kv"] + byts["logits"]
    step_s = ms_step / 1e3
    flops = attn_flops(cfg, step.prefix_sum)
    attn_bytes_launch = (byts["kv"] + byts["qkvo"]) / cfg.L
    achieved = attn_bytes_launch / (attn_ms_launch / 1e3) / 1e9
    traffic = load_traffic(cfg)
    value = job_throughput(world, step_s)
    res = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; Q/K/V and caches generated on the device, logits/drafts/uniforms by the "
                "parity tests' numpy recipe)",
        "config": {"workload": workload_desc(cfg, cfg.B), "batch": cfg.B,
                   "l2": "inputs larger than L2: every layer has its own KV cache "
                         f"({byts['kv'] / 1e6:.0f} MB KV per step vs 126 MB L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "hbm_roofline": {"kv_logit_frac": round(kvlog / step_s / 1e9 / hbm, 4),
                         "all_bytes_frac": round(total_bytes / step_s / 1e9 / hbm, 4),
                         "tensor_frac": round(flops / step_s / 1e12 / float(peaks["bf16_tflops"]), 4),
                         "kv_logit_bytes": kvlog, "all_bytes": total_bytes, "attn_flops": flops,
                         "peak_gbs": hbm, "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic,
                     "kernel": "attn_sm100_kernel (tidar_attn_step: one layer, split-KV merged in-kernel)",
                     "bytes_per_launch": attn_bytes_launch, "us_per_launch": round(attn_ms_launch * 1e3, 3),
                     "tensor_frac": round(flops / cfg.L / (attn_ms_launch / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
                                          4),
                     "peak_kind": peak_kind},
        "clocks": ck,
        "breakdown": breakdown,
        "e2e": e2e,
        "gpu_launches": kernels_per_step(cfg) * args.steps,
        "accept_len": accept.tolist(),
    }
    check_line(res)
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    return res if rank == 0 else None


def graph_us(stream, reps, fn):
    """Average duration of `fn`'s launches captured alone in a CUDA graph on `stream` (events on that stream)."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / reps


def copy_groups(L, cap=8):
    """Layers per host-to-device copy in the end-to-end step: 1, 2, 4, 8, 8, ... (the last group takes the rest),
    so that the first layer starts after one layer's inputs while the copies stay few (each copy costs a fixed
    overhead: one per layer ran the Qwen3-8B inputs at 45 GB/s, groups of 6-18 layers at 50.6-51.4, of a 55 GB/s
    link); the cap keeps a compute-bound step from waiting on one very large late copy."""
    groups, l0, n = [], 0, 1
    while l0 < L:
        groups.append((l0, min(L, l0 + n)))
        l0, n = l0 + n, min(cap, 2 * n)
    return groups


def e2e_step(step, stream, copy_stream, events, pin_in, pin_out):
    """One decode step through the C ABI as a user runs it: this step's inputs (every layer's Q / K_new /
    V_new, the p / q / group logits, drafts and uniforms) copied from pinned host memory, the L + 1 library
    calls, the results copied back and read on the host.  The input copies are issued on a second stream in
    groups of consecutive layers (copy_groups), so that later layers' inputs cross the host link while earlier
    layers compute; every attention call waits only for its own group's inputs, the verify/commit call for the
    last copy (its logits, drafts and uniforms)."""
    import torch
    cfg = step.cfg
    groups = copy_groups(cfg.L)
    copy_stream.wait_stream(stream)  # the previous step no longer reads the input buffer
    with torch.cuda.stream(copy_stream):
        for (l0, l1), ev in zip(groups, events):
            a, b = step.layer_bytes[l0][0], step.layer_bytes[l1 - 1][1]
            step.inbuf[a:b].copy_(pin_in[a:b], non_blocking=True)
            ev.record(copy_stream)
        a, b = step.layer_bytes[-1]
        step.inbuf[a:b].copy_(pin_in[a:b], non_blocking=True)
        events[-1].record(copy_stream)
    with torch.cuda.stream(stream):
        step.prefix.copy_(step.prefix0)
        for (l0, l1), ev in zip(groups, events):
            stream.wait_event(ev)
            for l in range(l0, l1):
                step.attn(l, stream.cuda_stream)
        stream.wait_event(events[-1])
        step.verify_commit(stream.cuda_stream)
        pin_out.copy_(step.outbuf[:step.out_bytes], non_blocking=True)
    stream.synchronize()
    return int(pin_out[:4].view(torch.int32).item())  # the accept length of sequence 0, read on the host


def e2e_leg(step, stream, args, barrier, max_over_ranks, world):
    """End-to-end steps/s through the public API with host buffers (host wall clock over the timed steps,
    the host waiting for each step's results; the slowest rank's time)."""
    import torch
    pin_in = torch.empty(step.in_bytes, dtype=torch.uint8, pin_memory=True)
    pin_in.copy_(step.inbuf[:step.in_bytes])
    pin_out = torch.empty(step.out_bytes, dtype=torch.uint8, pin_memory=True)
    copy_stream = torch.cuda.Stream(step.dev)
    events = [torch.cuda.Event() for _ in range(len(copy_groups(step.cfg.L)) + 1)]
    n = max(3, min(args.steps, 200))
    for _ in range(3):
        e2e_step(step, stream, copy_stream, events, pin_in, pin_out)
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for _ in range(n):
        acc = e2e_step(step, stream, copy_stream, events, pin_in, pin_out)
        assert 0 <= acc <= step.cfg.k
    s = max_over_ranks(time.perf_counter() - t0)
    torch.cuda.synchronize()
    assert step.status.item() == 0
    return {"value": round(world * n / s, 3), "unit": UNIT, "h2d_bytes_per_step": step.in_bytes,
            "d2h_bytes_per_step": step.out_bytes, "steps": n,
            "host_link_gbs": round(step.in_bytes * n / s / 1e9, 2)}


def check_line(res):
    """Sanity rules of the printed line: the end-to-end rate, which adds host copies to the same kernels,
    cannot exceed the device-timed rate; the dominant kernel cannot take longer than the step."""
    assert res["e2e"]["value"] <= res["value"] * 1.02, (res["e2e"]["value"], res["value"])
    us_attn = res["roofline"]["us_per_launch"]
    assert us_attn * (res["gpu_launches"] / res["steps"] - 2) <= res["ms_per_step"] * 1e3 * 1.05, res


def load_traffic(cfg):
    """DRAM bytes per attention launch from the committed ncu summary, if it matches this build."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("source_sha256") != kernel_source_hash() or d.get("workload") != cfg.name:
            return None
        return d.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None


def kernel_source_hash():
    """Hash of the attention kernel's code (its sources with comments and layout removed), so that the DRAM
    traffic recorded for it is dropped when the code changes but kept across comment edits."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ar_lm_decoding_b200", "csrc")
    for n in sorted(os.listdir(csrc)):
        if n.startswith("attn") or n in ("common.cuh", "tc.cuh"):
            with open(os.path.join(csrc, n)) as f:
                code = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)
            code = " ".join(re.sub(r"//[^\n]*", " ", code).split())
            h.update(n.encode() + code.encode())
    return h.hexdigest()


# ---------------------------------------------------------------------------
# the CPU oracle (baseline and reference arm)


class OracleWorkload:
    """The CPU oracle on the bench workload: inputs generated once, calls timed."""

    def __init__(self, cfg, seed=0):
        import numpy as np
        import oracle
        from ar_lm_decoding_b200 import synth
        self.np, self.oracle, self.cfg = np, oracle, cfg
        self.inp = synth.make_attn_inputs(cfg, seed=seed, poison=False)
        self.v = synth.make_verify_inputs(cfg, seed=seed)
        self.kc = np.zeros((1, cfg.B, cfg.Hkv, cfg.P_max, cfg.D), np.uint16)
        self.kn = np.zeros((1, cfg.B, cfg.R, cfg.Hkv, cfg.D), np.uint16)
        self.rng = np.random.default_rng(seed)
        self.cores = oracle.default_threads()
        self.threads = self.cores
        self.rows_total = cfg.B * cfg.Hq * cfg.R

    def attn_rows(self, rows):
        c = self.cfg
        sb = self.rng.integers(0, c.B, rows)
        sh = self.rng.integers(0, c.Hq, rows)
        sr = self.rng.integers(0, c.R, rows)
        t0 = time.perf_counter()
        self.oracle.attn_rows(self.inp, c.Hq, c.Hkv, c.D, c.k, sb, sh, sr, nthreads=self.threads)
        return time.perf_counter() - t0

    def attn_layer(self):
        """All query rows of one layer (every sequence, head and row)."""
        c = self.cfg
        t0 = time.perf_counter()
        self.oracle.attn(self.inp, c.Hq, c.Hkv, c.D, c.k, dense=False, nthreads=self.threads)
        return time.perf_counter() - t0

    def verify_commit(self):
        t0 = time.perf_counter()
        out = self.oracle.verify(self.v, nthreads=self.threads)
        self.oracle.kv_commit(self.kc, self.kc, self.kn, self.kn, self.inp["prefix_len"], out["accept_len"],
                              out["resampled"], self.v["group_logits"], self.v["u_draft"], nthreads=self.threads)
        return time.perf_counter() - t0

    def rows_for(self, seconds):
        n = max(self.cores, 8)
        per_row = self.attn_rows(n) / n
        return int(min(self.rows_total, max(1, seconds / max(per_row, 1e-7))))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def host_cores():
    return {"affinity": len(os.sched_getaffinity(0)), "nproc": os.cpu_count(), "cpu_model": cpu_model()}


def cpu_baseline(cfg, seconds):
    """Oracle steps/s on the host cores from a bounded sample of attention rows, with OpenMP over all the
    cores this process may use and single-threaded."""
    w = OracleWorkload(cfg)
    res = {}
    for label, threads, budget in (("all_cores", w.cores, seconds), ("single_thread", 1, seconds / 3)):
        w.threads = threads
        rows = max(threads, w.rows_for(budget))
        t_rows, reps = 0.0, 0
        while reps < 1 or (t_rows < budget and reps < 50):  # repeat the row sample up to ~`budget` seconds
            t_rows += w.attn_rows(rows)
            reps += 1
        t_rows /= reps
        t_vc = w.verify_commit()
        t_step = cfg.L * t_rows * w.rows_total / rows + t_vc
        res[label] = {"value": round(1.0 / t_step, 6), "threads": threads, "seconds_per_step": round(t_step, 3),
                      "sample": f"{rows} of {w.rows_total} attention rows of one layer, timed {reps}x (scaled "
                                f"x{w.rows_total / rows:.1f} and x{cfg.L} layers, which do identical work), plus "
                                f"the full verify and commit with draft selection; {reps * t_rows + t_vc:.1f} s "
                                f"of wall time"}
    a = res["all_cores"]
    return {"value": a["value"], "unit": UNIT, "cores": a["threads"], "kind": "oracle", "sample": a["sample"],
            "seconds_per_step": a["seconds_per_step"], "single_thread": res["single_thread"], "host": host_cores()}


def reference_arm(args, cfg):
    """The oracle as the reference implementation.  Every timed step is a whole decode step of the workload:
    the oracle's attention over all query rows of a layer, run once per layer (the same layer inputs L times:
    the layers do identical work), then its verify and its commit with draft selection.  The warm-up steps
    run one layer each (untimed)."""
    w = OracleWorkload(cfg)
    for _ in range(args.warmup):
        w.attn_layer()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(cfg.L):
            w.attn_layer()
        w.verify_commit()
    t_step = (time.perf_counter() - t0) / args.steps
    value = 1.0 / t_step
    sample = (f"each timed step: all {w.rows_total} attention rows of a layer x {cfg.L} layers (the same layer "
              f"inputs each time), then the full verify and commit with draft selection, on {w.cores} threads; "
              f"warm-up steps run one layer")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy)",
        "config": {"workload": workload_desc(cfg, cfg.B), "batch": cfg.B},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": w.cores, "kind": "oracle",
                         "sample": sample, "host": host_cores()},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def attn_prefix_sweep(args, cfg):
    """Attention time per launch against the prefix length at a fixed P_max (so a fixed split count): the
    intercept of the line is the per-launch fixed cost (set-up, first copies, epilogue), the slope the cost
    of one more key tile of a row tile.  One JSON line per prefix length, then the fit."""
    import torch
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    step = Step(cfg, device)
    stream = torch.cuda.Stream(device)
    pts = []
    for P in sorted({min(cfg.P_max, x) for x in (128, 1024, 2048, 3072, 4096)}):
        step.prefix.fill_(P)
        with torch.cuda.stream(stream):
            for l in range(cfg.L):
                step.attn(l, stream.cuda_stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for l in range(cfg.L):
                step.attn(l, stream.cuda_stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                g.replay()
            e0.record(stream)
            reps = max(3, min(args.steps, 50))
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * cfg.L)
        tiles = math.ceil(P / 128) + math.ceil(cfg.R / 128)
        pts.append((tiles, us))
        print(json.dumps({"mode": "attn_prefix_sweep", "workload": cfg.name, "prefix": P, "key_tiles": tiles,
                          "us_per_launch": round(us, 3), "status": int(step.status.item())}), flush=True)
        del g
    n = len(pts)
    mx = sum(t for t, _ in pts) / n
    my = sum(u for _, u in pts) / n
    slope = sum((t - mx) * (u - my) for t, u in pts) / max(1e-9, sum((t - mx) ** 2 for t, _ in pts))
    print(json.dumps({"mode": "attn_prefix_sweep_fit", "workload": cfg.name, "fixed_us": round(my - slope * mx, 3),
                      "us_per_key_tile": round(slope, 4)}), flush=True)


def replica_command(argv, n, port):
    """The torchrun command that runs this script as `n` replicas on one node (one process per GPU)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", str(n),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def k_sweep(args, cfg):
    """Step latency against the draft length k at the workload's other sizes (one JSON line per k): where the
    step leaves the memory-bound regime (the TiDAR summary's Fig. 1 observation of free token slots, here for
    this B200 step), and the draft length the step-latency model picks for a few per-draft acceptance rates
    (tidar_pick_draft_length)."""
    import torch
    from ar_lm_decoding_b200 import abi
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    peaks, _ = load_peaks()
    hbm, tf = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    ks = [int(x) for x in args.ks.split(",")]
    table = [0.0] * max(ks)
    for k in ks:
        c = cfg.with_(k=k)
        step = Step(c, device)
        stream = torch.cuda.Stream(device)
        with torch.cuda.stream(stream):
            step.run(stream.cuda_stream)
        torch.cuda.synchronize()
        assert step.status.item() == 0
        reps = max(3, min(args.steps, 50))
        us = graph_us(stream, reps, lambda: step.run(stream.cuda_stream))
        attn = graph_us(stream, reps, lambda: [step.attn(l, stream.cuda_stream) for l in range(c.L)]) / c.L
        byts = algorithmic_bytes(c, step.prefix_sum)
        flops = attn_flops(c, step.prefix_sum)
        table[k - 1] = us
        print(json.dumps({"mode": "k_sweep", "workload": workload_desc(c, c.B), "k": k, "query_rows": c.R,
                          "tokens_per_forward": c.R, "step_us": round(us, 2), "attn_us_per_launch": round(attn, 3),
                          "hbm_bound_us": round((byts["kv"] + byts["qkvo"] + byts["logits"]) / hbm / 1e3, 2),
                          "tensor_bound_us": round(flops / tf / 1e6, 2),
                          "kv_logit_frac": round((byts["kv"] + byts["logits"]) / (us * 1e-6) / 1e9 / hbm, 4),
                          "tensor_frac": round(flops / (us * 1e-6) / 1e12 / tf, 4)}), flush=True)
        del step
        torch.cuda.empty_cache()
    picks = {}
    for alpha in (0.3, 0.5, 0.7, 0.8, 0.9, 0.95):
        k, rate = abi.tidar_pick_draft_length(table, alpha)
        picks[str(alpha)] = {"k": k, "tokens_per_ms": round(rate * 1e3, 3)}
    print(json.dumps({"mode": "k_sweep_pick", "workload": cfg.name, "measured_k": ks, "pick": picks}), flush=True)


QWEN3_32B_LAYER = {"hidden": 5120, "intermediate": 25600, "Hq": 64, "Hkv": 8, "D": 128}


def layer_sweep(args, cfg):
    """Latency of one full decoder layer against the tokens per forward R = k(k+2), at several prefix lengths:
    the QKV projection (cuBLAS GEMM), the rotary embedding fused with the re-layout into the attention inputs
    (tidar_rope_qkv), the hybrid-mask attention (tidar_attn_step), the output projection and the MLP GEMMs
    (cuBLAS), with synthetic bf16 weights of the Qwen3-32B shape.  This is the B200 counterpart of the TiDAR
    summary's Fig. 1 (latency against tokens per forward: flat while the weights and the KV cache dominate,
    rising once the layer is compute-bound); the norms and the activation are left out (elementwise work that
    does not move the curve).  One JSON line per (prefix, k)."""
    import torch
    from ar_lm_decoding_b200 import abi
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    sh = QWEN3_32B_LAYER
    hid, inter, Hq, Hkv, D = sh["hidden"], sh["intermediate"], sh["Hq"], sh["Hkv"], sh["D"]
    g = torch.Generator(device=device).manual_seed(0)

    def w(n_in, n_out):
        return (torch.randn(n_in, n_out, generator=g, device=device) * n_in ** -0.5).to(torch.bfloat16)

    w_qkv, w_o = w(hid, (Hq + 2 * Hkv) * D), w(Hq * D, hid)
    w_gu, w_down = w(hid, 2 * inter), w(inter, hid)
    weight_bytes = 2 * sum(t.numel() for t in (w_qkv, w_o, w_gu, w_down))
    peaks, _ = load_peaks()
    hbm, tf = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    stream = torch.cuda.Stream(device)
    ks = [int(x) for x in args.ks.split(",")]
    for P in [int(x) for x in args.prefixes.split(",")]:
        P_max = (P + 16 + 63) // 64 * 64
        kc = torch.randn(1, Hkv, P_max, D, generator=g, device=device).to(torch.bfloat16)
        vc = torch.randn(1, Hkv, P_max, D, generator=g, device=device).to(torch.bfloat16)
        pl = torch.tensor([P], dtype=torch.int32, device=device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        for k in ks:
            R = k * (k + 2)
            x = torch.randn(R, hid, generator=g, device=device).to(torch.bfloat16)
            qkv = torch.empty(R, (Hq + 2 * Hkv) * D, dtype=torch.bfloat16, device=device)
            q = torch.empty(1, R, Hq, D, dtype=torch.bfloat16, device=device)
            kn = torch.empty(1, R, Hkv, D, dtype=torch.bfloat16, device=device)
            vn = torch.empty(1, R, Hkv, D, dtype=torch.bfloat16, device=device)
            o = torch.empty(1, R, Hq, D, dtype=torch.bfloat16, device=device)
            lse = torch.empty(1, R, Hq, dtype=torch.float32, device=device)

            def layer(with_attn=True):
                torch.matmul(x, w_qkv, out=qkv)
                abi.tidar_rope_qkv(qkv, pl, 1, Hq, Hkv, D, k, 1e6, q, kn, vn, st, stream.cuda_stream)
                if with_attn:
                    abi.tidar_attn_step(q, kn, vn, kc, vc, pl, 1, Hq, Hkv, D, k, P_max, D ** -0.5,
                                        abi.TIDAR_MASK_HYBRID, o, lse, None, 0, st, stream.cuda_stream)
                h = torch.matmul(o.view(R, Hq * D), w_o)
                gu = torch.matmul(h, w_gu)
                torch.matmul(gu[:, :inter], w_down)

            with torch.cuda.stream(stream):
                layer()
            torch.cuda.synchronize()
            assert st.item() == 0
            reps = max(3, min(args.steps, 30))
            us = graph_us(stream, reps, layer)
            attn_us = graph_us(stream, reps, lambda: abi.tidar_attn_step(
                q, kn, vn, kc, vc, pl, 1, Hq, Hkv, D, k, P_max, D ** -0.5, abi.TIDAR_MASK_HYBRID, o, lse, None, 0, st,
                stream.cuda_stream))
            rope_us = graph_us(stream, reps, lambda: abi.tidar_rope_qkv(qkv, pl, 1, Hq, Hkv, D, k, 1e6, q, kn, vn, st,
                                                                        stream.cuda_stream))
            flops = 2 * R * weight_bytes / 2 + 4 * Hq * R * D * P
            byts = weight_bytes + 4 * Hkv * D * P
            print(json.dumps({"mode": "layer_sweep", "shape": "Qwen3-32B layer (hidden 5120, intermediate 25600, "
                              "Hq 64 / Hkv 8, D 128), batch 1", "prefix": P, "k": k, "tokens_per_forward": R,
                              "layer_us": round(us, 2), "attn_us": round(attn_us, 2), "rope_us": round(rope_us, 2),
                              "hbm_bound_us": round(byts / hbm / 1e3, 2),
                              "tensor_bound_us": round(flops / tf / 1e6, 2)}), flush=True)
        del kc, vc
        torch.cuda.empty_cache()


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="qwen3-8b_k8")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attn-prefix-sweep", action="store_true",
                    help="print attention time per launch against the prefix length (not the benchmark line)")
    ap.add_argument("--k-sweep", action="store_true",
                    help="print the step latency for each draft length in --ks (not the benchmark line)")
    ap.add_argument("--ks", default="1,2,4,8,12,16")
    ap.add_argument("--layer-sweep", action="store_true",
                    help="print one full decoder layer's latency against tokens per forward (not the benchmark line)")
    ap.add_argument("--prefixes", default="1024,4096,16384")
    ap.add_argument("--replica-dry-run", action="store_true",
                    help="run only the replica bookkeeping on CPU (gloo) and print its fields (no GPU work)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    from ar_lm_decoding_b200 import synth
    cfg = synth.CONFIGS[args.config]
    world = os.environ.get("WORLD_SIZE")
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        import oracle
        oracle.build()
        print(json.dumps(reference_arm(args, cfg)), flush=True)
        return 0
    if args.attn_prefix_sweep:
        attn_prefix_sweep(args, cfg)
        return 0
    if args.k_sweep:
        k_sweep(args, cfg)
        return 0
    if args.layer_sweep:
        layer_sweep(args, cfg)
        return 0
    if world is None and args.gpus > 1:
        # not under a launcher: start the N replicas (one process per GPU) and pass on their exit status
        return subprocess.call(replica_command(argv, args.gpus, free_port()))
    if world is not None and int(world) != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {world} processes")
    res = replica_dry_run(args, cfg) if args.replica_dry_run else gpu_arm(args, cfg)
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
