"""Benchmark of the GPT-OSS-style MoE feed-forward layer on B200.

One step = one pass of the whole layer (route, permute, gather, mlp1, mlp2,
combine) over one batch of the GPT-OSS-20B-shaped workload (T=8192 tokens,
D=2880, E=32 experts, top-4, I=2880, bf16, synthetic seeded inputs), timed on
the device with CUDA events on the launching stream. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU under torchrun; tokens are independent, so each
rank runs its own batch with replicated weights and no collective on the data
path (weak scaling); the step time is the max over ranks.
``--impl reference`` times the CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WORKLOAD = "gptoss20b"
WORKLOAD_NAMES = {
    "gptoss20b": "gpt-oss-20b-shaped MoE FFN layer",
    "gptoss120b_zipf": "gpt-oss-120b-shaped MoE FFN layer, skewed routing",
    "gptoss20b_mxfp4": "gpt-oss-20b-shaped MoE FFN layer, MXFP4 expert weights",
    "gptoss20b_mxfp4_decode": "gpt-oss-20b-shaped MoE FFN layer, MXFP4 expert weights, 64 tokens",
    "debug": "debug-sized MoE FFN layer",
    "tiny": "tiny MoE FFN layer",
}
METRIC = "MoE layer tokens/s and TFLOP/s at 1 B200, % of tensor-core peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# kernels per step: route 1, permute 3, gather 1, mlp1 1, mlp2 1, combine 1
LAUNCHES_PER_STEP = 8
PERM_SINGLE_MAX = 1024  # T*k up to this: the permutation is one launch instead of three


def act_tuple(args):
    """(kind, alpha, limit) of the layer's activation: 0 plain SwiGLU, 1 the GPT-OSS variant."""
    if getattr(args, "act", "swiglu") == "gptoss":
        return (1, args.act_alpha, args.act_limit)
    return (0, 1.0, float("inf"))


def act_config(args):
    return {} if getattr(args, "act", "swiglu") == "swiglu" else {
        "activation": f"gpt-oss swiglu variant (alpha {args.act_alpha}, limit {args.act_limit})"}


def launches_per_step(T: int, D: int, mxfp4: bool, k: int = 4) -> int:
    """Kernel launches of one staged step: the eight above (the permutation
    in one launch instead of three when T*k <= PERM_SINGLE_MAX), plus for
    MXFP4 weights (prepared once) two more per GEMM -- the activation
    quantiser and the second of the two block-scaled GEMM kernels
    (small-expert and big-tile) -- plus the router's partial-logit reduction
    when it splits K (batches of at most 18 token tiles of 128, D over 64)."""
    n = LAUNCHES_PER_STEP + (4 if mxfp4 else 0) - (2 if T * k <= PERM_SINGLE_MAX else 0)
    tiles, kb = -(-T // 128), -(-D // 64)
    if tiles * 8 <= 148 and min(kb, 148 // tiles) > 1:
        n += 1
    return n


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Clocks:
    """SM clocks, power and clock-event (throttle) reasons sampled during the
    timed region: NVML polled from a thread every 10 ms (reads only), else
    nvidia-smi at its 100 ms minimum period."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.thread = None
        self.rows = []  # (sm_mhz, sm_max_mhz, power_w, reason bits)

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:  # the device torch uses, by PCI bus id (CUDA_VISIBLE_DEVICES may renumber)
            pr = torch.cuda.get_device_properties(self.idx)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def _sample(self):
        nv, h = self.nv, self.h
        self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), self.smax,
                          nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(self.reasons_fn(h))))

    def _poll(self):
        import time

        while not self.stop:
            time.sleep(0.01)
            try:
                self._sample()
            except Exception:
                break

    def __enter__(self):
        self.stop = False
        try:
            import threading

            self.nv, self.h = self._nvml_handle()
            self.smax = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            self.reasons_fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self._sample()  # one sample at the start, one at the end, the thread's in between
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
            self.rows = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
            try:
                self._sample()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if self.rows:
            sm = [r[0] for r in self.rows]
            reasons = sorted({n for r in self.rows for n, bit in self.REASONS.items() if r[3] & bit})
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(self.rows[0][1]), "reasons": reasons,
                    "samples": len(self.rows), "power_w_max": max(r[2] for r in self.rows), "source": "nvml 10 ms"}
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        smax = float(rows[0][2])
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].strip() not in ("", "[N/A]")),
                "source": "nvidia-smi 100 ms"}


GEMM_SOURCES = ("grouped_gemm.cu", "gemm_common.cuh", "sm100.cuh")
MX_SOURCES = ("mx_gemm.cu", "gemm_common.cuh", "sm100.cuh", "common.cuh", "tma_host.cuh")
# workload -> the ncu summary of its mlp1 kernel and the sources that kernel is built from
PROFILE_OF = {
    "gptoss20b": ("mlp1_gptoss20b_ncu.md", GEMM_SOURCES),
    "gptoss20b_mxfp4": ("mx_gemm_gptoss20b_mxfp4_ncu.md", MX_SOURCES),
    "gptoss20b_mxfp4_decode": ("mx_small_gptoss20b_mxfp4_decode_ncu.md", MX_SOURCES),
}


def source_hash(sources=GEMM_SOURCES) -> str:
    """Hash of the sources that make up a kernel."""
    h = hashlib.sha256()
    for name in sources:
        h.update(open(os.path.join(ROOT, "mixture_experts_ffn_layer_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def gemm_source_hash() -> str:
    return source_hash(GEMM_SOURCES)


def traffic_from_profile(workload=WORKLOAD):
    """DRAM bytes per launch of the workload's mlp1 kernel from its committed
    ncu summary, if that was taken on the current kernel sources; else None."""
    if workload not in PROFILE_OF:
        return None
    name, sources = PROFILE_OF[workload]
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    fields = {}
    for line in open(p):
        m = re.match(r"- (\w+): `([^`]*)`", line)
        if m:
            fields[m.group(1)] = m.group(2)
    if fields.get("kernel_sources_sha256_16") != source_hash(sources):
        return None
    try:
        return int(float(fields["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def max_over_ranks(times_ms, world, device="cpu"):
    """Element-wise max of per-rank CUDA-event times (the slowest rank sets
    the step time); identity on one rank."""
    t = torch.tensor(times_ms, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def step_throughput(elapsed_ms, steps, tokens_per_rank, world):
    """(ms per step, whole-job tokens/s): every rank processes its own batch of
    tokens_per_rank tokens per step (replicas, weak scaling)."""
    ms = elapsed_ms / steps
    return ms, tokens_per_rank * world / (ms / 1e3)


def rooflines(shape, inp, stage_ms, mlp1_ms, peak_tf, pk, pk_kind, workload):
    """The dominant kernel's roofline against the resource that bounds it, and
    the memory-bound stages' achieved HBM bandwidth.

    mlp1 (grouped GEMM + SwiGLU) dominates every workload. With few routed rows
    per expert (T*k <= 16*E, decode-sized MXFP4 batches) it is bound by
    streaming the expert weights from HBM: algorithmic bytes = W1 (codes and
    scales, or bf16) + the routed rows read + h written. Otherwise it is bound
    by the tensor cores: 4*R*D*I FLOP per launch."""
    T, D, E, k, I = shape.T, shape.D, shape.E, shape.k, shape.I
    R = T * k
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    w1_bytes = sum(t.numel() * t.element_size() for t in (inp.W1, inp.W1_scales) if t is not None)
    w2_bytes = sum(t.numel() * t.element_size() for t in (inp.W2, inp.W2_scales) if t is not None)
    decode = T * k <= 16 * E
    if decode:
        mlp1_bytes = w1_bytes + R * D * 2 + R * I * 2
        ach = mlp1_bytes / (mlp1_ms / 1e3) / 1e9
        roof = {"kernel": "grouped mlp1 + SwiGLU (tcgen05)", "bound": "hbm", "achieved": ach, "peak": hbm,
                "unit": "GB/s", "frac": ach / hbm, "traffic": traffic_from_profile(workload),
                "peak_kind": f"hbm_gbs ({pk_kind})",
                "algorithmic": f"W1 {w1_bytes} B + routed rows {R * D * 2} B + h {R * I * 2} B per launch"}
    else:
        mlp1_flops = 4.0 * R * D * I
        tf = mlp1_flops / (mlp1_ms / 1e3) / 1e12
        traffic = traffic_from_profile(workload)
        roof = {"kernel": "grouped mlp1 + SwiGLU (tcgen05)", "bound": "tensor", "achieved": tf, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": tf / peak_tf, "traffic": traffic,
                "algorithmic": f"4*R*D*I = {mlp1_flops:.4g} FLOP per launch"}
    # memory-bound stages: algorithmic bytes per launch / CUDA-event time
    mem = {
        "route": T * D * 2 + E * D * 2 + R * 8,
        "gather": T * D * 2 + R * D * 2 + R * 4,  # each token row read once (k copies from L2), R rows written
        "combine": R * D * 4 + T * D * 2 + R * 4,
    }
    if decode:
        mem["mlp2"] = w2_bytes + R * I * 2 + R * D * 4
    out = {}
    for name, nbytes in mem.items():
        ms = stage_ms.get(name)
        if ms:
            gbs = nbytes / (ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "bytes": nbytes, "ms": ms, "achieved_gbs": gbs, "frac": gbs / hbm}
    return roof, out


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import mixture_experts_ffn_layer_b200 as moe

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    workload = args.workload
    shape = synthetic.SHAPES[workload]
    inp = synthetic.make_inputs(workload, seed=synthetic.SEEDS[workload] + 1000 * rank, device=dev)
    T, D, E, k, I = shape.T, shape.D, shape.E, shape.k, shape.I
    R = T * k
    mx = shape.wfmt == "mxfp4"
    d = moe.dims(T, D, E, k, I, moe.MOE_W_MXFP4 if mx else moe.MOE_W_BF16, *act_tuple(args))
    ws = moe.alloc_workspace(d, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    topk_idx = torch.empty((T, k), **i32)
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    perm, inv = torch.empty(R, **i32), torch.empty(R, **i32)
    x_perm = torch.empty((R, D), dtype=torch.bfloat16, device=dev)
    h = torch.empty((R, I), dtype=torch.bfloat16, device=dev)
    o_perm = torch.empty((R, D), dtype=torch.float32, device=dev)
    y = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    stages = ["route", "permute", "gather", "mlp1", "mlp2", "combine"]
    # MXFP4 weights are prepared once (the block-scaled MMAs' scale layout),
    # as a serving process does at model load; not part of the timed step
    W1p = W2p = None
    if mx:
        W1p = moe.mxfp4_prepare(d, 1, inp.W1, inp.W1_scales)
        W2p = moe.mxfp4_prepare(d, 2, inp.W2, inp.W2_scales)

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)

        mark(0)
        moe.moe_route(d, inp.x, inp.Wr, inp.br, topk_idx, topk_w, ws)
        mark(1)
        moe.moe_permute(d, topk_idx, counts, offsets, perm, inv, ws)
        mark(2)
        moe.moe_gather(d, inp.x, perm, x_perm, ws)
        mark(3)
        moe.moe_mlp1(d, x_perm, offsets, inp.W1, inp.b1, h, ws, W1_scales=inp.W1_scales, W1_prepared=W1p)
        mark(4)
        moe.moe_mlp2(d, h, perm, offsets, topk_w, inp.W2, inp.b2, o_perm, ws, W2_scales=inp.W2_scales,
                     W2_prepared=W2p)
        mark(5)
        moe.moe_combine(d, o_perm, inv, y, ws)
        mark(6)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    st = moe.moe_read_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {moe.status_str(st)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    barrier()
    with Clocks(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    elapsed_ms = t_start.elapsed_time(t_end)
    st = moe.moe_read_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {moe.status_str(st)}")
    stage_ms = {s: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i, s in enumerate(stages)}

    # End to end through the one-call API with host buffers: every step copies
    # its input x from pinned host memory to the device, runs moe_forward and
    # copies y back, all inside the timed region. Serving-style pipeline: the
    # copies run on their own streams (one per direction) with double-buffered
    # device buffers, so step i's copies overlap the compute of its
    # neighbours. The plain serial loop is timed too (e2e_serial).
    nbuf = 2
    x_hosts = [inp.x.cpu().pin_memory() for _ in range(nbuf)]
    y_hosts = [torch.empty((T, D), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    x_devs = [torch.empty_like(inp.x) for _ in range(nbuf)]
    y_devs = [torch.empty((T, D), dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d_done = [torch.cuda.Event() for _ in range(nbuf)]
    comp_done = [torch.cuda.Event() for _ in range(nbuf)]
    d2h_done = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_pipelined(i):
        b = i % nbuf
        with torch.cuda.stream(h2d):
            h2d.wait_event(comp_done[b])  # x_devs[b] no longer read by step i - nbuf
            x_devs[b].copy_(x_hosts[b], non_blocking=True)
            h2d_done[b].record(h2d)
        stream.wait_event(h2d_done[b])
        stream.wait_event(d2h_done[b])  # y_devs[b] already copied out by step i - nbuf
        moe.moe_forward(d, x_devs[b], inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, y_devs[b], ws,
                        W1_scales=inp.W1_scales, W2_scales=inp.W2_scales, stream=stream, W1_prepared=W1p,
                        W2_prepared=W2p)
        comp_done[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[b])
            y_hosts[b].copy_(y_devs[b], non_blocking=True)
            d2h_done[b].record(d2h)

    def e2e_serial(i):
        x_devs[0].copy_(x_hosts[0], non_blocking=True)
        moe.moe_forward(d, x_devs[0], inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, y_devs[0], ws,
                        W1_scales=inp.W1_scales, W2_scales=inp.W2_scales, W1_prepared=W1p, W2_prepared=W2p)
        y_hosts[0].copy_(y_devs[0], non_blocking=True)

    def time_loop(body):
        for i in range(max(1, args.warmup)):
            body(i)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            body(i)
        for b in range(nbuf):
            stream.wait_event(d2h_done[b])  # the last results are on the host
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    e2e_ms = time_loop(e2e_pipelined)
    e2e_serial_ms = time_loop(e2e_serial)

    elapsed_ms, e2e_ms, e2e_serial_ms, mlp1_ms = max_over_ranks(
        [elapsed_ms, e2e_ms, e2e_serial_ms, stage_ms["mlp1"]], world, dev)
    ms_per_step, value = step_throughput(elapsed_ms, args.steps, T, world)
    tokens_total = T * world
    tflops = shape.flops * world / (ms_per_step / 1e3) / 1e12

    pk, pk_kind = peaks()
    clocks = clk.summary()
    # the sustained (power-capped) peak when the timed region ran under the power cap
    capped = "sw_power_cap" in clocks["reasons"] or elapsed_ms >= 1000.0
    peak_key = "bf16_tflops_sustained" if capped else "bf16_tflops"
    peak_tf = float(pk.get(peak_key, FALLBACK_PEAKS[peak_key]))
    mlp1_flops = 4.0 * R * D * I
    wbytes = sum(t.numel() * t.element_size() for t in (inp.W1, inp.W2, inp.W1_scales, inp.W2_scales) if t is not None)
    roofline, stage_roofline = rooflines(shape, inp, stage_ms, mlp1_ms, peak_tf, pk, pk_kind, workload)
    counts_h = counts.cpu().tolist()
    routing = {"tokens_per_expert": counts_h, "min": min(counts_h), "max": max(counts_h),
               "experts_le8": sum(c <= 8 for c in counts_h), "experts_gt1000": sum(c > 1000 for c in counts_h),
               "tile_rows_128": sum(-(-c // 128) * 128 for c in counts_h), "rows": R}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, budget_s=args.cpu_budget, act=act_tuple(args))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; random-init weights of the layer shape)",
            "config": {"workload": WORKLOAD_NAMES[workload], "T": T, "D": D, "E": E, "k": k, "I": I,
                       "weights": shape.wfmt, "tokens_per_gpu": T, "parallelism": f"replicas x{world} (token-sharded, "
                       "no collective)", "l2": f"inputs larger than L2 (expert weights {wbytes / 1e9:.2f} GB per step)",
                       **({"mxfp4_weights": "prepared once before timing (moe_mxfp4_prepare)"} if mx else {}),
                       **act_config(args)},
            "tflops": tflops, "pct_of_bf16_peak": 100.0 * tflops / peak_tf, "peak_kind": f"{peak_key} ({pk_kind})",
            "stages_ms": stage_ms,
            "roofline": roofline,
            "stage_rooflines": stage_roofline,
            "routing": routing,
            "e2e": {"value": T * world / (e2e_ms / args.steps / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2,
                    "how": "moe_forward per step with its x H2D and y D2H copies in the timed region; copies on "
                           "their own streams, double-buffered, overlapping neighbouring steps' compute"},
            "e2e_serial": {"value": T * world / (e2e_serial_ms / args.steps / 1e3), "unit": UNIT,
                           "how": "same, copy-compute-copy serialised on one stream"},
            "gpu_launches": launches_per_step(T, D, mx, k) * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def cpu_baseline(inp, budget_s=15.0, step_tokens=None, act=(0, 1.0, float("inf"))):
    """The oracle as it stands, on the host cores, on a bounded token sample."""
    import oracle

    x = inp.x.cpu()
    Wr, br = inp.Wr.cpu(), inp.br.cpu()
    W1, b1, W2, b2 = inp.W1.cpu(), inp.b1.cpu(), inp.W2.cpu(), inp.b2.cpu()
    W1s = None if inp.W1_scales is None else inp.W1_scales.cpu()
    W2s = None if inp.W2_scales is None else inp.W2_scales.cpu()
    k = inp.shape.k
    T = x.shape[0]

    def run(n, seed):
        g = torch.Generator().manual_seed(seed)
        toks = torch.randperm(T, generator=g)[:n]
        xs = x[toks].contiguous()
        t0 = time.perf_counter()
        _, idx, w = oracle.route(xs, Wr, br, k)
        oracle.ffn_tokens(xs, idx, w, W1, b1, W2, b2, W1_scales=W1s, W2_scales=W2s, act=act)
        return time.perf_counter() - t0

    t1 = run(2, 0)
    n = step_tokens or max(2, min(T, int(budget_s / max(t1 / 2, 1e-6))))
    t = run(n, 1)
    return {"value": n / t, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {T} tokens of the same workload (route + top-k + softmax + expert FFN + combine per "
                      f"token, fp64 accumulate), {t:.1f} s"}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle

    shape = synthetic.SHAPES[args.workload]
    inp = synthetic.make_inputs(args.workload, seed=synthetic.SEEDS[args.workload], device="cpu")
    x, Wr, br = inp.x, inp.Wr, inp.br
    k, T = shape.k, shape.T
    per_step_s = max(1.0, args.ref_budget / max(1, args.steps + args.warmup))

    def one(n, seed):
        g = torch.Generator().manual_seed(seed)
        toks = torch.randperm(T, generator=g)[:n]
        xs = x[toks].contiguous()
        t0 = time.perf_counter()
        _, idx, w = oracle.route(xs, Wr, br, k)
        oracle.ffn_tokens(xs, idx, w, inp.W1, inp.b1, inp.W2, inp.b2, W1_scales=inp.W1_scales,
                          W2_scales=inp.W2_scales, act=act_tuple(args))
        return time.perf_counter() - t0

    t1 = one(2, 0)
    n = max(1, min(T, int(per_step_s / max(t1 / 2, 1e-6))))
    for i in range(args.warmup):
        one(n, 100 + i)
    total = 0.0
    for i in range(args.steps):
        total += one(n, 1000 + i)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD_NAMES[args.workload], "T": T, "D": shape.D, "E": shape.E, "k": k,
                   "I": shape.I, "weights": shape.wfmt, **act_config(args)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{n} of {T} tokens per step (route + FFN + combine per token)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_NAMES), default=WORKLOAD,
                    help="the bench line is the 20B shape; the others are for inspection")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--act", choices=["swiglu", "gptoss"], default="swiglu",
                    help="activation: plain SwiGLU (the benchmark's) or the GPT-OSS variant")
    ap.add_argument("--act-alpha", type=float, default=1.702, help="GPT-OSS variant: sigmoid slope (caller's choice)")
    ap.add_argument("--act-limit", type=float, default=7.0, help="GPT-OSS variant: clamp limit (caller's choice)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=120.0, help="seconds of oracle work for --impl reference")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
