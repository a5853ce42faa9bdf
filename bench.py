"""Benchmark of the fine-grained FP8 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl fg8|reference]

One step is one pass of the whole layer path over one batch: for every
linear of the workload, dynamic per-token activation quantization (1x128
groups) followed by the block-scaled FP8 GEMM with the bf16 epilogue.  The
default workload is the largest configuration that fits one GPU: 16384
tokens through the square 12288 -> 12288 layer with float scales (4.95
TFLOP per step), on synthetic seeded inputs.  Others: the ESM-2 35M-shaped
FFN (8 x 1022 = 8176 tokens, hidden 480 -> FFN 1920 -> 480, float scales,
both GEMMs back to back, no activation function between them), the
Llama-3-8B and DeepSeek-V3 projections, the rest of the square sweep and
the MoE experts.  When a workload has several layers they chain: the first GEMM's epilogue quantizes its bf16 output for
the second layer (the same bytes a separate act-quant launch writes), so a
step is act-quant, GEMM, GEMM; --no-chain gives each layer its own act-quant.

Rank 0 prints ONE JSON line.  `value` is whole-job TFLOP/s (2*M*N*K summed
over the step's GEMMs and all ranks, / the median device time of a step,
max over ranks); weak
scaling: every rank runs its own batch with replicated weights and there is
no collective on the data path (token rows are independent).

--impl reference times the CPU oracle on a bounded sample of the same
workload (rows of the batch), reporting the same metric.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "block-scaled FP8 linear TFLOP/s and % of B200 dense FP8 peak; act-quant GB/s"
# the largest configuration that fits one GPU: the square sweep's 16384 tokens,
# K = N = 12288 (4.95 TFLOP per step), with float scales (the exact promotion)
DEFAULT_WORKLOAD = "square_m16384_float"
L2_FLUSH_BYTES = 256 << 20
SMALL_M_MAX, SMALL_M_ALWAYS, FUSED_M_MAX = 128, 32, 16  # fg8_linear's few-token dispatch


def layer_path(g):
    """Which kernels fg8_linear runs for this shape (the library's rule):
    "fused" one few-token kernel that also quantizes x (UE8M0, M <= 16);
    "small" the prepare step, then the few-token swap-AB kernel;
    "tiled" the prepare step, then the tiled GEMM."""
    small = g.M <= SMALL_M_ALWAYS or (g.M <= SMALL_M_MAX and (g.N + 255) // 256 * 4 <= 148)
    if small and g.fmt == 1 and g.M <= FUSED_M_MAX:
        return "fused"
    return "small" if small else "tiled"
FP8_PER_BF16 = 2.0  # nominal dense fp8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)


# ------------------------------------------------------------ workloads ----
def workload_layers(name):
    """[(cfg, Gemm, stage)] of one step."""
    if name == "esm2_ffn":
        return [("esm2", W.ESM_W1, 1), ("esm2", W.ESM_W2, 2)]
    if name.startswith("llama_"):        # llama_m4096: gate/up then down
        M = int(name.split("_m")[1])
        return [("llama", W.llama(M, "gate_up"), 1), ("llama", W.llama(M, "down"), 2)]
    if name == "dsv3_mlp":
        return [("dsv3", W.DSV3_UP, 1), ("dsv3", W.DSV3_DOWN, 2)]
    if name.startswith("square_"):       # square_m8192_float / square_m8192_ue8m0
        _, m, f = name.split("_")
        return [("square", W.square(int(m[1:]), 1 if f == "ue8m0" else 0), 1)]
    raise SystemExit(f"unknown workload {name}")


def workload_config(name, layers, block=128):
    g0 = layers[0][1]
    cfg = {"workload": name, "tokens": g0.M, "layers": [[g.K, g.N] for _, g, _ in layers],
           "scale_fmt": "ue8m0" if g0.fmt else "float", "block": [block, block], "act_group": block,
           "l2": "flushed between steps (256 MiB write, then 256 MiB read, outside the step events)"}
    if name == "esm2_ffn":
        cfg.update({"model": "ESM-2 35M FFN shape (hidden 480, ffn 1920, 8 x 1022 tokens)"})
    return cfg


# ---------------------------------------------------------- distributed ----
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(value, world, device):
    """Max of a float over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, world, device):
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed loop runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, power, reasons = [], None, [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                s, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            sm.append(s)
            smax = mx
            try:
                power.append(float(parts[2]))
            except ValueError:  # power may read [N/A]; the clocks still count
                pass
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------ roofline ----
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "fine_grained_fp8_act_b200", "csrc")


def source_hash():
    """sha256 of the kernel sources: DRAM traffic recorded from ncu holds only
    for the kernels it was taken from."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload, launch):
    """DRAM bytes (read + write) of the workload's `launch`-th GEMM launch of a
    step, from profiles/traffic.json, or None when absent or stale."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != source_hash():
        return None
    v = rec.get("workloads", {}).get(workload, {}).get("gemm_dram_bytes", [])
    return v[launch] if launch < len(v) else None


def record_traffic(csv_path, workload):
    """Stores, per GEMM launch of one step (in launch order), the
    dram__bytes_read.sum + dram__bytes_write.sum of an ncu raw CSV export
    (`ncu -i report --page raw --csv`) of that step's GEMM launches."""
    import csv
    with open(csv_path) as f:
        rows = list(csv.reader(f))
    head = rows[0]
    body = [r for r in rows[1:] if len(r) == len(head) and r[0].strip() and r[0].strip()[0].isdigit()]
    col = {h: i for i, h in enumerate(head)}

    def val(r, name):
        txt = r[col[name]].replace(",", "")
        return float(txt)
    unit_row = rows[1]

    def scale(name):
        u = unit_row[col[name]].strip().lower()
        return {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(u, 1)
    out = []
    for r in body:
        if "fg8_gemm_kernel" not in r[col["Kernel Name"]] and "fg8_small_m_kernel" not in r[col["Kernel Name"]]:
            continue
        out.append(val(r, "dram__bytes_read.sum") * scale("dram__bytes_read.sum") +
                   val(r, "dram__bytes_write.sum") * scale("dram__bytes_write.sum"))
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        rec = {}
    if rec.get("source_hash") != source_hash():
        rec = {"source_hash": source_hash(), "workloads": {}}
    rec["workloads"][workload] = {"gemm_dram_bytes": out, "from": os.path.basename(csv_path)}
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec["workloads"][workload]))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def gemm_bytes(g):
    """Algorithmic HBM bytes of one GEMM launch: xq + x scales + Wq + W scales + y + bias."""
    Kb, Nb = -(-g.K // 128), -(-g.N // 128)
    sb = 4 if g.fmt == 0 else 1
    return g.M * g.K + g.M * Kb * sb + g.N * g.K + Nb * Kb * sb + 2 * g.M * g.N + 2 * g.N


def quant_bytes(g):
    """Algorithmic HBM bytes of one activation-quant launch: read bf16 x, write e4m3 + scales."""
    Kb = -(-g.K // 128)
    return 2 * g.M * g.K + g.M * g.K + g.M * Kb * (4 if g.fmt == 0 else 1)


def gemm_flops(g):
    return 2.0 * g.M * g.N * g.K


def weight_quant_bytes(g, block):
    """HBM bytes of quantizing one weight: bf16 read, e4m3 written, block scales written."""
    nb, kb = -(-g.N // block), -(-g.K // block)
    return 3 * g.N * g.K + nb * kb * (4 if g.fmt == 0 else 1)


def time_weight_quant(fg8, w, wq, ws, fmt, block, flush_l2, reps=10):
    """The one-time weight quantization (outside the step), timed after the
    step's measurement so the clocks are those of a loaded GPU: mean
    CUDA-event time in ms of `reps` launches of the C entry point into scratch
    copies of wq / ws on the current stream, L2 flushed before each (the
    flush's device time also covers the host's enqueue of the launch)."""
    stream = torch.cuda.current_stream(w.device)
    wq_t, ws_t = torch.empty_like(wq), torch.empty_like(ws)
    N, K = w.shape
    evs = []
    for _ in range(reps):
        flush_l2()
        e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        e[0].record(stream)
        fg8.fg8_quantize_weight_block(w.data_ptr(), N, K, w.stride(0), wq_t.data_ptr(), ws_t.data_ptr(), fmt, block,
                                      stream.cuda_stream)
        e[1].record(stream)
        evs.append(e)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


# ------------------------------------------------------------ fg8 arm ----
def run_fg8(args, rank, world, local):
    import fine_grained_fp8_act_b200 as fg8
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    layers = workload_layers(args.workload)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    # weights (replicated), quantized once on the device
    plan = []
    x0 = None
    for i, (cfg, g, stage) in enumerate(layers):
        x, w, b = W.make_inputs(cfg, g, device=dev, stage=stage)
        if i == 0:
            # weak scaling: every rank runs its own batch of the same shape
            x0 = x if rank == 0 else x.roll(rank, 0).contiguous()
        wq, ws = fg8.quantize_weight(w, g.fmt, block=args.block)
        wsp = torch.zeros(fg8.fg8_linear_block_workspace_bytes(g.M, g.N, g.K, g.fmt, args.block), dtype=torch.uint8,
                          device=dev)
        y = torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev)
        plan.append(dict(g=g, wq=wq, ws=ws, b=b, wsp=wsp, y=y, w=w))  # w: the weight-quant timing below
    for i, L in enumerate(plan):
        L["x"] = x0 if i == 0 else plan[i - 1]["y"]
        assert L["x"].shape == (L["g"].M, L["g"].K), "consecutive layers must chain"

    # Each layer runs what fg8_linear runs for its shape: few tokens take the
    # swap-AB split-K kernel (after the prepare step, or with the
    # quantization fused in), more take the tiled GEMM.  When every layer is
    # tiled, consecutive layers chain: the GEMM of layer i also quantizes its
    # output for layer i+1 (fg8_linear_run_chain), so layer i+1 has no
    # act-quant launch.
    # block 32 / 64 (1 x b groups, b x b weight blocks): fg8_linear_block per layer
    paths = [("small_block" if args.block != 128 else layer_path(L["g"])) for L in plan]
    chain = not args.no_chain and len(plan) > 1 and all(pth == "tiled" for pth in paths)
    # --fused-quant: a tiled layer with K <= 4096 whose input is not already
    # quantized by the previous GEMM takes fg8_linear_fused, its act-quant
    # inside the GEMM's launch (in-kernel units published with flags).
    for i, L in enumerate(plan):
        if paths[i] == "tiled" and args.fused_quant and -(-L["g"].K // 128) <= 32 and (i == 0 or not chain):
            paths[i] = "tiled_fused_quant"
            g = L["g"]
            L["wsp"] = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(g.M, g.N, g.K, g.fmt), dtype=torch.uint8,
                                   device=dev)

    def launch_layer(i, ev_mid=None):
        L = plan[i]
        g = L["g"]
        if paths[i] == "small_block":  # act-quant, scale packing and GEMM in one call
            if ev_mid is not None:
                ev_mid.record(stream)
            fg8.fg8_linear_block(L["x"].data_ptr(), g.M, g.N, g.K, L["x"].stride(0), L["wq"].data_ptr(),
                                 L["ws"].data_ptr(), L["b"].data_ptr(), L["y"].data_ptr(), L["y"].stride(0), g.fmt,
                                 args.block,
                                 L["wsp"].data_ptr(), L["wsp"].numel(), sp)
            return
        if paths[i] == "tiled_fused_quant":  # act-quant inside the GEMM's launch (+ the next layer's requant)
            if ev_mid is not None:
                ev_mid.record(stream)
            nxt = plan[i + 1] if chain and i + 1 < len(plan) else None
            fg8.fg8_linear_fused(L["x"].data_ptr(), g.M, g.N, g.K, L["x"].stride(0), L["wq"].data_ptr(),
                                 L["ws"].data_ptr(), L["b"].data_ptr(), L["y"].data_ptr(), L["y"].stride(0), g.fmt,
                                 L["wsp"].data_ptr(), L["wsp"].numel(), 0 if nxt is None else nxt["g"].N,
                                 None if nxt is None else nxt["ws"].data_ptr(),
                                 None if nxt is None else nxt["wsp"].data_ptr(),
                                 0 if nxt is None else nxt["wsp"].numel(), sp)
            return
        if paths[i] == "fused":
            if ev_mid is not None:
                ev_mid.record(stream)
            fg8.fg8_linear(L["x"].data_ptr(), g.M, g.N, g.K, L["x"].stride(0), L["wq"].data_ptr(), L["ws"].data_ptr(),
                           L["b"].data_ptr(), L["y"].data_ptr(), L["y"].stride(0), g.fmt, L["wsp"].data_ptr(),
                           L["wsp"].numel(), sp)
            return
        if i == 0 or not chain:
            fg8.fg8_linear_prepare(L["x"].data_ptr(), g.M, g.N, g.K, L["x"].stride(0), L["ws"].data_ptr(), g.fmt,
                                   L["wsp"].data_ptr(), L["wsp"].numel(), sp)
        if ev_mid is not None:
            ev_mid.record(stream)
        if chain and i + 1 < len(plan):
            Ln = plan[i + 1]
            fg8.fg8_linear_run_chain(L["wq"].data_ptr(), L["ws"].data_ptr(), L["b"].data_ptr(), L["y"].data_ptr(),
                                     g.M, g.N, g.K, L["y"].stride(0), g.fmt, L["wsp"].data_ptr(), L["wsp"].numel(),
                                     Ln["g"].N, Ln["ws"].data_ptr(), Ln["wsp"].data_ptr(), Ln["wsp"].numel(), sp)
        else:
            fg8.fg8_linear_run(L["wq"].data_ptr(), L["ws"].data_ptr(), L["b"].data_ptr(), L["y"].data_ptr(), g.M,
                               g.N, g.K, L["y"].stride(0), g.fmt, L["wsp"].data_ptr(), L["wsp"].numel(), sp)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer larger than L2, then read another one: L2 ends up
        # holding clean lines, so no write-back of the flush lands in the step
        flush.zero_()
        flush_rd.sum()
    nl = len(plan)
    # Timed steps carry events only at their two ends, so consecutive kernels
    # keep their programmatic-launch overlap.  A second pass, with events
    # between the kernels, gives each kernel's own duration (roofline).
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    n_prof = max(3, min(args.steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(1 + 2 * nl)] for _ in range(n_prof)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        for i in range(nl):
            launch_layer(i, None if e is None else e[1 + 2 * i])
            if e is not None:
                e[2 + 2 * i].record(stream)

    def timed_step(pair):
        pair[0].record(stream)
        for i in range(nl):
            launch_layer(i)
        pair[1].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    for L in plan:
        st = fg8.fg8_check_device_status(L["wsp"].data_ptr(), sp)
        if st != 0:
            raise RuntimeError(f"device status {st} after warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2()
        timed_step(step_ev[k])
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    time.sleep(0.25)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    step_med = statistics.median(step_ms)

    # per-kernel pass (same kernels, events between them)
    for k in range(n_prof):
        flush_l2()
        step(evs[k])
    torch.cuda.synchronize()
    quant_ms = [[e[2 * i].elapsed_time(e[1 + 2 * i]) for e in evs] for i in range(nl)]
    for L in plan:
        L["wq_ms"] = time_weight_quant(fg8, L["w"], L["wq"], L["ws"], L["g"].fmt, args.block, flush_l2)
        del L["w"]
    gemm_ms = [[e[1 + 2 * i].elapsed_time(e[2 + 2 * i]) for e in evs] for i in range(nl)]
    # the step time is the median over the timed steps, the job's the slowest
    # rank's; the mean is reported beside it
    med_max = max_over_ranks(step_med, world, dev)
    mean_max = max_over_ranks(sum(step_ms) / len(step_ms), world, dev)
    flops_step = sum(gemm_flops(L["g"]) for L in plan)
    flops_all = sum_over_ranks(flops_step, world, dev)
    tflops = flops_all / (med_max * 1e-3) / 1e12

    peaks = measured_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    # per-kernel roofline: the dominant kernel is the GEMM launch with the largest median time
    gm = [statistics.median(v) for v in gemm_ms]
    qm = [statistics.median(v) for v in quant_ms]
    dom = max(range(nl), key=lambda i: gm[i])
    g = plan[dom]["g"]
    t_s = gm[dom] * 1e-3
    t_tensor = gemm_flops(g) / (fp8_peak * 1e12)
    t_hbm = gemm_bytes(g) / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": gemm_flops(g) / t_s / 1e12, "peak": fp8_peak, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": gemm_bytes(g) / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(args.workload, dom)  # ncu DRAM bytes per launch, None if stale
    roof["kernel"] = (f"fg8_gemm_kernel, {args.block} x {args.block} blocks, timed with its act-quant "
                      f"and scale packing" if paths[dom] == "small_block" else
                      "fg8_small_m_kernel" if paths[dom] not in ("tiled", "tiled_fused_quant") else
                      "fg8_gemm_kernel") + f" ({g.name}: M={g.M} K={g.K} N={g.N})" + (
        ", act-quant of x inside the launch" if paths[dom] == "tiled_fused_quant" else "") + (
        ", epilogue also quantizes y for the next layer" if chain and dom + 1 < nl else "")
    roof["kernel_us"] = gm[dom] * 1e3
    roof["peak_source"] = (f"{peaks['source']}: bf16 {peaks['bf16_tflops']} TF/s x {FP8_PER_BF16} (fp8:bf16 nominal), "
                           f"HBM {peaks['hbm_gbs']} GB/s")
    roof["timing"] = (f"kernel alone: median of CUDA events around each launch over {n_prof} flushed steps "
                      f"(no programmatic-launch overlap with its neighbours)")
    per_kernel = []
    for i, L in enumerate(plan):
        gi = L["g"]
        fused = paths[i] in ("fused", "small_block", "tiled_fused_quant") or (chain and i > 0)  # not timed alone
        per_kernel.append({"layer": gi.name, "path": paths[i], "act_quant_us": None if fused else qm[i] * 1e3,
                           "act_quant_gbs": None if fused else quant_bytes(gi) / (qm[i] * 1e-3) / 1e9,
                           "act_quant": ("fused into the few-token kernel" if paths[i] == "fused" else
                                         "inside the GEMM's launch (fg8_linear_fused)"
                                         if paths[i] == "tiled_fused_quant" else
                                         "timed with the GEMM (fg8_linear_block: act-quant, scale packing, GEMM)"
                                         if paths[i] == "small_block" else
                                         "fused into the previous GEMM" if fused else "own launch"),
                           "gemm_us": gm[i] * 1e3, "gemm_tflops": gemm_flops(gi) / (gm[i] * 1e-3) / 1e12,
                           "gemm_pct_fp8_peak": 100.0 * gemm_flops(gi) / (gm[i] * 1e-3) / 1e12 / fp8_peak,
                           # one-time, on load (not in the step): the weight's own quantization launch
                           "weight_quant_us": L["wq_ms"] * 1e3,
                           "weight_quant_gbs": weight_quant_bytes(gi, args.block) / (L["wq_ms"] * 1e-3) / 1e9})

    e2e = run_e2e(fg8, plan, args, stream, dev, world, chain, paths)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, budget_s=args.cpu_seconds, block=args.block)

    # prepare: act-quant (+ the weight-scale packing launch for UE8M0), then the GEMM;
    # fused few-token layers and act-quant inside the GEMM: one kernel
    prep = [0 if pth in ("fused", "tiled_fused_quant") else 1 + (1 if L["g"].fmt == 1 else 0)
            for pth, L in zip(paths, plan)]
    launches_per_step = (prep[0] if chain else sum(prep)) + nl
    out = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": med_max, "ms_per_step_mean": mean_max,
        "step_time": "median over the timed steps (max over ranks)", "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate)", "data": "synthetic",
        "config": dense_arm_config(args.workload, [(c, L["g"], s) for (c, _, s), L in zip(layers, plan)],
                                   args.block, world),
        "pct_fp8_peak": 100.0 * tflops / world / fp8_peak,
        "act_quant_gbs": [k["act_quant_gbs"] for k in per_kernel if k["act_quant_gbs"] is not None],
        "chained": chain,
        "per_kernel": per_kernel,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s": wall,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def host_link_ms(h2d_pairs, d2h_pairs, h2d, d2h, stream, steps, world, dev):
    """Per-step time of an end-to-end leg's host copies alone, with no kernels:
    the same buffers and bytes each way, both directions at once on their own
    streams.  This is the host link's bound for the end-to-end number (on the
    B200 boxes the two directions share the link: about 55 GB/s one way
    alone, 47 GB/s each way together)."""
    def copies():
        with torch.cuda.stream(h2d):
            for src, dst in h2d_pairs:
                dst.copy_(src, non_blocking=True)
        with torch.cuda.stream(d2h):
            for src, dst in d2h_pairs:
                dst.copy_(src, non_blocking=True)

    copies()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_event(e0)
    d2h.wait_event(e0)
    for _ in range(steps):
        copies()
    stream.wait_stream(h2d)
    stream.wait_stream(d2h)
    e1.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world, dev) / steps


def run_e2e(fg8, plan, args, stream, dev, world, chain, paths):
    """Same metric through the public calls with host buffers, as a serving
    loop runs it: every step copies its input from pinned host memory to the
    device, runs the layers (chained as in the device-timed step, else
    fg8_linear per layer) and copies its output back to pinned host memory,
    all inside the timed region.  The copies go on their own streams, so a
    step's input copy and the previous step's output copy overlap the
    kernels; two device buffers each for the input and the output, ordered
    by events, keep a copy from touching a buffer still in use."""
    L0, Ln = plan[0], plan[-1]
    slots = 2
    x_host = L0["x"].to("cpu").pin_memory()
    y_host = [torch.empty(Ln["y"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    x_dev = [torch.empty_like(L0["x"]) for _ in range(slots)]
    y_dev = [torch.empty_like(Ln["y"]) for _ in range(slots)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(slots)]     # x_dev[s] holds the step's input
    ev_done = [torch.cuda.Event() for _ in range(slots)]   # the step's kernels are done with x_dev[s], y_dev[s] written
    ev_out = [torch.cuda.Event() for _ in range(slots)]    # y_dev[s] has been copied out
    sp = stream.cuda_stream
    steps = max(3, min(args.steps, 50))

    def fused_layer(L, xin, y, nxt):
        g = L["g"]
        fg8.fg8_linear_fused(xin.data_ptr(), g.M, g.N, g.K, xin.stride(0), L["wq"].data_ptr(), L["ws"].data_ptr(),
                             L["b"].data_ptr(), y.data_ptr(), y.stride(0), g.fmt, L["wsp"].data_ptr(),
                             L["wsp"].numel(), 0 if nxt is None else nxt["g"].N,
                             None if nxt is None else nxt["ws"].data_ptr(),
                             None if nxt is None else nxt["wsp"].data_ptr(), 0 if nxt is None else nxt["wsp"].numel(),
                             sp)

    def layers(xin, yout):
        if chain:
            g = L0["g"]
            if paths[0] != "tiled_fused_quant":
                fg8.fg8_linear_prepare(xin.data_ptr(), g.M, g.N, g.K, xin.stride(0), L0["ws"].data_ptr(), g.fmt,
                                       L0["wsp"].data_ptr(), L0["wsp"].numel(), sp)
            for i, L in enumerate(plan):
                g = L["g"]
                y = yout if i + 1 == len(plan) else L["y"]
                if i == 0 and paths[0] == "tiled_fused_quant":
                    fused_layer(L, xin, y, plan[1] if len(plan) > 1 else None)
                elif i + 1 < len(plan):
                    Lx = plan[i + 1]
                    fg8.fg8_linear_run_chain(L["wq"].data_ptr(), L["ws"].data_ptr(), L["b"].data_ptr(),
                                             y.data_ptr(), g.M, g.N, g.K, y.stride(0), g.fmt,
                                             L["wsp"].data_ptr(), L["wsp"].numel(), Lx["g"].N, Lx["ws"].data_ptr(),
                                             Lx["wsp"].data_ptr(), Lx["wsp"].numel(), sp)
                else:
                    fg8.fg8_linear_run(L["wq"].data_ptr(), L["ws"].data_ptr(), L["b"].data_ptr(), y.data_ptr(),
                                       g.M, g.N, g.K, y.stride(0), g.fmt, L["wsp"].data_ptr(), L["wsp"].numel(), sp)
        else:
            for i, L in enumerate(plan):
                g = L["g"]
                y = yout if i + 1 == len(plan) else L["y"]
                if paths[i] == "tiled_fused_quant":
                    fused_layer(L, xin, y, None)
                    xin = y
                    continue
                fg8.fg8_linear_block(xin.data_ptr(), g.M, g.N, g.K, xin.stride(0), L["wq"].data_ptr(),
                                     L["ws"].data_ptr(), L["b"].data_ptr(), y.data_ptr(), y.stride(0), g.fmt,
                                     args.block, L["wsp"].data_ptr(), L["wsp"].numel(), sp)
                xin = y

    def one(k, start=None):
        s = k % slots
        with torch.cuda.stream(h2d):
            if start is not None:
                h2d.wait_event(start)
            h2d.wait_event(ev_done[s])           # the step two back has finished reading x_dev[s]
            x_dev[s].copy_(x_host, non_blocking=True)
            ev_in[s].record(h2d)
        stream.wait_event(ev_in[s])
        stream.wait_event(ev_out[s])             # y_dev[s] of the step two back has been copied out
        layers(x_dev[s], y_dev[s])
        ev_done[s].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[s])
            y_host[s].copy_(y_dev[s], non_blocking=True)
            ev_out[s].record(d2h)

    for k in range(3):
        one(k)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(steps):
        one(k, e0 if k == 0 else None)
    stream.wait_event(ev_out[(steps - 1) % slots])  # the last output is on the host (the d2h stream is in order)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    flops = sum_over_ranks(sum(gemm_flops(L["g"]) for L in plan) * steps, world, dev)
    link = host_link_ms([(x_host, x_dev[0])], [(y_dev[0], y_host[0])], h2d, d2h, stream, steps, world, dev)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": y_host[0].numel() * 2,
            "steps": steps, "ms_per_step": ms / steps,
            "host_link_ms_per_step": link, "frac_of_host_link": link / (ms / steps),
            "overlap": "input and output copies on their own streams, overlapping the neighbouring steps' kernels"}


# ---------------------------------------------------- MoE experts (fg8) ----
def moe_shapes():
    """[(name, K, N)] of the routed-expert layers: gate/up, then down."""
    c = W.DSV3_MOE
    return [("moe_dsv3_gate_up", c["hidden"], 2 * c["inter"]), ("moe_dsv3_down", c["inter"], c["hidden"])]


def moe_config(rows_routed, rows_padded):
    c = W.DSV3_MOE
    return {"workload": "moe_dsv3", "model": "DeepSeek-V3-shaped routed experts (hidden 7168, expert "
            "intermediate 2048, 256 experts, top-8), synthetic routing: log-normal expert popularity, sigma "
            f"{c['skew']}",
            "tokens": c["tokens"], "experts": c["experts"], "topk": c["topk"], "rows_routed": rows_routed,
            "rows_padded": rows_padded, "layers": [[K, N] for _, K, N in moe_shapes()], "scale_fmt": "ue8m0",
            "block": [128, 128], "act_group": 128, "layout": "contiguous grouped, expert runs padded to 128 rows",
            "l2": "flushed between steps (256 MiB write, then 256 MiB read, outside the step events)"}


def dense_arm_config(workload, layers, block, world):
    """The `config` of a dense workload's line, the same on both arms."""
    return dict(workload_config(workload, layers, block),
                parallelism=f"dp{world} (token rows, replicated weights, no collective)")


def moe_layout():
    """The seeded routing of the MoE workload: (row_token, row_expert, padded rows, routed rows)."""
    c = W.DSV3_MOE
    rt, re = W.moe_routing(c["tokens"], c["experts"], c["topk"], seed=5, skew=c["skew"])
    return rt, re, int(re.numel()), c["tokens"] * c["topk"]


def moe_arm_config(world):
    """The `config` of the MoE workload's line, the same on both arms."""
    _, _, Mp, routed = moe_layout()
    return dict(moe_config(routed, Mp), parallelism=f"dp{world} (token rows, replicated experts, no collective)")


def run_moe(args, rank, world, local):
    """The MoE expert layers through fg8_grouped_linear (prepare + grouped GEMM per
    layer).  TFLOP/s count the routed rows only (padding rows are work done but
    not counted)."""
    import fine_grained_fp8_act_b200 as fg8
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    c = W.DSV3_MOE
    T, E, topk, fmt = c["tokens"], c["experts"], c["topk"], 1
    rt, re, Mp, routed = moe_layout()
    re_d = re.to(dev)
    plan = []
    for i, (name, K, N) in enumerate(moe_shapes()):
        xt = W.x_student_t(T, K, seed=50 + i, device=dev)
        if rank:
            xt = xt.roll(rank, 0).contiguous()
        x = W.gather_rows(xt, rt)
        del xt
        wq = ws = None
        for e in range(E):  # one expert at a time: the bf16 stack would need twice the e4m3 bytes
            q, sc = fg8.quantize_weight(W.w_row_groups(N, K, 0.015, seed=1000 * (i + 1) + e, device=dev), fmt)
            if wq is None:  # the dtypes quantize_weight returns, so that the stores below copy bits
                wq = torch.empty((E,) + tuple(q.shape), dtype=q.dtype, device=dev)
                ws = torch.empty((E,) + tuple(sc.shape), dtype=sc.dtype, device=dev)
            wq[e] = q
            ws[e] = sc
        nb = fg8.fg8_grouped_linear_workspace_bytes(Mp, E, N, K, fmt)
        plan.append(dict(name=name, K=K, N=N, x=x, wq=wq, ws=ws, wsp=torch.zeros(nb, dtype=torch.uint8, device=dev),
                         y=torch.empty(Mp, N, dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()

    def prep(L):
        fg8.fg8_grouped_linear_prepare(L["x"].data_ptr(), Mp, L["K"], L["K"], E, L["N"], L["ws"].data_ptr(), fmt,
                                       L["wsp"].data_ptr(), L["wsp"].numel(), sp)

    def run(L):
        fg8.fg8_grouped_linear_run(re_d.data_ptr(), E, L["wq"].data_ptr(), L["ws"].data_ptr(), None,
                                   L["y"].data_ptr(), Mp, L["N"], L["K"], L["N"], fmt, L["wsp"].data_ptr(),
                                   L["wsp"].numel(), sp)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    for _ in range(args.warmup):
        flush_l2()
        for L in plan:
            prep(L)
            run(L)
    torch.cuda.synchronize()
    for L in plan:
        if fg8.fg8_check_device_status(L["wsp"].data_ptr(), sp) != 0:
            raise RuntimeError("device status after warm-up")
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2()
        step_ev[k][0].record(stream)
        for L in plan:
            prep(L)
            run(L)
        step_ev[k][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    time.sleep(0.25)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    med_max = max_over_ranks(statistics.median(step_ms), world, dev)
    mean_max = max_over_ranks(sum(step_ms) / len(step_ms), world, dev)
    flops_step = sum(2.0 * routed * L["N"] * L["K"] for L in plan)
    tflops = sum_over_ranks(flops_step, world, dev) / (med_max * 1e-3) / 1e12

    # per-kernel pass: events around each layer's prepare and grouped GEMM
    n_prof = max(3, min(args.steps, 20))
    pm = [[] for _ in plan]
    gm = [[] for _ in plan]
    for _ in range(n_prof):
        flush_l2()
        for i, L in enumerate(plan):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            prep(L)
            e[1].record(stream)
            run(L)
            e[2].record(stream)
            pm[i].append(e)
            gm[i].append(e)
    torch.cuda.synchronize()
    pm = [statistics.median(e[0].elapsed_time(e[1]) for e in v) for v in pm]
    gm = [statistics.median(e[1].elapsed_time(e[2]) for e in v) for v in gm]
    peaks = measured_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    dom = max(range(len(plan)), key=lambda i: gm[i])
    L = plan[dom]
    t_s = gm[dom] * 1e-3
    Kb, Nb = -(-L["K"] // 128), -(-L["N"] // 128)
    # every expert's weights once, the routed layout's codes, scales and output
    moe_bytes = E * L["N"] * L["K"] + E * Nb * Kb + Mp * L["K"] + Mp * Kb + 2 * Mp * L["N"]
    moe_flops = 2.0 * Mp * L["N"] * L["K"]  # the tensor cores run the padding rows too
    if moe_flops / (fp8_peak * 1e12) >= moe_bytes / (peaks["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": moe_flops / t_s / 1e12, "peak": fp8_peak, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": moe_bytes / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof.update({"frac": roof["achieved"] / roof["peak"], "traffic": recorded_traffic("moe_dsv3", dom),
                 "kernel": f"fg8_gemm_kernel, grouped ({L['name']}: {Mp} rows of which {routed} routed, "
                           f"K={L['K']} N={L['N']}, {E} experts)",
                 "kernel_us": gm[dom] * 1e3,
                 "algorithmic": (f"{moe_bytes / 1e9:.3f} GB per launch (all experts' e4m3 weights + scales, the "
                                 f"routed layout's e4m3 codes + scales, bf16 y); {moe_flops / 1e12:.3f} TFLOP "
                                 f"(padded rows)"),
                 "routed_tflops": 2.0 * routed * L["N"] * L["K"] / t_s / 1e12,
                 "peak_source": (f"{peaks['source']}: bf16 {peaks['bf16_tflops']} TF/s x {FP8_PER_BF16} (fp8:bf16 "
                                 f"nominal), HBM {peaks['hbm_gbs']} GB/s"),
                 "timing": f"kernel alone: CUDA events around each launch over {n_prof} flushed steps"})
    per_kernel = [{"layer": L["name"], "path": "grouped", "prepare_us": pm[i] * 1e3,
                   "act_quant_gbs": (3 * Mp * L["K"] + Mp * (-(-L["K"] // 128))) / (pm[i] * 1e-3) / 1e9,
                   "gemm_us": gm[i] * 1e3,
                   "gemm_tflops": 2.0 * routed * L["N"] * L["K"] / (gm[i] * 1e-3) / 1e12}
                  for i, L in enumerate(plan)]

    # end to end: routed rows and the expert index in from pinned host memory,
    # both layers, the last layer's rows out.  As in the dense leg, the copies
    # run on their own streams (a step's input copy and the previous step's
    # output copy overlap the kernels) with two device slots ordered by events.
    slots = 2
    xh = [L["x"].to("cpu").pin_memory() for L in plan]
    reh = re.pin_memory()
    yh = [torch.empty(plan[-1]["y"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    xd = [[torch.empty_like(L["x"]) for L in plan] for _ in range(slots)]
    red = [torch.empty_like(re_d) for _ in range(slots)]
    yd = [torch.empty_like(plan[-1]["y"]) for _ in range(slots)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(slots)]    # slot s holds the step's inputs
    ev_done = [torch.cuda.Event() for _ in range(slots)]  # the step's kernels are done with slot s
    ev_out = [torch.cuda.Event() for _ in range(slots)]   # yd[s] has been copied out
    e2e_steps = max(3, min(args.steps, 20))

    def one(k, start=None):
        s = k % slots
        with torch.cuda.stream(h2d):
            if start is not None:
                h2d.wait_event(start)
            h2d.wait_event(ev_done[s])  # the step two back has finished reading slot s
            red[s].copy_(reh, non_blocking=True)
            for a, b in zip(xh, xd[s]):
                b.copy_(a, non_blocking=True)
            ev_in[s].record(h2d)
        stream.wait_event(ev_in[s])
        stream.wait_event(ev_out[s])    # yd[s] of the step two back has been copied out
        for i, (L, b) in enumerate(zip(plan, xd[s])):
            y = yd[s] if i + 1 == len(plan) else L["y"]
            fg8.fg8_grouped_linear(b.data_ptr(), Mp, L["K"], L["K"], red[s].data_ptr(), E, L["N"], L["wq"].data_ptr(),
                                   L["ws"].data_ptr(), None, y.data_ptr(), L["N"], fmt, L["wsp"].data_ptr(),
                                   L["wsp"].numel(), sp)
        ev_done[s].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[s])
            yh[s].copy_(yd[s], non_blocking=True)
            ev_out[s].record(d2h)

    for k in range(3):
        one(k)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(e2e_steps):
        one(k, e0 if k == 0 else None)
    stream.wait_event(ev_out[(e2e_steps - 1) % slots])  # the last output is on the host (d2h runs in order)
    e1.record(stream)
    torch.cuda.synchronize()
    ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
    link = host_link_ms(list(zip(xh + [reh], xd[0] + [red[0]])), [(yd[0], yh[0])], h2d, d2h, stream, e2e_steps,
                        world, dev)
    e2e = {"value": sum_over_ranks(flops_step * e2e_steps, world, dev) / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": sum(a.numel() * 2 for a in xh) + reh.numel() * 4,
           "d2h_bytes_per_step": yh[0].numel() * 2, "steps": e2e_steps, "ms_per_step": ems / e2e_steps,
           "host_link_ms_per_step": link, "frac_of_host_link": link / (ems / e2e_steps),
           "overlap": "input and output copies on their own streams, overlapping the neighbouring steps' kernels"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_moe(budget_s=args.cpu_seconds)
    out = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": med_max, "ms_per_step_mean": mean_max,
        "step_time": "median over the timed steps (max over ranks)", "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate)", "data": "synthetic",
        "config": moe_arm_config(world),
        "pct_fp8_peak": 100.0 * tflops / world / fp8_peak,
        "per_kernel": per_kernel, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": 3 * len(plan) * args.steps,  # act-quant, scale packing, grouped GEMM per layer
        "clocks": clk, "wall_s": wall,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def threads_note(rows, threads):
    """The oracle's GEMM spreads sampled rows over its threads: say so when some stay idle there."""
    return "" if rows >= threads else f"; the GEMM keeps {rows} of the {threads} threads busy"


def oracle_moe_sample():
    """Inputs of the CPU oracle's MoE sample, built once: the first expert block's
    routed rows of each expert layer and that expert's quantized weights.
    Returns (run, expert): run(R) times the oracle's grouped layer on the first
    R rows (R <= 128) of both layers and returns (seconds, FLOPs)."""
    import oracle
    c = W.DSV3_MOE
    rt, re, _, _ = moe_layout()
    e0 = int(re[0])
    ops = []
    for i, (name, K, N) in enumerate(moe_shapes()):
        xt = W.x_student_t(c["tokens"], K, seed=50 + i)
        x = W.bf16_bits(W.gather_rows(xt, rt[:128]))
        wq, ws = oracle.quantize_weight(W.bf16_bits(W.w_row_groups(N, K, 0.015, seed=1000 * (i + 1) + e0)), 1)
        ops.append((K, N, x, wq[None], ws[None]))
    rexp = np.zeros(128, dtype=np.int32)  # the block's expert, renumbered 0 in the one-expert table

    def run(R):
        t0 = time.perf_counter()
        for K, N, x, wq, ws in ops:
            oracle.grouped_linear(x[:R], rexp[:R], wq, ws, None, 1)
        return time.perf_counter() - t0, sum(2.0 * R * N * K for K, N, _, _, _ in ops)

    return run, e0


def cpu_baseline_moe(budget_s=15.0, rows=None):
    """The CPU oracle's grouped layer, as it stands, on the first R rows of the
    routed layout (all in the first expert block) of each expert layer; weights
    of that block's expert quantized outside the timing.  TFLOP/s of those rows."""
    import oracle
    run, e0 = oracle_moe_sample()
    if rows is None:
        t, _ = run(2)
        rows = int(max(2, min(128, 2 * budget_s / max(t, 1e-6))))
    t, flops = run(rows)
    nt = oracle.num_threads()
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
            "sample": f"first {rows} routed rows (expert {e0}) through both expert layers ({t:.1f} s; weights "
                      f"quantized outside the timing{threads_note(rows, nt)})", "seconds": t, "rows": rows}


# ------------------------------------------------------ oracle (CPU) arm ----
def oracle_dense_sample(workload, block=128):
    """Inputs of the CPU oracle's sample of a dense workload, built once (the
    batch's bf16 rows, every layer's quantized weights and bias).  run(R) times
    the first R token rows through every layer (quantize, dequantized double
    GEMM, bf16 out) and returns (seconds, FLOPs)."""
    import oracle
    layers = workload_layers(workload)
    ops = []
    xb = None
    for i, (cfg, g, stage) in enumerate(layers):
        x, w, b = W.make_inputs(cfg, g, device="cpu", stage=stage)
        if i == 0:
            xb = W.bf16_bits(x)
        wq, ws = oracle.quantize_weight(W.bf16_bits(w), g.fmt, block)
        ops.append((g, wq, ws, W.bf16_bits(b)))

    def run(R):
        t0 = time.perf_counter()
        a = xb[:R]
        for g, wq, ws, bb in ops:
            _, _, ybf = oracle.linear(a, wq, ws, bb, g.fmt, block=block)
            a = ybf
        return time.perf_counter() - t0, sum(2.0 * R * g.N * g.K for g, _, _, _ in ops)

    return run


def cpu_baseline(workload, budget_s=15.0, rows=None, block=128):
    """The CPU oracle, as it stands, on a bounded sample of the workload: the
    first R token rows of the batch through every layer, weights quantized once
    outside the timing.  Reported in TFLOP/s of the sampled rows."""
    import oracle
    layers = workload_layers(workload)
    run = oracle_dense_sample(workload, block)
    if rows is None:
        probe = 16
        t, _ = run(probe)
        rows = int(max(16, min(layers[0][1].M, probe * budget_s / max(t, 1e-6))))
    t, flops = run(rows)
    nt = oracle.num_threads()
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
            "sample": f"first {rows} of {layers[0][1].M} token rows through all {len(layers)} layers "
                      f"({t:.1f} s; weights quantized outside the timing{threads_note(rows, nt)})",
            "seconds": t, "rows": rows}


def run_reference_moe(args, world):
    import oracle
    run, _ = oracle_moe_sample()
    # size each step so warm-up + steps take about --ref-seconds (2 minutes by default)
    budget = max(0.05, args.ref_seconds / max(1, args.steps + args.warmup))
    t_probe, _ = run(2)
    rows = int(max(1, min(128, 2 * budget / max(t_probe, 1e-6))))
    for _ in range(args.warmup):
        run(rows)
    ts = [run(rows)[0] for _ in range(args.steps)]
    flops = sum(2.0 * rows * N * K for _, K, N in moe_shapes())
    value = flops * len(ts) / sum(ts) / 1e12
    nt = oracle.num_threads()
    cpu = {"value": value, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
           "sample": f"first {rows} routed rows through both expert layers per step on the host cores of "
                     f"rank 0{threads_note(rows, nt)}"}
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * sum(ts) / len(ts), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle: float32 quantization, double GEMM)",
           "data": "synthetic", "impl": "reference",
           "config": moe_arm_config(world),
           "cpu_baseline": cpu,
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference(args, rank, world):
    if rank != 0:
        return
    if args.workload.startswith("moe_"):
        run_reference_moe(args, world)
        return
    import oracle
    layers = workload_layers(args.workload)
    run = oracle_dense_sample(args.workload, args.block)
    # size each step so warm-up + steps take about --ref-seconds (2 minutes by default)
    budget = max(0.05, args.ref_seconds / max(1, args.steps + args.warmup))
    t_probe, _ = run(16)
    rows = int(max(1, min(layers[0][1].M, 16 * budget / max(t_probe, 1e-6))))
    for _ in range(args.warmup):
        run(rows)
    ts = [run(rows)[0] for _ in range(args.steps)]
    flops = sum(2.0 * rows * g.N * g.K for _, g, _ in layers)
    tot = sum(ts)
    value = flops * len(ts) / tot / 1e12
    nt = oracle.num_threads()
    cpu = {"value": value, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
           "sample": f"first {rows} of {layers[0][1].M} token rows through all {len(layers)} layers per step "
                     f"on the host cores of rank 0{threads_note(rows, nt)}"}
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(ts), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle: float32 quantization, double GEMM)",
           "data": "synthetic", "impl": "reference",
           "config": dense_arm_config(args.workload, layers, args.block, world),
           "cpu_baseline": cpu,
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1, help="ranks (one per GPU, launched by torchrun when > 1)")
    ap.add_argument("--steps", type=int, default=200, help="timed steps")
    ap.add_argument("--warmup", type=int, default=10, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help=f"{DEFAULT_WORKLOAD} (default: the largest single-GPU configuration, float scales), "
                         "esm2_ffn, dsv3_mlp, llama_m<M> (e.g. llama_m16), "
                         "square_m<M>_float or square_m<M>_ue8m0 (K = N = 12288), moe_dsv3")
    ap.add_argument("--impl", default="fg8", choices=["fg8", "reference"],
                    help="fg8: this library; reference: the CPU oracle on a bounded sample")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU time the oracle baseline of the fg8 arm aims at (rank 0, one GPU)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle baseline of the fg8 arm")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: CPU seconds that the warm-up and timed steps together aim at")
    ap.add_argument("--block", type=int, default=128, choices=[128, 64, 32],
                    help="weight_block_size (block, block) and 1 x block activation groups (either scale format)")
    ap.add_argument("--no-chain", action="store_true",
                    help="quantize every layer's input in its own launch instead of in the previous GEMM")
    ap.add_argument("--fused-quant", action="store_true",
                    help="quantize a tiled layer's input inside its GEMM's launch (fg8_linear_fused) instead of in "
                         "the separate act-quant launch the GEMM overlaps (the default: measured faster)")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="store the DRAM bytes of the GEMM launches in an ncu raw CSV export for --workload, then exit")
    args = ap.parse_args(argv)
    if args.record_traffic:
        record_traffic(args.record_traffic, args.workload)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_env()
    if args.block != 128 and args.workload.startswith("moe_"):
        raise SystemExit("--block 32 / 64 runs the dense workloads (the expert GEMM takes 128 x 128 blocks)")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.workload.startswith("moe_"):
        if args.workload != "moe_dsv3":
            raise SystemExit(f"unknown workload {args.workload}")
        run_moe(args, rank, world, local)
        return
    run_fg8(args, rank, world, local)


if __name__ == "__main__":
    main()
