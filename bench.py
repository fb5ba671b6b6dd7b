"""Benchmark of the MoE layer with zero-computation experts on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the whole path on one batch: route (router GEMM +
softmax + biased top-K + counts) -> dispatch to FFN experts -> SwiGLU expert
GEMMs (gate/up, down) -> combine with the identity experts -> expert-bias
update.  With N > 1 every rank processes its own batch with a full
weight replica (weak scaling); the count histograms are summed over ranks with
NCCL before the bias update, the one exchange step of the method.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle instead, on a bounded sample of the same workload.

At N=1 the default LongCat line also carries a "decode" object: the mid layer at
T = 16, 64, 256 tokens, one CUDA graph per step with L2 flushed before every
step, and its HBM fraction (--no-decode skips it).  ``--gpus N`` without
torchrun starts the N ranks itself (one process per GPU).

Options: --graph (replay one captured CUDA graph per step), --fp8-experts
(MXFP8 expert weights), --fused-gather (no x_perm copy), --lb-stats (the
load-balance statistics each step), --backward (also time a training step:
forward keeping the pre-activations, then the backward pass).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_30_b200 import binding as B  # noqa: E402
from mixture_experts_layer_30_b200 import configs as C  # noqa: E402
from mixture_experts_layer_30_b200 import dist as MD  # noqa: E402
from mixture_experts_layer_30_b200 import inputs as IN  # noqa: E402

METRIC = "MoE-layer tokens/sec at LongCat shape (bf16) + % of tensor/HBM roofline"
DEFAULT_WORKLOAD = C.LONGCAT_PREFILL.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
TC_SOURCE = os.path.join(ROOT, "mixture_experts_layer_30_b200", "csrc", "gemm_tc.cuh")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(path=TC_SOURCE, text=None):
    """sha256 prefix of the GEMM source with comments and blank lines removed
    (a comment edit does not invalidate counters taken on the same code)."""
    import re
    if text is None:
        with open(path) as f:
            text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def committed_traffic(kernel, workload):
    """dram bytes per launch of ``kernel`` from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_sha") != source_digest() or e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region.  start()
    returns once the first sample has arrived, so that a short region is
    covered too."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx, self.proc, self.lines, self.reader = gpu_index, None, [], None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        first = threading.Event()

        def read():
            for line in self.proc.stdout:
                self.lines.append(line)
                first.set()
        self.reader = threading.Thread(target=read, daemon=True)
        self.reader.start()
        first.wait(timeout=3.0)
        self.n0 = len(self.lines)  # samples from before the region are dropped

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.reader.join(timeout=5)
        lines = self.lines[max(0, self.n0 - 1):]  # the last sample before the region, onwards
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_config(cfg, world, args):
    """The ``config`` object of the JSON line; both arms print the same one."""
    tiled = cfg.dtype == "bf16" and cfg.d % 128 == 0 and cfg.I % 128 == 0
    fp8 = getattr(args, "fp8_experts", False)
    wsz = (1 + 1 / 32) if fp8 else (2 if cfg.dtype == "bf16" else 4)
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "N": cfg.N, "Z": cfg.Z,
            "K": cfg.K, "I": cfg.I, "K_e": cfg.K_e, "tokens_per_rank": cfg.T,
            "expert_weights": ("mxfp8 (moe_quantize_weights_mxfp8)" if fp8
                               else "tiled (moe_pack_weights)" if tiled else "row-major"),
            "parallelism": f"token-dp{world} (weights replicated, counts all-reduced)",
            "l2": ("flushed before every timed step (256 MB memset, outside the "
                   "per-step events)") if getattr(args, "flush_l2", False) else
                  (f"inputs larger than L2 ({cfg.N * 3 * cfg.I * cfg.d * wsz / 1e9:.2f} GB "
                   "of expert weights, 126 MB L2; the touched experts' weights are "
                   "streamed every step)")}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args, rank, world, local_rank):
    cfg = C.CONFIGS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    tiled = cfg.dtype == "bf16" and cfg.d % 128 == 0 and cfg.I % 128 == 0
    shape = B.shape_of(cfg, weight_layout=B.WEIGHTS_TILED if tiled else B.WEIGHTS_ROW_MAJOR)
    L = IN.make_layer_inputs(cfg, device=dev, base_seed=0)
    # every rank routes its own batch: x drawn with a per-rank seed
    seed = MD.rank_x_seed(rank)
    if seed is not None:
        L["x"] = IN.make_x(cfg, dev, seed=seed)
    # expert weights repacked once into the tiled order, or quantised to MXFP8
    # (untimed set-up); the row-major originals stay for the oracle baseline
    fp8 = args.fp8_experts
    # decode-sized batches: the route call also builds the dispatch layout and the
    # gate/up GEMM reads x through row_token (no x_perm copy, one launch fewer)
    gather = args.fused_gather or (cfg.T <= DECODE_MAX_T and not fp8 and not args.x_perm_copy)
    if fp8:
        W = {k: B.quantize_weights_mxfp8(L[k]) for k in ("w1", "w3", "w2")}
        fbuf = B.Mxfp8Buffers(shape, device=dev)
    else:
        W = {k: (B.pack_weights(L[k]) if tiled else L[k]) for k in ("w1", "w3", "w2")}
    torch.cuda.synchronize()
    buf = B.LayerBuffers(shape, device=dev)
    bias = L["bias"].clone()
    counts_global = torch.empty_like(buf.counts)
    T_all = MD.global_tokens(cfg.T)
    K_e, mu = float(np.float32(cfg.K_e)), float(np.float32(cfg.mu))
    if world > 1:
        import torch.distributed as dist

    lb = None
    if args.lb_stats:
        D_groups = 32 if cfg.N % 32 == 0 else 1
        lb = dict(D=D_groups, prob_sum=torch.empty(cfg.E, dtype=torch.float32, device=dev),
                  f=torch.empty(D_groups + 1, dtype=torch.float32, device=dev),
                  P=torch.empty(D_groups + 1, dtype=torch.float32, device=dev),
                  loss=torch.empty(1, dtype=torch.float32, device=dev))

    # Eq. (2) needs only this step's counts: in a captured step it runs on a
    # second stream beside the expert path (joined before the step ends)
    fork_bias = bool(args.graph)
    side = torch.cuda.Stream(dev)

    def step(x, ev=None):
        s = shape
        if ev: ev[0].record(stream)
        psum = None if lb is None else lb["prob_sum"]
        if gather:
            # the selection and the dispatch layout in one call; no x_perm copy
            B.route_dispatch(s, x, L["w_router"], bias, buf.ws, buf.topk_idx, buf.topk_gate,
                             buf.counts, buf.n_ffn, buf.offsets, buf.row_token, buf.slot_pos,
                             prob_sum=psum)
        else:
            B.route(s, x, L["w_router"], bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts,
                    buf.n_ffn, prob_sum=psum)
        if fork_bias and not ev:
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                c = MD.global_counts(buf.counts, counts_global) if world > 1 else buf.counts
                B.bias_update(cfg.N, cfg.Z, c, T_all, cfg.K, K_e, mu, bias, stream=side)
        if lb is not None:
            # Eq. (3)-(5) statistics on this rank's batch
            B.lb_stats(cfg.N, cfg.Z, lb["D"], buf.counts, lb["prob_sum"], cfg.T, cfg.K, K_e,
                       0.001, lb["f"], lb["P"], lb["loss"])
        if ev: ev[1].record(stream)
        if fp8:
            B.permute_mxfp8(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token,
                            buf.slot_pos, fbuf.x_perm_q, fbuf.x_perm_sf, buf.ws)
            if ev: ev[2].record(stream)
            B.expert_gate_up_mxfp8(s, fbuf.x_perm_q, fbuf.x_perm_sf, W["w1"], W["w3"],
                                   buf.offsets, fbuf.h_q, fbuf.h_sf, buf.ws)
            if ev: ev[3].record(stream)
            B.expert_down_mxfp8(s, fbuf.h_q, fbuf.h_sf, W["w2"], buf.offsets, buf.y_perm, buf.ws)
        else:
            if not gather:
                B.permute(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token,
                          buf.slot_pos, buf.x_perm, buf.ws)
            if ev: ev[2].record(stream)
            if gather:
                B.expert_gate_up_gather(s, x, buf.row_token, W["w1"], W["w3"], buf.offsets,
                                        buf.h, buf.ws)
            else:
                B.expert_gate_up(s, buf.x_perm, W["w1"], W["w3"], buf.offsets, buf.h, buf.ws)
            if ev: ev[3].record(stream)
            B.expert_down(s, buf.h, W["w2"], buf.offsets, buf.y_perm, buf.ws)
        if ev: ev[4].record(stream)
        B.combine(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, cfg.gamma, buf.out)
        if ev: ev[5].record(stream)
        if ev or not fork_bias:
            c = MD.global_counts(buf.counts, counts_global) if world > 1 else buf.counts
            B.bias_update(cfg.N, cfg.Z, c, T_all, cfg.K, K_e, mu, bias)
        else:
            stream.wait_stream(side)  # the bias update of this step is done
        if ev: ev[6].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    x = L["x"]
    for _ in range(args.warmup):
        step(x)
    barrier()
    st = B.device_status(buf.ws)
    if st:
        raise RuntimeError(f"device status 0x{st:x} after warm-up")

    # ---- device-resident timing ----
    n_ev = 7
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else local_rank)
    graph = None
    if args.graph:
        # one step captured once and replayed: no host launch cost per kernel
        graph = torch.cuda.CUDAGraph()
        n0 = B.kernel_launches()
        with torch.cuda.graph(graph):
            step(x)
        per_step_launches = B.kernel_launches() - n0
        graph.replay()
        barrier()
    launches0 = B.kernel_launches()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None
    fl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)] if flush is not None else None
    barrier()
    bias_t0 = bias.clone()  # the timed steps are replayed from here (realised work)
    clocks.start()
    t0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            # evict the previous step's data: write 256 MB (> the 126 MB L2), then
            # time the step alone
            flush.zero_()
            fl_ev[i][0].record(stream)
        if graph is None:
            step(x)
        else:
            graph.replay()
        if flush is not None:
            fl_ev[i][1].record(stream)
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    launches = (B.kernel_launches() - launches0) if graph is None else per_step_launches * args.steps
    ms_total = t0.elapsed_time(t1)
    if flush is not None:
        ms_total = sum(a.elapsed_time(b) for a, b in fl_ev)
    # realised work of the timed steps: the bias (and so the routing) changes every
    # step, and the layer is deterministic, so the steps are replayed from the same
    # bias to read each one's counts; the replay must end on the same bias bits
    bias_end = bias.clone()
    bias.copy_(bias_t0)
    timed_counts = []
    for i in range(args.steps):
        step(x)
        timed_counts.append(buf.counts.cpu().numpy().astype(np.int64))
    replay_equal = bool(torch.equal(bias, bias_end))
    # per-call breakdown from a separate eager pass: events between the calls
    # would keep the launches of the timed steps from overlapping
    pc = ClockSampler(clocks.idx)
    pc.start()
    per_counts = []
    for i in range(args.steps):
        step(x, evs[i])
        per_counts.append(buf.counts.cpu().numpy().astype(np.int64))
    barrier()
    per_clk = pc.stop()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n_ev - 1)]
                    for i in range(args.steps)])
    ms_step = MD.max_over_ranks(ms_total / args.steps, dev)

    # ---- end to end through the public API with host buffers ----
    # Every step copies its x from pinned host memory and reads its output back.
    # Copies run on their own streams, double-buffered, so the copy of step i+1
    # and the read-back of step i-1 overlap the layer of step i.
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x.cpu())
    out_host = [torch.empty(buf.out.shape, dtype=buf.out.dtype, pin_memory=True) for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    out_dev = [buf.out, torch.empty_like(buf.out)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    x_ready, x_free = [ev(), ev()], [ev(), ev()]
    done, out_free = [ev(), ev()], [ev(), ev()]

    def e2e_loop(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(x_free[j])
                x_dev[j].copy_(x_host, non_blocking=True)
                x_ready[j].record(s_in)
            stream.wait_event(x_ready[j])
            if i >= 2:
                stream.wait_event(out_free[j])
            s = shape
            if gather:
                B.route_dispatch(s, x_dev[j], L["w_router"], bias, buf.ws, buf.topk_idx,
                                 buf.topk_gate, buf.counts, buf.n_ffn, buf.offsets,
                                 buf.row_token, buf.slot_pos)
            else:
                B.route(s, x_dev[j], L["w_router"], bias, buf.ws, buf.topk_idx, buf.topk_gate,
                        buf.counts, buf.n_ffn)
            if fp8:
                B.permute_mxfp8(s, x_dev[j], buf.topk_idx, buf.counts, buf.offsets,
                                buf.row_token, buf.slot_pos, fbuf.x_perm_q, fbuf.x_perm_sf,
                                buf.ws)
                B.expert_gate_up_mxfp8(s, fbuf.x_perm_q, fbuf.x_perm_sf, W["w1"], W["w3"],
                                       buf.offsets, fbuf.h_q, fbuf.h_sf, buf.ws)
                B.expert_down_mxfp8(s, fbuf.h_q, fbuf.h_sf, W["w2"], buf.offsets, buf.y_perm,
                                    buf.ws)
            else:
                if not gather:
                    B.permute(s, x_dev[j], buf.topk_idx, buf.counts, buf.offsets,
                              buf.row_token, buf.slot_pos, buf.x_perm, buf.ws)
                if gather:
                    B.expert_gate_up_gather(s, x_dev[j], buf.row_token, W["w1"], W["w3"],
                                            buf.offsets, buf.h, buf.ws)
                else:
                    B.expert_gate_up(s, buf.x_perm, W["w1"], W["w3"], buf.offsets, buf.h,
                                     buf.ws)
                B.expert_down(s, buf.h, W["w2"], buf.offsets, buf.y_perm, buf.ws)
            B.combine(s, x_dev[j], buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos,
                      cfg.gamma, out_dev[j])
            x_free[j].record(stream)
            c = MD.global_counts(buf.counts, counts_global) if world > 1 else buf.counts
            B.bias_update(cfg.N, cfg.Z, c, T_all, cfg.K, K_e, mu, bias)
            done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[j])
                out_host[j].copy_(out_dev[j], non_blocking=True)
                out_free[j].record(s_out)

    # the same K steps as the device-timed loop: the first step's copy in and the
    # last step's read-back have nothing to overlap with, a fixed cost per run
    e2e_steps = max(4, args.steps)
    e2e_loop(2)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_loop(e2e_steps)
    stream.wait_stream(s_out)
    e1.record(stream)
    barrier()
    e2e_ms = MD.max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    st = B.device_status(buf.ws)
    if st:
        raise RuntimeError(f"device status 0x{st:x} after timing")

    # ---- silent-data-corruption check: one step recomputed bit for bit ----
    # The layer is deterministic (fixed reduction orders, no atomics in any sum),
    # so the same step from the same bias and input must repeat exactly.
    bias_saved = bias.clone()
    step(x)
    ref_out, ref_idx, ref_counts = buf.out.clone(), buf.topk_idx.clone(), buf.counts.clone()
    bias.copy_(bias_saved)
    step(x)
    barrier()
    sdc_equal = bool(torch.equal(ref_out, buf.out) and torch.equal(ref_idx, buf.topk_idx)
                     and torch.equal(ref_counts, buf.counts))
    n_ffn = buf.n_ffn.float()
    load = buf.counts[:cfg.N].float()
    routing_stats = {"ffn_experts_per_token_mean": round(float(n_ffn.mean()), 4),
                     "ffn_experts_per_token_std": round(float(n_ffn.std()), 4),
                     "max_over_mean_expert_load": round(float(load.max() / load.mean()), 4)}

    # ---- algorithmic work of the routed batch: per-step means over the steps
    # each figure timed (touched experts and routed rows move with the bias) ----
    def work(cl):
        return (float(np.mean([(c[:cfg.N] > 0).sum() for c in cl])),
                float(np.mean([c[:cfg.N].sum() for c in cl])))
    touched, R = work(timed_counts)          # the timed steps (value, layer fractions)
    touched_pc, R_pc = work(per_counts)      # the per-call steps (per-kernel rooflines)
    touched_all = [int((c[:cfg.N] > 0).sum()) for c in timed_counts]
    esz = 2 if cfg.dtype == "bf16" else 4
    # expert operands: bf16/fp32, or MXFP8 (1 byte + a scale byte per 32 values)
    wsz = (1 + 1 / 32) if fp8 else esz
    w13_bytes = touched * 2 * cfg.I * cfg.d * wsz
    w2_bytes = touched * cfg.d * cfg.I * wsz
    # FFN: 6 d I flop per routed row (gate, up, down); router: 2 d E per token
    layer_flops = 6.0 * cfg.d * cfg.I * R + 2.0 * cfg.d * cfg.E * cfg.T
    layer_bytes = (w13_bytes + w2_bytes + cfg.E * cfg.d * esz + 2 * cfg.T * cfg.d * esz)
    med = np.median(per, axis=0)
    peaks, peak_kind = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    tflops_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    gu_ms = float(per[:, 2].mean())
    # the per-kernel figures use the work of the steps their events timed
    gate_up_bytes_pc = (touched_pc * 2 * cfg.I * cfg.d * wsz + R_pc * cfg.d * wsz +
                        R_pc * cfg.I * wsz)
    ffn_flops_pc = 6.0 * cfg.d * cfg.I * R_pc
    achieved = gate_up_bytes_pc / (gu_ms * 1e-3) / 1e9
    traffic = committed_traffic("gate_up", cfg.name)
    ffn_ms = float((per[:, 2] + per[:, 3]).mean())

    if rank != 0:
        if args.backward:
            time_training(args, cfg, shape, L, W, dev, stream, L["bias"].clone())
        return None, L
    tokens_per_s = cfg.T * world / (ms_step * 1e-3)
    line = {
        "metric": METRIC,
        "value": round(tokens_per_s, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) activations, random-init weights of the stated shape)",
        "config": workload_config(cfg, world, args),
        "roofline": {"kernel": ("moe_expert_gate_up_mxfp8 (tcgen05 block-scaled grouped GEMM)"
                                if fp8 else "moe_expert_gate_up (tcgen05 grouped GEMM + SwiGLU)"),
                     "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": int(gate_up_bytes_pc),
                     "avg_launch_ms": round(gu_ms, 4)},
        "layer": {
            "routed_rows": round(R, 1), "touched_experts": round(touched, 2),
            "touched_experts_per_step": {"min": min(touched_all), "max": max(touched_all)},
            "work_accounting": ("per-step means over the timed steps, read by replaying them "
                                "from the same bias"),
            "replay_bitwise_equal": replay_equal,
            "ffn_tflops": round(ffn_flops_pc / (ffn_ms * 1e-3) / 1e12, 2),
            "tensor_frac_of_sustained": round(layer_flops / (ms_step * 1e-3) / 1e12 / tflops_peak, 4),
            "hbm_frac": round(layer_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak, 4),
            "roofline_frac": round(max(layer_flops / (tflops_peak * 1e12),
                                       layer_bytes / (hbm_peak * 1e9)) / (ms_step * 1e-3), 4),
            "per_call_ms_median": {k: round(float(v), 4) for k, v in zip(
                ["route", "permute", "gate_up", "down", "combine", "bias_update"], med)},
            # the same times in SM cycles at the median clock of that pass (ms x MHz =
            # thousands of cycles): separates a lower clock (power cap) from the kernel
            "per_call_kcycles_at_median_clock": None if not per_clk else {
                k: round(float(v) * per_clk["sm_mhz"], 1) for k, v in zip(
                    ["route", "permute", "gate_up", "down", "combine", "bias_update"], med)},
            "per_call_clock_mhz": None if not per_clk else per_clk["sm_mhz"],
        },
        "e2e": {"value": round(cfg.T * world / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(buf.out.numel() * buf.out.element_size())},
        "gpu_launches": int(launches),
        "routing": routing_stats,
        "sdc_check": {"bitwise_equal": sdc_equal,
                      "method": "one step recomputed from the same bias and input"},
        "cuda_graph": graph is not None,
        "lb_stats": lb is not None,
        "expert_format": "mxfp8" if fp8 else cfg.dtype,
        "dispatch": ("layout built by the route call, gate/up reads x through row_token"
                     if gather else "x_perm copy"),
        "clocks": clk,
    }
    if args.backward:
        line["training"] = time_training(args, cfg, shape, L, W, dev, stream, L["bias"].clone())
    return line, L


# ---------------------------------------------------------------------------
# decode-sized batches (memory-bound): reported beside the headline
# ---------------------------------------------------------------------------
DECODE_WORKLOADS = (C.DECODE_T16, C.DECODE_T64, C.DECODE_T256)
DECODE_MAX_T = 256  # batches up to this size dispatch without the x_perm copy


def decode_block(args, local_rank):
    """The mid layer at T = 16, 64 and 256 tokens, measured as its HBM target is
    stated: one captured CUDA graph per step, L2 flushed (256 MB written) before
    every step, each step timed alone, and the HBM fraction taken on the bytes
    the step must move (the touched experts' weights, W_r, x in and out)."""
    res = {}
    for cfg in DECODE_WORKLOADS:
        sub = argparse.Namespace(**vars(args))
        sub.workload, sub.graph, sub.flush_l2 = cfg.name, True, True
        sub.backward, sub.lb_stats, sub.fp8_experts = False, False, False
        sub.steps = max(args.steps, 200)  # >= 36 ms timed: a few clock samples
        line, _ = run_gpu(sub, 0, 1, local_rank)
        res[f"T{cfg.T}"] = {
            "workload": cfg.name, "tokens_per_s": line["value"],
            "ms_per_step": line["ms_per_step"], "hbm_frac": line["layer"]["hbm_frac"],
            "touched_experts": line["layer"]["touched_experts"],
            "per_call_ms_median_eager": line["layer"]["per_call_ms_median"],
            "gpu_launches_per_step": line["gpu_launches"] // sub.steps,
            "clocks": line["clocks"]}
        torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# training step (forward keeping the pre-activations + backward), --backward
# ---------------------------------------------------------------------------

def time_training(args, cfg, shape, L, W, dev, stream, bias):
    """Per-step time of forward_train + backward on the same batch, with the
    per-call split and the roofline of the expert backward call."""
    buf = B.LayerBuffers(shape, device=dev, with_probs=True)
    bb = B.BackwardBuffers(shape, device=dev)
    dout = IN.make_x(cfg, dev, seed=424242)  # synthetic upstream gradient, N(0, 1)
    x = L["x"]
    K_e, mu = float(np.float32(cfg.K_e)), float(np.float32(cfg.mu))
    names = ["route", "permute", "gate_up_save", "down", "combine", "combine_bwd", "route_bwd",
             "expert_ffn_bwd", "permute_bwd"]

    def tstep(ev=None):
        s = shape
        if ev: ev[0].record(stream)
        B.route(s, x, L["w_router"], bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts,
                buf.n_ffn, probs_out=buf.probs)
        if ev: ev[1].record(stream)
        B.permute(s, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
                  buf.x_perm, buf.ws)
        if ev: ev[2].record(stream)
        B.expert_gate_up_save(s, buf.x_perm, W["w1"], W["w3"], buf.offsets, buf.h, bb.au, buf.ws)
        if ev: ev[3].record(stream)
        B.expert_down(s, buf.h, W["w2"], buf.offsets, buf.y_perm, buf.ws)
        if ev: ev[4].record(stream)
        B.combine(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, cfg.gamma, buf.out)
        if ev: ev[5].record(stream)
        B.combine_backward(s, x, buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos, dout,
                           cfg.gamma, bb.dy_perm, bb.dgate)
        if ev: ev[6].record(stream)
        B.route_backward(s, x, L["w_router"], buf.probs, buf.topk_idx, bb.dgate, bb.dw_router,
                         bb.dx_router, bb.bws)
        if ev: ev[7].record(stream)
        B.expert_ffn_backward(s, buf.x_perm, W["w1"], W["w3"], W["w2"], buf.offsets, buf.h,
                              bb.au, bb.dy_perm, bb.dx_perm, bb.dw1, bb.dw3, bb.dw2, bb.bws)
        if ev: ev[8].record(stream)
        B.permute_backward(s, dout, buf.topk_idx, buf.topk_gate, buf.slot_pos, bb.dx_perm,
                           bb.dx_router, cfg.gamma, bb.dx)
        if ev: ev[9].record(stream)
        B.bias_update(cfg.N, cfg.Z, buf.counts, cfg.T, cfg.K, K_e, mu, bias)

    for _ in range(args.warmup):
        tstep()
    torch.cuda.synchronize()
    for ws in (buf.ws, bb.bws):
        st = B.device_status(ws)
        if st:
            raise RuntimeError(f"device status 0x{st:x} in the training step")
    n = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(n):
        tstep()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    for i in range(n):
        tstep(evs[i])
    torch.cuda.synchronize()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(9)] for i in range(n)])
    med = np.median(per, axis=0)
    counts = buf.counts.cpu().numpy().astype(np.int64)
    R = int(counts[:cfg.N].sum())
    touched = int((counts[:cfg.N] > 0).sum())
    esz = 2 if cfg.dtype == "bf16" else 4
    wbytes = touched * 3 * cfg.I * cfg.d * esz   # W1, W3, W2 of the touched experts
    gbytes = cfg.N * 3 * cfg.I * cfg.d * esz     # dW1, dW3, dW2 written (every expert)
    # token-row operands: dy (read twice), a|u, h, x_perm read; da|du written and
    # read twice; dx_perm written
    rows = R * esz * (2 * cfg.d + 2 * cfg.I + cfg.I + cfg.d + 3 * 2 * cfg.I + cfg.d)
    ffn_bwd_bytes = wbytes + gbytes + rows
    ffn_bwd_flops = 12.0 * cfg.d * cfg.I * R
    bwd_ms = float(per[:, 7].mean())
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    tfl = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    achieved = ffn_bwd_bytes / (bwd_ms * 1e-3) / 1e9
    return {
        "ms_per_step": round(ms, 4),
        "tokens_per_s": round(cfg.T / (ms * 1e-3), 1),
        "dout": "synthetic N(0, 1) upstream gradient",
        "per_call_ms_median": {k: round(float(v), 4) for k, v in zip(names, med)},
        "expert_ffn_backward": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_launch": int(ffn_bwd_bytes),
            "tflops": round(ffn_bwd_flops / (bwd_ms * 1e-3) / 1e12, 2),
            "tensor_frac_of_sustained": round(ffn_bwd_flops / (bwd_ms * 1e-3) / 1e12 / tfl, 4),
            "avg_launch_ms": round(bwd_ms, 4)},
    }


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
# The fp64 oracle is timed as it stands on the host cores, on a bounded sample
# of the same workload: routing (router GEMM, softmax, biased top-K, counts) on
# every token of the batch, and the expert FFNs + combine on a seeded sample of
# tokens through the whole oracle layer.  Tokens/s extrapolates the sample to
# the batch: T / (t_route(all T) + t_sample * T / n_sample).

def oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if blas:
            return int(blas[0])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _host_bits(t):
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 \
        else t.numpy()


class OracleWorkload:
    """Host copies of the batch for the oracle (expert weights fetched per call)."""

    def __init__(self, cfg, L):
        from oracle import moe_oracle as orc
        self.cfg, self.L, self.orc = cfg, L, orc
        self.dec = orc.bf16_bits_to_f64 if cfg.dtype == "bf16" else orc.as_f64
        self.x = _host_bits(L["x"])
        self.wr = _host_bits(L["w_router"])
        self.bias = L["bias"].detach().cpu().numpy()

    def time_routing(self):
        """Seconds for routing every token (decode, logits, softmax, top-K, counts)."""
        orc = self.orc
        t = time.perf_counter()
        probs = orc.softmax_rows(orc.router_logits(self.dec(self.x), self.dec(self.wr)))
        idx, _ = orc.biased_topk(probs, self.bias, self.cfg.K)
        orc.expert_counts(idx, self.cfg.E)
        return time.perf_counter() - t

    def time_sample(self, tokens):
        """Seconds for the whole oracle layer on the given tokens (their experts'
        weights decoded from the stored bits inside the timed region)."""
        orc, cfg = self.orc, self.cfg
        x = self.x[tokens]
        probs = orc.softmax_rows(orc.router_logits(self.dec(x), self.dec(self.wr)))
        idx, _ = orc.biased_topk(probs, self.bias, cfg.K)
        touched = sorted(set(int(e) for e in idx.reshape(-1) if e < cfg.N))
        w1 = {e: _host_bits(self.L["w1"][e]) for e in touched}
        w3 = {e: _host_bits(self.L["w3"][e]) for e in touched}
        w2 = {e: _host_bits(self.L["w2"][e]) for e in touched}
        t = time.perf_counter()
        orc.moe_layer(self.dec(x), self.dec(self.wr), w1, w3, w2, self.bias, N=cfg.N, K=cfg.K,
                      gamma=cfg.gamma, decode=self.dec)
        return time.perf_counter() - t, len(touched)


def sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=min(n, T), replace=False))


def cpu_baseline(cfg, L, n_tok):
    W = OracleWorkload(cfg, L)
    t_route = W.time_routing()
    toks = sample_tokens(cfg.T, n_tok, seed=12345)
    t_smp, touched = W.time_sample(toks)
    sec = t_route + t_smp * cfg.T / len(toks)
    return {"value": round(cfg.T / sec, 4), "unit": "tokens/s", "cores": oracle_threads(),
            "kind": "oracle",
            "sample": f"routing on all {cfg.T} tokens of the {cfg.name} batch ({t_route:.1f} s), "
                      f"then the whole fp64 oracle layer on a seeded sample of {len(toks)} "
                      f"tokens ({touched} experts decoded from bf16, {t_smp:.1f} s), "
                      f"extrapolated to the batch"}


def run_reference(args, rank, world):
    """--impl reference: the fp64 CPU oracle on the host cores (rank 0 only).
    Each step: routing on every token plus the oracle layer on a seeded sample
    of --ref-tokens tokens (a different sample each step), extrapolated to the
    whole batch."""
    if rank != 0:
        return None
    cfg = C.CONFIGS[args.workload]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    if cfg.dtype == "bf16" and dev.type != "cuda":
        return {"impl": "reference", "unavailable": "the bf16 workload is drawn on the GPU"}
    L = IN.make_layer_inputs(cfg, device=dev)
    W = OracleWorkload(cfg, L)
    n_tok = args.ref_tokens

    def step(i):
        toks = sample_tokens(cfg.T, n_tok, seed=1000 + i)
        t_smp, _ = W.time_sample(toks)
        return W.time_routing() + t_smp * cfg.T / len(toks)
    for w in range(args.warmup):
        step(w)
    secs = [step(args.warmup + i) for i in range(args.steps)]
    sec = sum(secs) / len(secs)
    v = round(cfg.T / sec, 4)
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded workload as the GPU arm)",
        "config": workload_config(cfg, world, args),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle_threads(),
                         "kind": "oracle",
                         "sample": f"each step: routing on all {cfg.T} tokens, then the whole "
                                   f"fp64 oracle layer on a seeded sample of {n_tok} tokens, "
                                   "extrapolated to the batch"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(C.CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-baseline-tokens", type=int, default=16,
                    help="token sample of the CPU baseline's FFN + combine leg")
    ap.add_argument("--ref-tokens", type=int, default=2,
                    help="token sample of each reference-arm step's FFN + combine leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-batch block of the default (LongCat) line")
    ap.add_argument("--lb-stats", action="store_true",
                    help="also compute the device-level load-balance statistics each step")
    ap.add_argument("--fp8-experts", action="store_true",
                    help="expert weights and routed activations in MXFP8 (block-scaled E4M3)")
    ap.add_argument("--backward", action="store_true",
                    help="also time a training step (forward keeping pre-activations + "
                         "backward pass) and report it under \"training\"")
    ap.add_argument("--fused-gather", action="store_true",
                    help="no x_perm copy: the route call builds the dispatch layout "
                         "(moe_route_dispatch) and the gate/up GEMM reads the token rows from "
                         "x (moe_expert_gate_up_gather); the default at T <= 256")
    ap.add_argument("--x-perm-copy", action="store_true",
                    help="dispatch with the x_perm copy (moe_route + moe_permute) at every T")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer before every timed step and time the steps "
                         "alone (per-step events)")
    ap.add_argument("--graph", action="store_true",
                    help="replay one captured CUDA graph per step (single GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.backward and args.fp8_experts:
        ap.error("--backward runs on bf16 experts")
    if args.fused_gather and args.fp8_experts:
        ap.error("--fused-gather is a bf16 path")

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not launched by torchrun: start one process per GPU ourselves
        if args.impl == "native" and torch.cuda.device_count() < args.gpus:
            ap.error(f"--gpus {args.gpus} but {torch.cuda.device_count()} GPUs are visible")
        sys.exit(MD.launch_ranks([sys.executable, os.path.abspath(__file__)] + sys.argv[1:],
                                 args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} disagrees with WORLD_SIZE={world}")
    if args.graph and world > 1:
        ap.error("--graph is single-GPU only")
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line, L = run_gpu(args, rank, world, local_rank)
        if line is not None:
            if (world == 1 and not args.no_decode and args.workload == DEFAULT_WORKLOAD
                    and not args.fp8_experts):
                line["decode"] = decode_block(args, local_rank)
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(C.CONFIGS[args.workload], L,
                                                    args.cpu_baseline_tokens)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
