"""Throughput of the NVFP4 MoE expert-FFN hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--config decode|mid|prefill|tiny|sweep|dense_decode|dense_prefill|
                              shared_decode|shared_prefill]
                    [--impl ours|reference] [--no-cpu-baseline] [--experts E] [--tokens T]

A step is one pass of the whole path over one batch: routing (top-k + expert buckets), amax ->
global scale -> NVFP4 quantization of the activations, L1 grouped GEMM with SwiGLU + FP4
re-quantization, L2 grouped GEMM with routing weight + scatter-add, bf16 output.  Inputs are
resident in HBM when the timed region starts; the same work through moe_ffn_forward with
host<->device copies inside the timed region gives `e2e`.

The default workload is the prefill configuration (T=8192 tokens, hidden 7168, intermediate 2048,
256 experts, top-8 over uniform random logits), the largest that the metric is quoted on:
65536 slots, 5.77 TFLOP and 6.8 GB of algorithmic traffic per step.  Its arithmetic intensity
(about 850 FLOP/B) sits below the FP4 ridge, so `value` is the algorithmic HBM traffic per second
(GB/s) and `tflops` rides along; the roofline object gives the dominant kernel's fraction of both
peaks.  --config decode (T=16) and --config mid (T=512) are the weight-streaming shapes.

Multi-GPU runs are independent replicas (the path has no exchange step on one node's data-parallel batch), so the
scaling is weak and `value` sums the ranks' bytes over the slowest rank's time.

--config sweep times the standalone 2D x 3D grouped GEMM instead (E=32 groups, M_g ~ U{0..4096},
K=7168, N=4096, bf16 output): a step is one grouped-GEMM launch over NVFP4 operands already in HBM.

--config dense_decode | dense_prefill times the dense NVFP4 linear with the RMSNorm fused into its
activation quantizer (the MoE shared expert's gate/up projection: M = 16 or 8192 rows, K = 7168,
N = 4096): a step is RMSNorm + amax -> quantize -> dense GEMM, bf16 out, with L2 flushed before
every step (the 16.5 MB weight would otherwise stay in the 126 MB L2).

--config shared_decode | shared_prefill times the whole shared expert (M = 16 or 8192 rows,
hidden 7168, intermediate 2048): RMSNorm + quantize -> L1 with SwiGLU + FP4 re-quantization ->
down projection, bf16 out, L2 flushed before every step.

--impl reference times the CPU oracle (numpy, float64) on a bounded sample of the same workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE FFN TFLOPS & HBM GB/s on 1 B200, % of NVFP4 tensor/HBM roofline"
FP4_ELEM_BYTES = 0.5 + 1.0 / 16.0  # E2M1 code + one E4M3 scale per 16 elements
FP4_PER_BF16 = 4.0  # nominal dense tensor throughput ratio FP4 : BF16 on B200 (9 : 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="prefill")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller weight set for profiling captures)")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling captures)")
    ap.add_argument("--soak", type=float, default=1.0,
                    help="seconds of extra warm-up load so clock samples cover the timed region")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting

def algorithmic(cfg, counts):
    """FLOPs and bytes of one step, and per-kernel bytes of the two GEMM launches.

    Weights of the experts that received tokens (codes + scales), x read as bf16, x codes written
    and read once per token, h codes written and read once per slot, bf16 output written, logits
    read.  Padding rows and the FP32 scatter buffer are implementation overhead, not counted."""
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    active = sum(1 for c in counts if c > 0)
    slots = sum(counts)
    w1 = 2 * I * H * FP4_ELEM_BYTES
    w2 = H * I * FP4_ELEM_BYTES
    x_q = T * H * FP4_ELEM_BYTES
    h_q = slots * I * FP4_ELEM_BYTES
    total = active * (w1 + w2) + T * H * 2 + 2 * x_q + 2 * h_q + T * H * 2 + T * E * 4
    flops = 2 * slots * (H * 2 * I + I * H)
    l1 = active * w1 + slots * H * FP4_ELEM_BYTES + h_q
    l2 = active * w2 + h_q + T * H * 4
    return dict(flops=flops, bytes=total, active=active, slots=slots, l1_bytes=l1, l2_bytes=l2,
                l1_flops=2 * slots * H * 2 * I, l2_flops=2 * slots * I * H)


DEVICE_SIDE_END = b"// ------------------------------------------------------------------------------ host side"


def kernel_sources_sha16():
    """Hash of the grouped GEMM's device code: gemm.cu up to its host-side section, then
    common.cuh.  Host launch code and the other kernels of gemm.cu do not change the captured
    kernel's DRAM traffic."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_block_scaled_gsa_b200", "csrc")
    with open(os.path.join(csrc, "gemm.cu"), "rb") as fh:
        text = fh.read()
    cut = text.find(DEVICE_SIDE_END)
    h.update(text if cut < 0 else text[:cut])
    with open(os.path.join(csrc, "common.cuh"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the dominant kernel,
# from one ncu capture per workload, keyed by the hash of the grouped GEMM's device code at the
# time of the capture (the capture command and the raw counters are in profiles/).  Figures of
# a reduced capture are scaled to the full launch by the units it processes, as noted there.
CAPTURED_TRAFFIC = {
    # workload: (kernel_sources_sha16 at the capture, bytes per launch)
    "decode": ("49adf8f15b32f17f", 1672600000),
    "prefill": ("49adf8f15b32f17f", 4669000000),
}


def captured_traffic(cfg):
    """DRAM bytes per launch of the dominant kernel from the ncu capture of this workload, or None
    when there is none or the kernel's device code changed since that capture."""
    entry = CAPTURED_TRAFFIC.get(cfg.name)
    if entry is None or entry[0] != kernel_sources_sha16():
        return None
    return entry[1]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# ----------------------------------------------------------------------------- ranks

def slowest_rank_ms(ms, world, device="cpu"):
    """The timed region's length on the slowest rank: every rank passes its own CUDA-event time
    and gets the maximum over ranks (a no-op for one process)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank, steps, world, total_ms):
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_step_per_rank * steps / (total_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.p = None
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        self.p.terminate()
        out, _ = self.p.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(smax) if smax else None, reasons=sorted(reasons),
                    samples=len(sm))


# ----------------------------------------------------------------------------- our arm

class Plan:
    """Pre-allocated buffers for the step run call by call (the kernels moe_ffn_forward chains),
    with events between the calls for the stage breakdown."""

    def __init__(self, nv, cfg, x, logits, w1, w2, gs_h):
        import torch
        self.nv, self.cfg = nv, cfg
        T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
        dev = x.device
        self.x, self.logits, self.w1, self.w2, self.gs_h = x, logits, w1, w2, gs_h
        self.R = nv.rows_max(T, E, k)
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        e = lambda n, t: torch.empty(max(int(n), 1), dtype=t, device=dev)  # noqa: E731
        self.ids, self.w = e(T * k, i32), e(T * k, f32)
        self.offs, self.dst = e(E + 1, i32), e(T * k, i32)
        self.row_slot, self.row_w = e(self.R, i32), e(self.R, f32)
        self.pws = e(max(nv.lib().moe_permute_workspace_size(T, E, k), 1), torch.uint8)
        self.xq, self.xsf = e(self.R * H // 2, u8), e(self.R * H // 16, u8)
        self.gs_x, self.qws = e(1, f32), e(256, u8)
        self.hq, self.hsf = e(self.R * I // 2, u8), e(self.R * I // 16, u8)
        # the L2 form moe_ffn_forward uses for this batch: 1 = token-row reductions (an FP32
        # [T][H] accumulator), 0 = per-slot rows [T*k][H] summed in slot order
        self.l2_form = nv.l2_form(T, k, E)
        self.ys = e(T * H if self.l2_form else T * k * H, f32)
        self.out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=i32, device=dev)
        self.ffn_ws = e(nv.ffn_workspace_bytes(T, H, I, E, k), torch.uint8)
        self.ffn_out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    def forward(self):
        """One step through the product call, moe_ffn_forward (the kernels step() runs one by
        one, chained inside the library)."""
        self.nv.moe_ffn_forward(self.x, self.logits, self.cfg.k, self.w1, self.w2, self.gs_h,
                                out=self.ffn_out, ws=self.ffn_ws, status=self.status)

    def step(self, ev=None):
        from nvfp4_block_scaled_gsa_b200._native import call
        import torch
        nv, c = self.nv, self.cfg
        T, H, I, E, k = c.T, c.H, c.I, c.E, c.k
        s = torch.cuda.current_stream().cuda_stream
        p = lambda t: t.data_ptr()  # noqa: E731
        if ev:
            ev[0].record()
        call("moe_permute", p(self.logits), T, E, k, 1, p(self.ids), p(self.w), p(self.offs),
             p(self.dst), p(self.row_slot), p(self.row_w), p(self.pws), self.pws.numel(),
             p(self.status), s)
        if ev:
            ev[1].record()
        call("nvfp4_quantize", p(self.x), T, H, H, p(self.dst), k, self.R, p(self.xq), p(self.xsf),
             p(self.gs_x), 1, p(self.qws), 256, p(self.status), s)
        if ev:
            ev[2].record()
        call("moe_grouped_gemm_l1_swiglu_q", p(self.xq), p(self.xsf), p(self.gs_x),
             p(self.w1.codes), p(self.w1.sf), p(self.w1.gs), p(self.offs), p(self.row_slot),
             E, H, I, self.R,
             p(self.gs_h), p(self.hq), p(self.hsf), p(self.status), s)
        if ev:
            ev[3].record()
        if self.l2_form:
            call("moe_grouped_gemm_l2_scatter_add", p(self.hq), p(self.hsf), p(self.gs_h),
                 p(self.w2.codes), p(self.w2.sf), p(self.w2.gs), p(self.offs), p(self.row_slot),
                 p(self.row_w), p(self.dst), E, H, I, T, k, self.R, p(self.ys), p(self.out),
                 p(self.status), s)
        else:
            call("moe_grouped_gemm_l2_scatter", p(self.hq), p(self.hsf), p(self.gs_h),
                 p(self.w2.codes), p(self.w2.sf), p(self.w2.gs), p(self.offs), p(self.row_slot),
                 p(self.row_w), p(self.dst), E, H, I, T, k, self.R, p(self.ys), None, p(self.out),
                 p(self.status), s)
        if ev:
            ev[4].record()


def kernels_per_step(nv, cfg):
    """Kernels one moe_ffn_forward launches: the routing (one kernel below 4096 slots, the row map
    taking the top-k itself; from 4096 slots a top-k, a count and a row-map kernel), amax,
    quantize, the L1 GEMM, the L2 GEMM, and the combine or the bf16 rounding."""
    multi = nv.lib().moe_permute_workspace_size(cfg.T, cfg.E, cfg.k) > 0
    return (3 if multi else 1) + 5


def make_config(args):
    from dataclasses import replace

    from synth import CONFIGS
    cfg = CONFIGS[args.config]
    if args.experts:
        cfg = replace(cfg, E=args.experts, name=f"{cfg.name}-E{args.experts}")
    if args.tokens:
        cfg = replace(cfg, T=args.tokens, name=f"{cfg.name}-T{args.tokens}")
    return cfg


def setup_inputs(cfg, dev):
    import torch

    import nvfp4_block_scaled_gsa_b200 as nv
    from synth import gen_logits, gen_weight_expert, gen_x
    logits = gen_logits(cfg)
    x = gen_x(cfg)
    w1 = nv.quantize_w1(lambda e: gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H, device=dev),
                        cfg.E, cfg.I, cfg.H, device=dev)
    w2 = nv.quantize_weights(lambda e: gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I, device=dev),
                             cfg.E, cfg.H, cfg.I, device=dev)
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=dev)
    return logits, x, w1, w2, gs_h


def run_ours(args):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_gsa_b200 as nv
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = make_config(args)
    logits_cpu, x_cpu, w1, w2, gs_h = setup_inputs(cfg, dev)
    logits, x = logits_cpu.to(dev), x_cpu.to(dev)
    plan = Plan(nv, cfg, x, logits, w1, w2, gs_h)

    for _ in range(max(args.warmup, 3)):
        plan.step()
        plan.forward()
    torch.cuda.synchronize()
    ids = plan.ids[: cfg.T * cfg.k].cpu()  # tokens per expert, for the byte count
    real = torch.bincount(ids[ids >= 0].long(), minlength=cfg.E).tolist()
    acc = algorithmic(cfg, real)

    # clock soak: keep the GPU under the same load so samples cover the timed region
    sampler = ClockSampler(local) if rank == 0 else None
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(8):
            plan.forward()
        torch.cuda.synchronize()

    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    start.record()
    for i in range(K):
        plan.forward()
    stop.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = start.elapsed_time(stop)
    # stage breakdown from separate steps with events between the stages (an event between two
    # kernels also stops the next one from starting early, so these steps are not the timed ones)
    ks = max(1, min(K, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(ks)]
    for i in range(ks):
        plan.step(evs[i])
    torch.cuda.synchronize()
    stage = [[evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(ks)] for j in range(4)]
    l1_ms = statistics.mean(stage[2])
    l2_ms = statistics.mean(stage[3])
    code, rc = nv.read_status(plan.status)
    if code != 0:
        raise RuntimeError(f"device status {code} after the timed region")

    total_ms = slowest_rank_ms(total_ms, world, dev)
    ms_step = total_ms / K
    value = whole_job_rate(acc["bytes"], K, world, total_ms) / 1e9
    tflops = whole_job_rate(acc["flops"], K, world, total_ms) / 1e12

    # ---- end to end through moe_ffn_forward with host buffers (pinned), copies timed.  Every
    # step copies its inputs in from pinned host memory and its output back.  Served the way a
    # stream of batches is served: the copy-in, compute and copy-out of consecutive steps run on
    # three streams with two device buffer sets, so step i's copies overlap steps i-1 and i+1's
    # compute (the timed region still holds every step's copies).  The fully serialized form
    # (copy in, compute, copy out, one stream) is timed too.
    x_h = x_cpu.pin_memory()
    lg_h = logits_cpu.pin_memory()
    out_h = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(x) for _ in range(2)]
    lg_d = [torch.empty_like(logits) for _ in range(2)]
    out_d = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = torch.empty(nv.ffn_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8,
                     device=dev)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_serial():
        x_d[0].copy_(x_h, non_blocking=True)
        lg_d[0].copy_(lg_h, non_blocking=True)
        nv.moe_ffn_forward(x_d[0], lg_d[0], cfg.k, w1, w2, gs_h, out=out_d[0], ws=ws,
                           status=plan.status)
        out_h[0].copy_(out_d[0], non_blocking=True)

    def e2e_pipelined(n):
        for i in range(n):
            b = i % 2
            if i >= 2:  # buffer set b was read by step i-2's compute and copy-out
                s_in.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_in):
                x_d[b].copy_(x_h, non_blocking=True)
                lg_d[b].copy_(lg_h, non_blocking=True)
                ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            if i >= 2:
                s_cmp.wait_event(ev_out[b])
            with torch.cuda.stream(s_cmp):
                nv.moe_ffn_forward(x_d[b], lg_d[b], cfg.k, w1, w2, gs_h, out=out_d[b], ws=ws,
                                   status=plan.status)
                ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                out_h[b].copy_(out_d[b], non_blocking=True)
                ev_out[b].record(s_out)

    def timed(fn, first_stream, last_stream):
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(first_stream)
        for st in (s_in, s_cmp, s_out):  # nothing of the timed steps starts before t0
            st.wait_event(t0)
        fn()
        for st in (s_in, s_cmp, s_out):  # t1 follows every stream's last operation
            last_stream.wait_stream(st)
        t1.record(last_stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return t0.elapsed_time(t1)

    cur = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        e2e_serial()
    e2e_pipelined(max(args.warmup, 3))
    serial_ms = slowest_rank_ms(
        timed(lambda: [e2e_serial() for _ in range(K)], cur, cur), world, dev)
    e2e_ms = slowest_rank_ms(timed(lambda: e2e_pipelined(K), s_in, s_out), world, dev)
    e2e_value = whole_job_rate(acc["bytes"], K, world, e2e_ms) / 1e9
    serial_value = whole_job_rate(acc["bytes"], K, world, serial_ms) / 1e9
    h2d = x_h.numel() * x_h.element_size() + lg_h.numel() * lg_h.element_size()
    d2h = out_h[0].numel() * out_h[0].element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, logits_cpu, x_cpu, dev)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks = load_peaks()
    l1_gbs = acc["l1_bytes"] / (l1_ms * 1e-3) / 1e9
    l1_tflops = acc["l1_flops"] / (l1_ms * 1e-3) / 1e12
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    tensor_bound = acc["l1_flops"] / acc["l1_bytes"] > fp4_peak * 1e12 / (peaks["hbm"] * 1e9)
    if tensor_bound:
        roof = {"bound": "tensor", "kernel": "grouped_gemm_kernel<L1_SWIGLU>",
                "achieved": round(l1_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                "frac": round(l1_tflops / fp4_peak, 4), "traffic": captured_traffic(cfg),
                "algorithmic_flops_per_launch": int(acc["l1_flops"]),
                "peak_source": f"{peaks['src']} bf16 burst x {FP4_PER_BF16} (nominal FP4/BF16 "
                               "dense ratio)",
                "step_frac": round(tflops / world / fp4_peak, 4)}
    else:
        roof = {"bound": "hbm", "kernel": "grouped_gemm_kernel<L1_SWIGLU>",
                "achieved": round(l1_gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(l1_gbs / peaks["hbm"], 4), "traffic": captured_traffic(cfg),
                "algorithmic_bytes_per_launch": int(acc["l1_bytes"]),
                "peak_source": peaks["src"],
                "step_frac": round(value / world / peaks["hbm"], 4)}
    # the other bound's fraction for the same launch (prefill sits near the ridge)
    roof["tensor_frac"] = round(l1_tflops / fp4_peak, 4)
    roof["hbm_frac"] = round(l1_gbs / peaks["hbm"], 4)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 + e4m3/16), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) bf16 activations, N(0,0.02) bf16 weights quantized "
                "to NVFP4 on the GPU; no trained weights)",
        "config": {"workload": f"{cfg.name} MoE FFN: T={cfg.T}, H={cfg.H}, I={cfg.I}, E={cfg.E}, "
                               f"top-{cfg.k} ({cfg.logits} logits)",
                   "parallelism": f"replicas x{world}",
                   "l2": f"no flush: each step streams {acc['active']} experts' weights "
                         f"({acc['active'] * (3 * cfg.I * cfg.H) * FP4_ELEM_BYTES / 1e9:.2f} GB) "
                         "> 126 MB L2"},
        "tflops": round(tflops, 3),
        "algorithmic": {"bytes_per_step": int(acc["bytes"]), "flops_per_step": int(acc["flops"]),
                        "active_experts": acc["active"], "slots": acc["slots"]},
        "roofline": roof,
        "stages_ms": {"route": round(statistics.mean(stage[0]), 4),
                      "quantize": round(statistics.mean(stage[1]), 4),
                      "l1_gemm_swiglu_q": round(l1_ms, 4), "l2_gemm_scatter": round(l2_ms, 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 4),
                "schedule": "copy-in, compute and copy-out on three streams, two buffer sets: "
                            "each step's copies overlap its neighbours' compute",
                "serialized": {"value": round(serial_value, 2), "unit": "GB/s",
                               "ms_per_step": round(serial_ms / K, 4)}},
        "gpu_launches": kernels_per_step(nv, cfg) * K,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- oracle

class _SparseWeights:
    """Quantized weights of a few experts, for the oracle's sampled run."""

    def __init__(self, E, N, parts):
        self.E, self.N, self.parts = E, N, parts

    def dequant(self, e):
        return self.parts[e].dequant(0)


def _oracle_sample(cfg, logits_cpu, x_cpu, dev, n_tokens=1, n_experts=1):
    """Bounded oracle sample: the first n_tokens tokens of the workload, evaluated through the
    first n_experts of the experts they route to (the oracle's `experts` restriction).  Weight
    pre-packing (quantizing the float weights with the oracle) is done here, untimed."""
    import numpy as np

    from oracle import moe as M
    from oracle import routing as R
    from synth import gen_weight_expert
    lg = logits_cpu[:n_tokens].numpy()
    x = x_cpu[:n_tokens].float().numpy()
    ids, _ = R.route_topk(lg, cfg.k)
    routed = []
    for e in ids.ravel():
        if e >= 0 and int(e) not in routed:
            routed.append(int(e))
    experts = sorted(routed[:n_experts])
    p1, p2 = {}, {}
    for e in experts:
        w1 = gen_weight_expert(cfg.seed, 1, e, 2 * cfg.I, cfg.H, device=dev).float().cpu().numpy()
        w2 = gen_weight_expert(cfg.seed, 2, e, cfg.H, cfg.I, device=dev).float().cpu().numpy()
        p1[e] = M.QuantWeights.from_float(w1[None])
        p2[e] = M.QuantWeights.from_float(w2[None])
    W1 = _SparseWeights(cfg.E, 2 * cfg.I, p1)
    W2 = _SparseWeights(cfg.E, cfg.H, p2)

    def run():
        return M.moe_ffn(x, lg, cfg.k, W1, W2, np.float32(cfg.gs_h), experts=experts)

    counts = [0] * cfg.E
    for e in ids.ravel():
        if int(e) in experts:
            counts[int(e)] += 1
    from dataclasses import replace
    return run, algorithmic(replace(cfg, T=n_tokens), counts), experts


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    except Exception:
        n = 1
    return n


def cpu_baseline(cfg, logits_cpu, x_cpu, dev):
    """The oracle on a bounded sample (about 10-30 s of CPU work): the first tokens of the
    workload through their first routed expert each, repeated until 10 s have passed."""
    run, acc, experts = _oracle_sample(cfg, logits_cpu, x_cpu, dev)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= 10.0:
            break
    return {"value": round(acc["bytes"] * reps / dt / 1e9, 4), "unit": "GB/s", "cores": _threads(),
            "kind": "oracle",
            "sample": f"token 0 of the {cfg.name} workload through expert {experts[0]} "
                      f"({acc['bytes'] / 1e6:.0f} MB algorithmic), {reps} repetitions in "
                      f"{dt:.1f} s; numpy float64, BLAS threads for the matmuls, elementwise "
                      "work single-threaded"}


def run_reference_sweep(args):
    """The oracle's grouped GEMM on a bounded sample of the sweep: 256 rows of the largest group
    against that group's weights, both quantized by the oracle (untimed), float64 matmul per step."""
    import numpy as np

    from oracle import moe as M
    from oracle import quant as Q
    from synth import CONFIGS, gen_weight_expert
    from synth.inputs import gen_sweep, gen_sweep_a
    cfg = CONFIGS["sweep"]
    m = gen_sweep(cfg)
    g = int(np.argmax(m))
    n = min(256, m[g])
    r0 = sum(m[:g])
    a = gen_sweep_a(cfg, r0 + n)[r0:].to(__import__("torch").bfloat16).float().numpy()
    gs_a = Q.global_scale(a)
    a_deq = Q.dequantize(*Q.quantize(a, gs_a), gs_a)
    wq = M.QuantWeights.from_float(gen_weight_expert(cfg.seed, 1, g, cfg.N, cfg.K).float().numpy()[None])
    b = wq.dequant(0)
    flops = 2 * n * cfg.N * cfg.K
    for _ in range(args.warmup):
        a_deq @ b.T
    t0 = time.perf_counter()
    for _ in range(args.steps):
        a_deq @ b.T
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = f"each step: {n} rows of group {g} x {cfg.N} x {cfg.K}, float64 matmul of the decoded operands"
    print(json.dumps({
        "impl": "reference", "metric": SWEEP_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"grouped GEMM sweep: E={cfg.E} groups, M_g ~ U{{0..{cfg.m_max}}}, "
                               f"K={cfg.K}, N={cfg.N}, bf16 out"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def run_reference(args):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    if args.config == "sweep":
        run_reference_sweep(args)
        return
    import torch
    cfg = make_config(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    from synth import gen_logits, gen_x
    logits_cpu, x_cpu = gen_logits(cfg), gen_x(cfg)
    run, acc, experts = _oracle_sample(cfg, logits_cpu, x_cpu, dev)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = acc["bytes"] * args.steps / dt / 1e9
    sample = (f"each step: token 0 of {cfg.T} of the {cfg.name} workload through {len(experts)} "
              f"of its experts ({acc['bytes'] / 1e6:.0f} MB algorithmic)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} MoE FFN: T={cfg.T}, H={cfg.H}, I={cfg.I}, E={cfg.E}, "
                               f"top-{cfg.k} ({cfg.logits} logits)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": _threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- sweep

SWEEP_METRIC = "grouped GEMM TFLOP/s on 1 B200 (NVFP4 2D x 3D, bf16 out), % of NVFP4 tensor peak"


def sweep_operands(cfg, dev):
    """Group sizes, 128-padded offsets and NVFP4 operands of the grouped-GEMM sweep: A rows
    N(0,1) (zero padding rows), B = per-group weights N(0,0.02), both quantized on the GPU."""
    import torch

    import nvfp4_block_scaled_gsa_b200 as nv
    from synth import gen_weight_expert
    from synth.inputs import gen_sweep, gen_sweep_a
    m = gen_sweep(cfg)
    pad = [(x + 127) // 128 * 128 for x in m]
    offs_l = [0]
    for p_ in pad:
        offs_l.append(offs_l[-1] + p_)
    R = offs_l[-1]
    a_rows = gen_sweep_a(cfg, sum(m), device=dev).to(torch.bfloat16)
    a = torch.zeros(R, cfg.K, dtype=torch.bfloat16, device=dev)
    r0 = 0
    for g, mg in enumerate(m):
        a[offs_l[g]:offs_l[g] + mg] = a_rows[r0:r0 + mg]
        r0 += mg
    w = nv.quantize_weights(lambda e: gen_weight_expert(cfg.seed, 1, e, cfg.N, cfg.K, device=dev),
                            cfg.E, cfg.N, cfg.K, device=dev)
    offs = torch.tensor(offs_l, dtype=torch.int32, device=dev)
    return m, offs, a, w


def run_sweep(args):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_gsa_b200 as nv
    from synth import CONFIGS
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = make_config(args)  # the sweep, or a reduced one with --experts (profiling captures)
    m, offs, a_bf16, w = sweep_operands(cfg, dev)
    R = a_bf16.shape[0]
    codes, sf, gs = nv.quantize(a_bf16)
    out = torch.empty(R, cfg.N, dtype=torch.bfloat16, device=dev)
    flops = 2 * sum(m) * cfg.N * cfg.K

    def step():
        nv.grouped_gemm(codes, sf, gs, w, offs, out_dtype=torch.bfloat16, out=out)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(8):
            step()
        torch.cuda.synchronize()
    K = args.steps
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    start.record()
    for _ in range(K):
        step()
    stop.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    total_ms = slowest_rank_ms(start.elapsed_time(stop), world, dev)
    ms = total_ms / K
    value = whole_job_rate(flops, K, world, total_ms) / 1e12

    # end to end: bf16 A from pinned host memory, quantize, GEMM, bf16 result back to the host
    a_h = a_bf16.cpu().pin_memory()
    out_h = torch.empty(R, cfg.N, dtype=torch.bfloat16).pin_memory()
    a_d = torch.empty_like(a_bf16)

    def e2e_step():
        a_d.copy_(a_h, non_blocking=True)
        c2, s2_, g2 = nv.quantize(a_d)
        nv.grouped_gemm(c2, s2_, g2, w, offs, out_dtype=torch.bfloat16, out=out)
        out_h.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ke = max(1, min(K, 5))
    e0.record()
    for _ in range(ke):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / ke
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = sweep_cpu_baseline(cfg, m, offs, codes, sf, gs, w)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks = load_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    line = {
        "metric": SWEEP_METRIC, "value": round(value, 1), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 + e4m3/16), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) A rows, N(0,0.02) weights, quantized on the GPU)",
        "config": {"workload": f"grouped GEMM sweep: E={cfg.E} groups, M_g ~ U{{0..{cfg.m_max}}} "
                               f"(sum {sum(m)}), K={cfg.K}, N={cfg.N}, bf16 out",
                   "parallelism": f"replicas x{world}",
                   "l2": "no flush: A (NVFP4, %.0f MB) + B (%.0f MB) > 126 MB L2" % (
                       R * cfg.K * FP4_ELEM_BYTES / 1e6, cfg.E * cfg.N * cfg.K * FP4_ELEM_BYTES / 1e6)},
        "roofline": {"bound": "tensor", "kernel": "grouped_gemm_kernel<PLAIN_BF16>",
                     "achieved": round(value / world, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(value / world / fp4_peak, 4), "traffic": None,
                     "algorithmic_flops_per_launch": int(flops),
                     "peak_source": f"{peaks['src']} bf16 burst x {FP4_PER_BF16} (nominal FP4/BF16 "
                                    "dense ratio)"},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
                "h2d_bytes_per_step": a_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": K,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _sweep_oracle_sample(cfg, m, offs, codes, sf, gs, w, rows=4096):
    """The oracle's grouped GEMM on (up to `rows` rows of) the largest group, decoded from the
    same NVFP4 operands the GPU used."""
    import numpy as np

    from oracle import quant as Q
    g = int(np.argmax(m))
    o = int(offs[g])
    n = min(rows, m[g])
    K, N = cfg.K, cfg.N
    cols = np.arange(K // 16)

    def scales(flat, r0, nrows):
        rr, cc = np.meshgrid(np.arange(r0, r0 + nrows), cols, indexing="ij")
        return flat[Q.sf_tile_offset(rr, cc, K // 16)]

    a = Q.dequantize_packed(codes[o:o + n].cpu().numpy(), scales(sf.cpu().numpy(), o, n),
                           float(gs.item()))
    b = Q.dequantize_packed(w.codes[g * N:(g + 1) * N].cpu().numpy(),
                            scales(w.sf.cpu().numpy(), g * N, N), float(w.gs[g].item()))

    def run():
        return a @ b.T

    return run, 2 * n * N * K, n, g


def sweep_cpu_baseline(cfg, m, offs, codes, sf, gs, w):
    run, flops, n, g = _sweep_oracle_sample(cfg, m, offs, codes, sf, gs, w)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(),
            "kind": "oracle",
            "sample": f"{n} rows of group {g} x {cfg.N} x {cfg.K} (float64 matmul of the decoded "
                      f"NVFP4 operands) in {dt:.2f} s"}


# ----------------------------------------------------------------------------- dense linear

DENSE_METRIC = ("dense NVFP4 linear (RMSNorm fused) on 1 B200, % of NVFP4 tensor/HBM roofline")
L2_FLUSH_BYTES = 256 << 20  # written between steps: larger than the 126 MB L2


def dense_algorithmic(cfg):
    """Bytes and FLOPs of one dense step and of its GEMM launch: x read as bf16 (and gamma),
    activation codes written and read once, weight codes + scales read once, bf16 out written."""
    a_q = cfg.M * cfg.K * FP4_ELEM_BYTES
    w_q = cfg.N * cfg.K * FP4_ELEM_BYTES
    out = cfg.M * cfg.N * 2
    return dict(flops=cfg.flops(), bytes=cfg.M * cfg.K * 2 + cfg.K * 2 + 2 * a_q + w_q + out,
                gemm_bytes=a_q + w_q + out)


def dense_operands(cfg, dev):
    import torch

    import nvfp4_block_scaled_gsa_b200 as nv
    from synth import gen_dense
    x, gamma, w = gen_dense(cfg, device=dev)
    wd = nv.quantize_weights(lambda e: w, 1, cfg.N, cfg.K, device=dev)
    return x, gamma.to(dev), wd, torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)


def _timed_steps(step, flush, K):
    """Device time of K steps, each timed by its own pair of events after an L2 flush."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    for a, b in evs:
        flush.zero_()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs)


def run_dense(args):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_gsa_b200 as nv
    from synth import CONFIGS
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = CONFIGS[args.config]
    x_cpu, gamma, wd, flush = dense_operands(cfg, dev)
    x = x_cpu.to(dev)
    out = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.linear_workspace_bytes(cfg.M, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    acc = dense_algorithmic(cfg)

    def step():
        nv.linear(x, wd, gamma=gamma, eps=cfg.eps, out=out, ws=ws, status=status)

    # the step as a CUDA graph (one launch of its 3-4 kernels: no host gaps at decode sizes)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(8):
            graph.replay()
        torch.cuda.synchronize()
    K = args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    total_ms = _timed_steps(graph.replay, flush, K)
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    eager_ms = _timed_steps(step, flush, max(1, min(K, 50)))
    eager_ms /= max(1, min(K, 50))

    # the GEMM stage alone (the dominant kernel, plus its split-K reduction), on the codes the
    # fused quantizer wrote
    Mp = (cfg.M + 127) // 128 * 128
    codes, sf, gs = nv.rmsnorm_quantize(x, gamma, cfg.eps, out_rows=Mp)
    gws_n = int(nv.lib().nvfp4_gemm_dense_workspace_size(cfg.M, cfg.N, cfg.K))
    gws = torch.empty(max(gws_n, 256), dtype=torch.uint8, device=dev)
    kg = max(1, min(K, 50))

    def gemm_stage():
        nv.gemm_dense(codes, sf, gs, cfg.M, wd, out=out, ws=gws)

    gemm_stage()
    torch.cuda.synchronize()
    g_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_graph, capture_error_mode="thread_local"):
        gemm_stage()
    gemm_ms = _timed_steps(g_graph.replay, flush, kg) / kg
    split = nv.lib().nvfp4_gemm_dense_workspace_size(cfg.M, cfg.N, cfg.K) > 0
    code, rc = nv.read_status(status)
    if code != 0:
        raise RuntimeError(f"device status {code} after the timed region")

    total_ms = slowest_rank_ms(total_ms, world, dev)
    ms_step = total_ms / K
    gbs = whole_job_rate(acc["bytes"], K, world, total_ms) / 1e9
    tflops = whole_job_rate(acc["flops"], K, world, total_ms) / 1e12

    # end to end through nvfp4_linear: x from pinned host memory, bf16 result back to the host
    x_h = x_cpu.pin_memory()
    out_h = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(x)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        nv.linear(x_d, wd, gamma=gamma, eps=cfg.eps, out=out, ws=ws, status=status)
        out_h.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ke = max(1, min(K, 50))
    e2e_ms = slowest_rank_ms(_timed_steps(e2e_step, flush, ke), world, dev) / ke

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = dense_cpu_baseline(cfg)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks = load_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    tensor_bound = acc["flops"] / acc["gemm_bytes"] > fp4_peak * 1e12 / (peaks["hbm"] * 1e9)
    kname = "grouped_gemm_kernel<PLAIN_F32> + splitk_reduce_kernel" if split else \
        "grouped_gemm_kernel<PLAIN_BF16>"
    g_tflops = acc["flops"] / (gemm_ms * 1e-3) / 1e12
    g_gbs = acc["gemm_bytes"] / (gemm_ms * 1e-3) / 1e9
    if tensor_bound:
        value, unit = tflops, "TFLOP/s"
        roof = {"bound": "tensor", "kernel": kname, "achieved": round(g_tflops, 1),
                "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(g_tflops / fp4_peak, 4),
                "traffic": None, "algorithmic_flops_per_launch": int(acc["flops"]),
                "peak_source": f"{peaks['src']} bf16 burst x {FP4_PER_BF16} (nominal FP4/BF16 "
                               "dense ratio)",
                "step_frac": round(tflops / world / fp4_peak, 4)}
    else:
        value, unit = gbs, "GB/s"
        roof = {"bound": "hbm", "kernel": kname, "achieved": round(g_gbs, 1),
                "peak": peaks["hbm"], "unit": "GB/s", "frac": round(g_gbs / peaks["hbm"], 4),
                "traffic": None, "algorithmic_bytes_per_launch": int(acc["gemm_bytes"]),
                "peak_source": peaks["src"], "step_frac": round(gbs / world / peaks["hbm"], 4)}
    e2e_rate = (world * acc["flops"] / (e2e_ms * 1e-3) / 1e12 if tensor_bound
                else world * acc["bytes"] / (e2e_ms * 1e-3) / 1e9)
    line = {
        "metric": DENSE_METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + e4m3/16), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) bf16 activations, gamma 1 + 0.1 N(0,1), N(0,0.02) "
                "weight quantized to NVFP4 on the GPU)",
        "config": {"workload": f"{cfg.name}: RMSNorm + dense NVFP4 linear, M={cfg.M}, "
                               f"K={cfg.K}, N={cfg.N}, bf16 out",
                   "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (256 MB write, outside the timed events)",
                   "cuda_graph": True, "k_splits": bool(split)},
        "tflops": round(tflops, 3), "gbs": round(gbs, 2),
        "algorithmic": {"bytes_per_step": int(acc["bytes"]), "flops_per_step": int(acc["flops"]),
                        "gemm_bytes_per_launch": int(acc["gemm_bytes"])},
        "roofline": roof,
        "stages_ms": {"gemm": round(gemm_ms, 5), "eager_step": round(eager_ms, 5)},
        "e2e": {"value": round(e2e_rate, 2), "unit": unit,
                "h2d_bytes_per_step": x_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": (4 if split else 3) * K,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _dense_oracle_sample(cfg, rows=16):
    """The oracle's RMSNorm + linear on the first `rows` rows of the workload (the global scale
    then comes from those rows' amax); weight pre-packing by the oracle, untimed."""
    from oracle import dense as D
    from oracle import formats as F
    from oracle import moe as M
    from synth import gen_dense
    x, gamma, w = gen_dense(cfg)
    x = x[:rows].float().numpy()
    g = gamma.float().numpy()
    qw = M.QuantWeights.from_float(w.float().numpy()[None])
    wc = F.unpack_nibbles(qw.codes[0])

    def run():
        y, _ = D.rmsnorm(x, g, cfg.eps)
        return D.linear(y, wc, qw.sf[0], qw.gs[0])

    n = x.shape[0]
    flops = 2 * n * cfg.N * cfg.K
    nbytes = n * cfg.K * 2 + cfg.K * 2 + 2 * n * cfg.K * FP4_ELEM_BYTES + \
        cfg.N * cfg.K * FP4_ELEM_BYTES + n * cfg.N * 2
    return run, flops, nbytes, n


def dense_cpu_baseline(cfg):
    run, flops, nbytes, n = _dense_oracle_sample(cfg)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= 10.0:
            break
    unit = "GB/s" if cfg.M <= 128 else "TFLOP/s"
    val = nbytes * reps / dt / 1e9 if unit == "GB/s" else flops * reps / dt / 1e12
    return {"value": round(val, 6), "unit": unit, "cores": _threads(), "kind": "oracle",
            "sample": f"first {n} rows of {cfg.name}: RMSNorm, quantize, decode and float64 matmul "
                      f"against the {cfg.N} x {cfg.K} weight, {reps} repetitions in {dt:.1f} s"}


def run_reference_dense(args):
    from synth import CONFIGS
    cfg = CONFIGS[args.config]
    run, flops, nbytes, n = _dense_oracle_sample(cfg)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    unit = "GB/s" if cfg.M <= 128 else "TFLOP/s"
    value = nbytes * args.steps / dt / 1e9 if unit == "GB/s" else flops * args.steps / dt / 1e12
    sample = f"each step: the first {n} rows of {cfg.name} through the oracle's RMSNorm + linear"
    print(json.dumps({
        "impl": "reference", "metric": DENSE_METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: RMSNorm + dense NVFP4 linear, M={cfg.M}, "
                               f"K={cfg.K}, N={cfg.N}, bf16 out"},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": _threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


# ----------------------------------------------------------------------------- shared expert

SHARED_METRIC = "MoE shared expert (RMSNorm fused) on 1 B200, % of NVFP4 tensor/HBM roofline"


def shared_algorithmic(cfg):
    """Bytes and FLOPs of one shared-expert step and of its L1 launch: x read as bf16 (and
    gamma), x codes written and read once, W1 and W2 codes + scales read once, h codes written
    and read once, bf16 out written."""
    M, H, I = cfg.M, cfg.H, cfg.I
    x_q = M * H * FP4_ELEM_BYTES
    h_q = M * I * FP4_ELEM_BYTES
    w1 = 2 * I * H * FP4_ELEM_BYTES
    w2 = H * I * FP4_ELEM_BYTES
    return dict(flops=cfg.flops(), bytes=M * H * 2 + H * 2 + 2 * x_q + w1 + 2 * h_q + w2 + M * H * 2,
                l1_flops=2 * M * H * 2 * I, l1_bytes=x_q + w1 + h_q)


def run_shared(args):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_gsa_b200 as nv
    from nvfp4_block_scaled_gsa_b200._native import call
    from synth import CONFIGS, gen_shared
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = CONFIGS[args.config]
    x_cpu, gamma, w1f, w2f = gen_shared(cfg, device=dev)
    gamma = gamma.to(dev)
    w1 = nv.quantize_w1(lambda e: w1f, 1, cfg.I, cfg.H, device=dev)
    w2 = nv.quantize_weights(lambda e: w2f, 1, cfg.H, cfg.I, device=dev)
    del w1f, w2f
    gs_h = torch.tensor([cfg.gs_h], dtype=torch.float32, device=dev)
    x = x_cpu.to(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = torch.empty(cfg.M, cfg.H, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.shared_expert_workspace_bytes(cfg.M, cfg.H, cfg.I), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    acc = shared_algorithmic(cfg)

    def step():
        nv.shared_expert(x, w1, w2, gs_h, gamma=gamma, eps=cfg.eps, out=out, ws=ws, status=status)

    def graph_of(fn):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        torch.cuda.synchronize()
        return g

    for _ in range(max(args.warmup, 3)):
        step()
    graph = graph_of(step)
    sampler = ClockSampler(local) if rank == 0 else None
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(8):
            graph.replay()
        torch.cuda.synchronize()
    K = args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    total_ms = _timed_steps(graph.replay, flush, K)
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()

    # the L1 stage alone (the dominant kernel), on the codes the fused quantizer wrote, in the
    # form the step runs: with few rows the L1 GEMM is split along K (FP32 partials, then an
    # ordered sum; timed here with the bf16 reduction in place of the SwiGLU kernel), otherwise
    # the fused GEMM + SwiGLU + FP4 epilogue over one dense segment (offsets [0, rows])
    Mp = (cfg.M + 127) // 128 * 128
    codes, sf, gs = nv.rmsnorm_quantize(x, gamma, cfg.eps, out_rows=Mp)
    l1_split = nv.lib().nvfp4_gemm_dense_workspace_size(cfg.M, 2 * cfg.I, cfg.H) > 0
    if l1_split:
        g_ws = torch.empty(int(nv.lib().nvfp4_gemm_dense_workspace_size(cfg.M, 2 * cfg.I, cfg.H)),
                           dtype=torch.uint8, device=dev)
        c1 = torch.empty(cfg.M, 2 * cfg.I, dtype=torch.bfloat16, device=dev)

        def l1_stage():
            nv.gemm_dense(codes, sf, gs, cfg.M, w1, out=c1, ws=g_ws)
    else:
        offs = torch.tensor([0, Mp], dtype=torch.int32, device=dev)
        hq = torch.empty(Mp, cfg.I // 2, dtype=torch.uint8, device=dev)
        hsf = torch.empty(nv.sf_bytes(Mp, cfg.I), dtype=torch.uint8, device=dev)
        s_ = lambda: torch.cuda.current_stream().cuda_stream  # noqa: E731

        def l1_stage():
            call("moe_grouped_gemm_l1_swiglu_q", codes.data_ptr(), sf.data_ptr(), gs.data_ptr(),
                 w1.codes.data_ptr(), w1.sf.data_ptr(), w1.gs.data_ptr(), offs.data_ptr(), None,
                 1, cfg.H, cfg.I, Mp, gs_h.data_ptr(), hq.data_ptr(), hsf.data_ptr(),
                 status.data_ptr(), s_())

    kg = max(1, min(K, 50))
    l1_ms = _timed_steps(graph_of(l1_stage).replay, flush, kg) / kg
    code, rc = nv.read_status(status)
    if code != 0:
        raise RuntimeError(f"device status {code} after the timed region")

    total_ms = slowest_rank_ms(total_ms, world, dev)
    ms_step = total_ms / K
    gbs = whole_job_rate(acc["bytes"], K, world, total_ms) / 1e9
    tflops = whole_job_rate(acc["flops"], K, world, total_ms) / 1e12

    x_h = x_cpu.pin_memory()
    out_h = torch.empty(cfg.M, cfg.H, dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(x)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        nv.shared_expert(x_d, w1, w2, gs_h, gamma=gamma, eps=cfg.eps, out=out, ws=ws,
                         status=status)
        out_h.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ke = max(1, min(K, 50))
    e2e_ms = slowest_rank_ms(_timed_steps(e2e_step, flush, ke), world, dev) / ke

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = shared_cpu_baseline(cfg)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks = load_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    tensor_bound = acc["l1_flops"] / acc["l1_bytes"] > fp4_peak * 1e12 / (peaks["hbm"] * 1e9)
    l1_tf = acc["l1_flops"] / (l1_ms * 1e-3) / 1e12
    l1_gb = acc["l1_bytes"] / (l1_ms * 1e-3) / 1e9
    kname = ("grouped_gemm_kernel<PLAIN_F32> (L1, split along K) + reduction" if l1_split
             else "grouped_gemm_kernel<L1_SWIGLU>")
    if tensor_bound:
        value, unit = tflops, "TFLOP/s"
        roof = {"bound": "tensor", "kernel": kname, "achieved": round(l1_tf, 1),
                "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(l1_tf / fp4_peak, 4),
                "traffic": None, "algorithmic_flops_per_launch": int(acc["l1_flops"]),
                "peak_source": f"{peaks['src']} bf16 burst x {FP4_PER_BF16} (nominal FP4/BF16 "
                               "dense ratio)",
                "step_frac": round(tflops / world / fp4_peak, 4)}
    else:
        value, unit = gbs, "GB/s"
        roof = {"bound": "hbm", "kernel": kname, "achieved": round(l1_gb, 1),
                "peak": peaks["hbm"], "unit": "GB/s", "frac": round(l1_gb / peaks["hbm"], 4),
                "traffic": None, "algorithmic_bytes_per_launch": int(acc["l1_bytes"]),
                "peak_source": peaks["src"], "step_frac": round(gbs / world / peaks["hbm"], 4)}
    e2e_rate = (world * acc["flops"] / (e2e_ms * 1e-3) / 1e12 if tensor_bound
                else world * acc["bytes"] / (e2e_ms * 1e-3) / 1e9)
    split = nv.lib().nvfp4_gemm_dense_workspace_size(cfg.M, cfg.H, cfg.I) > 0
    line = {
        "metric": SHARED_METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + e4m3/16), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) bf16 activations, gamma 1 + 0.1 N(0,1), N(0,0.02) "
                "weights quantized to NVFP4 on the GPU)",
        "config": {"workload": f"{cfg.name}: RMSNorm + shared expert FFN, M={cfg.M}, "
                               f"H={cfg.H}, I={cfg.I}, bf16 out",
                   "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (256 MB write, outside the timed events)",
                   "cuda_graph": True, "l1_k_splits": bool(l1_split),
                   "down_projection_k_splits": bool(split)},
        "tflops": round(tflops, 3), "gbs": round(gbs, 2),
        "algorithmic": {"bytes_per_step": int(acc["bytes"]), "flops_per_step": int(acc["flops"]),
                        "l1_bytes_per_launch": int(acc["l1_bytes"])},
        "roofline": roof,
        "stages_ms": {"l1_gemm_swiglu_q": round(l1_ms, 5)},
        "e2e": {"value": round(e2e_rate, 2), "unit": unit,
                "h2d_bytes_per_step": x_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": (4 + (1 if split else 0) + (1 if l1_split else 0)) * K,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _shared_oracle_sample(cfg, rows=4):
    """The oracle's shared expert on the first `rows` rows (their own global scale); weight
    pre-packing by the oracle, untimed."""
    from oracle import dense as D
    from oracle import moe as M
    from synth import gen_shared
    x, gamma, w1, w2 = gen_shared(cfg)
    x = x[:rows].float().numpy()
    g = gamma.float().numpy()
    q1 = M.QuantWeights.from_float(w1.float().numpy()[None])
    q2 = M.QuantWeights.from_float(w2.float().numpy()[None])

    def run():
        return D.shared_expert(x, q1, q2, cfg.gs_h, gamma=g, eps=cfg.eps)

    n = x.shape[0]
    flops = 6 * n * cfg.H * cfg.I
    nbytes = (n * cfg.H * 2 + cfg.H * 2 + 2 * n * cfg.H * FP4_ELEM_BYTES
              + 3 * cfg.I * cfg.H * FP4_ELEM_BYTES + 2 * n * cfg.I * FP4_ELEM_BYTES
              + n * cfg.H * 2)
    return run, flops, nbytes, n


def shared_cpu_baseline(cfg):
    run, flops, nbytes, n = _shared_oracle_sample(cfg)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= 10.0:
            break
    unit = "GB/s" if cfg.M <= 128 else "TFLOP/s"
    val = nbytes * reps / dt / 1e9 if unit == "GB/s" else flops * reps / dt / 1e12
    return {"value": round(val, 6), "unit": unit, "cores": _threads(), "kind": "oracle",
            "sample": f"first {n} rows of {cfg.name} through the oracle's RMSNorm + shared expert, "
                      f"{reps} repetitions in {dt:.1f} s"}


def run_reference_shared(args):
    from synth import CONFIGS
    cfg = CONFIGS[args.config]
    run, flops, nbytes, n = _shared_oracle_sample(cfg)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    unit = "GB/s" if cfg.M <= 128 else "TFLOP/s"
    value = nbytes * args.steps / dt / 1e9 if unit == "GB/s" else flops * args.steps / dt / 1e12
    sample = f"each step: the first {n} rows of {cfg.name} through the oracle's shared expert"
    print(json.dumps({
        "impl": "reference", "metric": SHARED_METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: RMSNorm + shared expert FFN, M={cfg.M}, "
                               f"H={cfg.H}, I={cfg.I}, bf16 out"},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": _threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def main():
    args = parse()
    dense = args.config.startswith("dense_")
    shared = args.config.startswith("shared_")
    if args.impl == "reference":
        if dense or shared:
            if int(os.environ.get("RANK", 0)) == 0:
                (run_reference_dense if dense else run_reference_shared)(args)
        else:
            run_reference(args)
    elif args.config == "sweep":
        run_sweep(args)
    elif dense:
        run_dense(args)
    elif shared:
        run_shared(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
