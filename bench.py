"""Throughput of the Hiera-B+ backbone forward (512x512x4 images, bf16) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One forward = the whole backbone (patch embedding + pos_embed + Unroll, 24 blocks, Reroll
of the four stage features) over one batch of 8 synthetic images per GPU, replayed from a
CUDA graph of the library's launches. One step = R consecutive forwards (R chosen from the
warm-up so that the K timed steps last about a second: enough clock samples under load).
Inputs are resident in HBM when a timed step starts; L2 is flushed (256 MiB write) before
every step, and inside a step each forward's working set (138 MB of weights plus its
activations) exceeds the 126 MB L2. Steps are timed with CUDA events on the launching
stream; the timed value sums the K step windows and takes the max over ranks. Multi-GPU
runs are independent replicas (one batch per rank, no collective on the data path):
value = all images / max time.

Rank 0 prints one JSON line with the headline images/s, the roofline of the dominant
kernel (the launch shape with the largest share of the forward, timed with per-launch
CUDA events inside a separately captured graph of the same forward) against the burst
bf16 peak, the end-to-end number through the public API with host buffers, SM clocks
sampled during the timed region, the batch-1 latency of the same forward, the 2048^2
batch-1 throughput, and the CPU oracle timed on a bounded sample.

--impl reference times the CPU oracle (fp64 numpy, formulation U) on the same metric:
each step is one 512^2 image through the whole backbone; the number of steps is capped
so that the run ends within a few minutes.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "Hiera-B+ backbone images/s (512², bf16, 1 B200); attn+GEMM % of BF16 peak"
UNIT = "images/s"
IMG = 512
BATCH = 8
SEED = 3
L2_FLUSH_BYTES = 256 << 20
STAGE_DIMS = (112, 224, 448, 896)
STAGE_HEADS = (2, 4, 8, 16)
STAGE_DEPTHS = (2, 3, 16, 3)
HD = 56


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]),
                "measured")
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a kernel shape,
# from one ncu capture of one launch of that shape in this workload; the summaries under
# profiles/ give the commands. Keyed by (kernel kind, GFLOP per launch rounded to 0.01). A
# shape missing here reports traffic null; an entry must be removed whenever its kernel
# changes.
DRAM_BYTES_PER_LAUNCH = {
    # stage-2 global attention, 8 x 8 x 1024 x 1024 (profiles/attention_tcgen05_stage2_512_b8.md)
    ("attention_tcgen05", 15.03): 25_421_056,
}


def reroll_bytes(img: int, B: int):
    """Algorithmic bytes (read + write, bf16) of the four feature Rerolls, in launch order."""
    G0 = img // 4
    return [2 * 2 * B * (G0 >> s) ** 2 * STAGE_DIMS[s] for s in range(4)]


def launch_flops(img: int, B: int, fused_mlp: bool = True, fused_attn: bool = True):
    """Algorithmic FLOPs of every library launch of one backbone forward, in launch order
    (head_dim 56, not the padded 64). Returns list of (kind-class, flops). With fused_mlp,
    the MLPs of dims 112 and 224 are one launch (fc1 + fc2 FLOPs); with fused_attn, the
    stage-0 blocks' qkv, attention and proj are one launch (class attn_block)."""
    G0 = img // 4
    out = [("patch_embed", 2.0 * B * G0 * G0 * 112 * 196)]
    prev = STAGE_DIMS[0]
    i = 0
    for s, depth in enumerate(STAGE_DEPTHS):
        Gs = G0 >> s
        for j in range(depth):
            trans = s > 0 and j == 0
            d_in = prev if trans else STAGE_DIMS[s]
            d = STAGE_DIMS[s]
            n_in = (2 * Gs) ** 2 if trans else Gs * Gs
            nq = Gs * Gs
            mua = s < 2
            flat_mu = 64 >> (2 * s)
            window = flat_mu * (4 if trans else 1)
            nW = n_in // window if mua else 1
            tkv = n_in // nW
            tq = tkv // (4 if trans else 1)
            n1 = 3 * d + (d if trans else 0)
            qkv = 2.0 * B * n_in * d_in * n1
            attn = 4.0 * B * STAGE_HEADS[s] * nW * tq * tkv * HD
            proj = 2.0 * B * nq * d * d
            if fused_attn and s == 0 and nW % 2 == 0:
                out.append(("attn_block", qkv + attn + proj))
            else:
                out.append(("gemm", qkv))
                out.append(("attention", attn))
                out.append(("gemm", proj))
            if fused_mlp and d in (112, 224):
                out.append(("gemm", 4.0 * B * nq * d * 4 * d))
            else:
                out.append(("gemm", 2.0 * B * nq * d * 4 * d))
                out.append(("gemm", 2.0 * B * nq * 4 * d * d))
            if i in (1, 4, 20, 23):
                out.append(("unroll_reroll", 0.0))
            i += 1
        prev = STAGE_DIMS[s]
    return out


KIND_CLASS = {"patch_embed": "patch_embed", "unroll_reroll": "unroll_reroll",
              "gemm_qkv_lnfold": "gemm", "gemm_fc1_lnfold_gelu": "gemm",
              "gemm_bias_residual": "gemm", "attention_window": "attention",
              "attention_tcgen05": "attention", "mlp_fused": "gemm",
              "attention_block_fused": "attn_block"}
TENSOR_CLASSES = ("gemm", "attention", "attn_block")

KIND_DESCRIPTION = {
    "gemm_qkv_lnfold": "tcgen05 GEMM: norm1 folded, qkv (+ transition proj) with window scatter",
    "gemm_fc1_lnfold_gelu": "tcgen05 GEMM: norm2 folded, fc1 + GELU",
    "gemm_bias_residual": "tcgen05 GEMM: attention proj or fc2, + bias + residual",
    "mlp_fused": "tcgen05 fused MLP (norm2, fc1, GELU, fc2, residual)",
    "attention_tcgen05": "tcgen05 attention, 128-key tiles (global attention)",
    "attention_window": "tcgen05 attention, several mask-unit windows per tile",
    "attention_block_fused": "stage-0 attention half in one kernel (norm1, qkv, windowed "
                             "attention, proj, residual; tcgen05)",
}


def shape_breakdown(per_launch, flops, tf_burst, tf_sust):
    """Group launches by (kind, GFLOP per launch): the shapes a forward is made of."""
    shapes = {}
    for (n, ms), (c, fl) in zip(per_launch, flops):
        key = (n, round(fl / 1e9, 2))
        e = shapes.setdefault(key, {"kind": n, "class": c, "launches": 0, "ms": 0.0,
                                    "gflop": 0.0})
        e["launches"] += 1
        e["ms"] += ms
        e["gflop"] += fl / 1e9
    for e in shapes.values():
        e["tflops"] = e["gflop"] / e["ms"] if e["ms"] > 0 else 0.0
        e["frac_of_bf16_burst"] = e["tflops"] / tf_burst
        e["frac_of_bf16_sustained"] = e["tflops"] / tf_sust
    return shapes


def time_steps(graph, stream, flush, steps, replays):
    """K steps of `replays` graph replays each, L2 flushed before every step; per-step ms."""
    import torch
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(steps):
            flush.fill_(k & 0xFF)
            starts[k].record(stream)
            for _ in range(replays):
                graph.replay()
            ends[k].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(starts, ends)]


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clock record
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        return False

    def record(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for bit, n in self.REASONS.items() if self.reasons & bit]}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_images_per_s(budget_s: float, max_steps: int, warmup: int):
    """Time the CPU oracle: each step one 512^2 image through the whole backbone."""
    from mask_unit_windowed_b200 import synthetic as syn
    from oracle import unrolled as U
    p = syn.backbone_params(SEED, IMG, dtype="bf16")
    img = syn.image(SEED, 1, IMG)
    for _ in range(min(warmup, 1)):
        U.backbone_forward(img, p)
    times = []
    t_start = time.perf_counter()
    while len(times) < max_steps:
        t0 = time.perf_counter()
        U.backbone_forward(img, p)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start + times[-1] > budget_s:
            break
    return len(times) / sum(times), len(times)


def run_reference(args, rank: int):
    if rank != 0:
        return
    value, steps = oracle_images_per_s(150.0, args.steps, args.warmup)
    cores = blas_threads()
    cpu = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"{steps} step(s) of one {IMG}x{IMG}x4 image through the full backbone "
                     "(fp64 numpy oracle, unrolled formulation)"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": steps, "warmup": min(args.warmup, 1),
            "ms_per_step": 1000.0 / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"Hiera-B+ backbone forward, {IMG}x{IMG}x4 bf16 images, "
                                   f"batch {args.batch} per GPU (random-init weights, seed "
                                   f"{SEED})", "img": IMG, "batch_per_gpu": args.batch,
                       "global_batch": args.batch,
                       "sample": "each timed step runs one image of the batch through the "
                                 "CPU oracle (bf16-valued inputs, fp64 arithmetic)"},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _weights_dev(params, dev):
    import torch

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev, torch.bfloat16)

    return {"patch_w": t(params["patch_w"]), "patch_b": t(params["patch_b"]),
            "pos_embed": t(params["pos_embed"]),
            "blocks": [{k: t(v) for k, v in blk.items()} for blk in params["blocks"]]}


def _graph_of(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


def extra_forward_timing(hb, syn, dev, stream, flush, img, B, seed, reps):
    """ms per forward of the backbone at (img, B), CUDA graph, L2 flushed before each
    forward, median of `reps`; also returns the algorithmic GFLOP per forward."""
    import torch
    params = syn.backbone_params(seed, img, dtype="bf16")
    desc = hb.BackboneDesc(B=B, img=img)
    packed = hb.backbone_pack(desc, _weights_dev(params, dev))
    del params
    x = torch.from_numpy(syn.image(seed, B, img)).to(dev, torch.bfloat16)
    feats = [torch.empty(sh, dtype=torch.bfloat16, device=dev) for sh in desc.feature_shapes()]
    ws = torch.empty(hb.backbone_workspace_bytes(desc), dtype=torch.uint8, device=dev)

    def fwd():
        hb.backbone_forward(desc, packed, x, feats=feats, workspace=ws)

    with torch.cuda.stream(stream):
        fwd()
    torch.cuda.synchronize()
    if hb.device_status(stream) != 0:
        raise RuntimeError("device status after the extra forward")
    g = _graph_of(fwd, stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    ms = sorted(time_steps(g, stream, flush, reps, 1))
    if hb.device_status(stream) != 0:
        raise RuntimeError("device status after the extra timing")
    gflop = sum(fl for _, fl in launch_flops(img, B)) / 1e9
    del g, packed, ws, feats, x
    torch.cuda.synchronize()
    return ms[len(ms) // 2], gflop


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from mask_unit_windowed_b200 import binding as hb
    from mask_unit_windowed_b200 import replicas
    from mask_unit_windowed_b200 import synthetic as syn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    hb.set_option(hb.OPT_FUSED_MLP, 1 if args.mlp == "fused" else 0)
    hb.set_option(hb.OPT_PDL, 1 if args.pdl == "on" else 0)
    hb.set_option(hb.OPT_FUSED_ATTN, 1 if args.attn == "fused" else 0)
    hb.set_option(hb.OPT_SPLIT_BATCH, 1 if args.split == "on" else 0)
    if args.gemm224 != "default":
        hb.set_option(hb.OPT_GEMM224, {"8warp": hb.GEMM224_EIGHT_WARPS,
                                       "16warp": hb.GEMM224_SIXTEEN_WARPS,
                                       "pair": hb.GEMM224_PAIR}[args.gemm224])
    hbm_gbs, tf_burst, tf_sust, peak_src = peaks()
    B = args.batch

    # ---- weights and inputs (synthetic, seeded; random-init Hiera-B+)
    params = syn.backbone_params(SEED, IMG, dtype="bf16")
    desc = hb.BackboneDesc(B=B, img=IMG)
    packed = hb.backbone_pack(desc, _weights_dev(params, dev))
    del params
    img_host = torch.from_numpy(syn.image(SEED + rank, B, IMG)).to(torch.bfloat16).pin_memory()
    img = img_host.to(dev)
    feats = [torch.empty(s, dtype=torch.bfloat16, device=dev) for s in desc.feature_shapes()]
    ws = torch.empty(hb.backbone_workspace_bytes(desc), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def forward():
        hb.backbone_forward(desc, packed, img, feats=feats, workspace=ws)

    with torch.cuda.stream(stream):
        forward()
    torch.cuda.synchronize()
    st = hb.device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {hb.status_string(st)}")

    # ---- CUDA graph of one forward (the library's launches only)
    graph = _graph_of(forward, stream)

    # ---- instrumented graph: an event before every launch (kernel breakdown / roofline)
    prof = hb.LaunchProfile(capacity=256, stream=stream)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=stream):
        with prof:
            forward()
    torch.cuda.synchronize()
    n_launches = prof.count
    # (the profiled forward runs as one batch: the library does not split a batch while a
    # launch profile is open; split, each half makes the same launches)
    split = args.split == "on" and B >= 2
    launches_per_forward = n_launches * (2 if split else 1)

    # ---- warm-up steps (one forward each), which also size a step: R forwards such that
    # the K timed steps last about a second
    warm = time_steps(graph, stream, flush, max(args.warmup, 3), 1)
    est_ms = statistics.median(warm)
    replays = args.replays if args.replays > 0 else \
        max(1, math.ceil(args.timed_seconds * 1e3 / (args.steps * est_ms)))

    # ---- timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        step_ms = time_steps(graph, stream, flush, args.steps, replays)
    if world > 1:
        dist.barrier()
    total_ms = sum(step_ms)
    st = hb.device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {hb.status_string(st)}")
    total_ms = replicas.max_over_ranks(total_ms, dev)
    images = B * replays * args.steps * world
    value = replicas.job_throughput(B * replays * args.steps, world, total_ms)
    ms_per_step = total_ms / args.steps
    ms_per_forward = ms_per_step / replays

    # ---- per-launch breakdown from the instrumented graph (same workload, L2 flushed)
    reps = 5
    per_launch = None
    with torch.cuda.stream(stream):
        for r in range(reps):
            flush.fill_(r)
            pgraph.replay()
            torch.cuda.synchronize()
            d = prof.durations_ms()
            per_launch = [(n, ms) for n, ms in d] if per_launch is None else \
                [(n, a + ms) for (n, a), (_, ms) in zip(per_launch, d)]
    per_launch = [(n, ms / reps) for n, ms in per_launch]
    flops = launch_flops(IMG, B, fused_mlp=hb.get_option(hb.OPT_FUSED_MLP) == 1,
                         fused_attn=hb.get_option(hb.OPT_FUSED_ATTN) == 1)
    if len(flops) != len(per_launch) or any(KIND_CLASS.get(n) != c for (n, _), (c, _) in
                                            zip(per_launch, flops)):
        raise RuntimeError("the launch sequence differs from the bench's work model")
    classes, by_kernel = {}, {}
    for (n, ms), (c, fl) in zip(per_launch, flops):
        for e in (classes.setdefault(c, {"launches": 0, "ms": 0.0, "gflop": 0.0}),
                  by_kernel.setdefault(n, {"launches": 0, "ms": 0.0, "gflop": 0.0})):
            e["launches"] += 1
            e["ms"] += ms
            e["gflop"] += fl / 1e9
    step_ms_prof = sum(ms for _, ms in per_launch)
    for e in list(classes.values()) + list(by_kernel.values()):
        e["share"] = e["ms"] / step_ms_prof if step_ms_prof > 0 else None
        e["tflops"] = e["gflop"] / e["ms"] if e["ms"] > 0 else 0.0
        e["frac_of_bf16_burst"] = e["tflops"] / tf_burst
        e["frac_of_bf16_sustained"] = e["tflops"] / tf_sust
    shapes = shape_breakdown(per_launch, flops, tf_burst, tf_sust)
    for e in shapes.values():
        e["share"] = e["ms"] / step_ms_prof if step_ms_prof > 0 else None
    # dominant kernel: the tensor-core launch shape with the largest share of the forward
    dom_key = max((k for k, e in shapes.items() if e["class"] in TENSOR_CLASSES),
                  key=lambda k: shapes[k]["ms"])
    dom = shapes[dom_key]
    traffic = DRAM_BYTES_PER_LAUNCH.get(dom_key)
    attn_gemm_gflop = sum(fl for c, fl in flops if c in TENSOR_CLASSES) / 1e9
    roofline = {"bound": "tensor", "achieved": dom["tflops"], "peak": tf_burst,
                "unit": "TFLOP/s", "frac": dom["tflops"] / tf_burst, "traffic": traffic,
                "kernel": dom_key[0], "kernel_description": KIND_DESCRIPTION.get(dom_key[0]),
                "gflop_per_launch": dom_key[1], "launches_per_forward": dom["launches"],
                "ms_per_launch": dom["ms"] / dom["launches"],
                "share_of_forward": dom["share"],
                "peak_kind": f"bf16 dense burst ({peak_src}); the kernels run inside a "
                             "ms-scale forward, not a seconds-long loop",
                "peak_sustained": tf_sust, "frac_of_sustained": dom["tflops"] / tf_sust,
                "traffic_unit": "bytes per launch (dram__bytes_read.sum + "
                                "dram__bytes_write.sum, one ncu capture of this kernel)",
                "timing": "per-launch CUDA events in an instrumented graph of the same "
                          "forward run as one batch on one stream (the events bracket "
                          "consecutive launches), mean of 5 replays, L2 flushed before each"}
    shape_list = sorted(({"kernel": k[0], "gflop_per_launch": k[1], **{kk: vv for kk, vv in
                          e.items() if kk not in ("kind",)}} for k, e in shapes.items()),
                        key=lambda e: -e["ms"])

    rr_ms = [ms for n, ms in per_launch if n == "unroll_reroll"]
    rr_bytes = reroll_bytes(IMG, B)
    reroll_hbm = None
    if len(rr_ms) == len(rr_bytes) and sum(rr_ms) > 0:
        gbs = sum(rr_bytes) / (sum(rr_ms) * 1e-3) / 1e9
        big = max(range(len(rr_bytes)), key=lambda i: rr_bytes[i])
        gbs_big = rr_bytes[big] / (rr_ms[big] * 1e-3) / 1e9
        reroll_hbm = {"bytes_per_forward": sum(rr_bytes), "ms": sum(rr_ms), "gbs": gbs,
                      "frac_of_hbm": gbs / hbm_gbs, "largest_launch_bytes": rr_bytes[big],
                      "largest_launch_gbs": gbs_big, "largest_launch_frac": gbs_big / hbm_gbs,
                      "peak_gbs": hbm_gbs, "note": "event-timed inside the instrumented "
                      "graph (includes the per-launch event gap)"}

    # ---- Unroll / Reroll alone: a stage-0 tensor of 32 images (235 MB, both directions 470 MB,
    # far beyond the 126 MB L2), 10 launches back to back between two events
    G0 = IMG // 4
    xs = torch.randn(32, G0 * G0, 112, device=dev).to(torch.bfloat16)
    ys = torch.empty_like(xs)
    nbytes = 2 * xs.numel() * xs.element_size()
    res = {}
    with torch.cuda.stream(stream):
        for name, fn in (("unroll", hb.unroll), ("reroll", hb.reroll)):
            for _ in range(3):
                fn(xs, G0, 3, out=ys, stream=stream)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(10):
                fn(xs, G0, 3, out=ys, stream=stream)
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1) / 10
            res[name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                         "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm_gbs}
    rr_alone = {"bytes": nbytes, "shape": [32, G0 * G0, 112], "dtype": "bf16",
                "timing": "10 launches back to back, tensor > L2", **res}
    del xs, ys
    if reroll_hbm is not None:
        reroll_hbm["standalone"] = rr_alone

    # ---- end to end through the public API with host buffers: binding.BackbonePipeline
    # uploads each step's image from pinned host memory, calls hiera_backbone_forward and
    # downloads all four features into pinned host memory; the copies of a step overlap the
    # compute of its neighbours (three streams, two device buffer sets). The timed region
    # spans the first upload to the last download. No L2 flush: a step's working set
    # (weights ~140 MB, activations several hundred MB) exceeds the 126 MB L2.
    e2e = None
    if not args.no_e2e:
        n = args.e2e_steps
        pipe = hb.BackbonePipeline(desc, packed, device=dev)
        host_feats = pipe.host_feature_buffers()
        pipe.run([img_host] * 3, [host_feats] * 3)  # warm-up
        pipe.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        pipe.run([img_host] * n, [host_feats] * n, start_event=e0, end_event=e1)
        pipe.synchronize()
        e2e_ms = replicas.max_over_ranks(e0.elapsed_time(e1), dev)
        st = hb.device_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after e2e: {hb.status_string(st)}")
        e2e = {"value": replicas.job_throughput(B * n, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": img_host.numel() * img_host.element_size(),
               "d2h_bytes_per_step": sum(f.numel() * f.element_size() for f in host_feats),
               "steps": n, "images_per_step": B,
               "api": "binding.BackbonePipeline: pinned H2D image, hiera_backbone_forward, "
                      "pinned D2H of the four features per step, copies overlapping "
                      "neighbouring steps",
               "l2": "not flushed; per-step working set > L2"}
        del pipe

    del graph, pgraph, packed, ws, feats
    torch.cuda.synchronize()

    # ---- other workloads of the same forward (one GPU each, not part of the headline):
    # batch-1 latency at 512^2 and batch-1 throughput at 2048^2
    extra = {}
    if not args.no_extra:
        ms1, gf1 = extra_forward_timing(hb, syn, dev, stream, flush, IMG, 1, SEED, 30)
        extra["latency_512_b1"] = {"ms_per_forward": ms1, "images_per_s": 1e3 / ms1,
                                   "tflops": gf1 / ms1, "gflop_per_forward": gf1,
                                   "timing": "CUDA graph, L2 flushed before each forward, "
                                             "median of 30"}
        ms5, gf5 = extra_forward_timing(hb, syn, dev, stream, flush, 2048, 1, 4, 10)
        extra["throughput_2048_b1"] = {"ms_per_forward": ms5, "images_per_s": 1e3 / ms5,
                                       "tflops": gf5 / ms5, "gflop_per_forward": gf5,
                                       "frac_of_bf16_burst": gf5 / ms5 / tf_burst,
                                       "timing": "CUDA graph, L2 flushed before each "
                                                 "forward, median of 10"}

    if rank != 0:
        return
    clock_rec = clocks.record()
    if dom_key[0].startswith("attention"):
        # The attention kernels are bound by their exponentials rather than the tensor pipe:
        # one ex2.approx per score (B x heads x Tq x Tkv = GFLOP / (4 x 56) per launch) on the
        # SM's MUFU unit, taken as 16 results per clock per SM (the rate the CUDA programming
        # guide tables give for exp2 on recent compute capabilities), 148 SMs at the median
        # SM clock of the timed region.
        sms = torch.cuda.get_device_properties(local_rank).multi_processor_count
        mhz = (clock_rec or {}).get("sm_mhz") or 1965.0
        exps = dom_key[1] * 1e9 / (4 * 56)
        ach = exps / (roofline["ms_per_launch"] * 1e-3)
        peak = 16.0 * sms * mhz * 1e6
        roofline["mufu_context"] = {"exp_per_launch": exps, "achieved_exp_per_s": ach,
                                    "peak_exp_per_s": peak, "frac": ach / peak,
                                    "peak_basis": "16 ex2 per clock per SM x SMs x median SM "
                                                  "clock (assumed rate, not measured)"}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, n = oracle_images_per_s(20.0, 3, 0)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} image(s) of {IMG}x{IMG}x4 through the full backbone "
                         "(fp64 numpy oracle, unrolled formulation)"}
    gflop_per_image = sum(fl for _, fl in flops) / B / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"Hiera-B+ backbone forward, {IMG}x{IMG}x4 bf16 images, "
                               f"batch {B} per GPU (random-init weights, seed {SEED})",
                   "img": IMG, "batch_per_gpu": B, "global_batch": B * world,
                   "forwards_per_step": replays, "images_per_step_per_gpu": B * replays,
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "flushed before every step (256 MiB write); within a step each "
                         "forward's working set (138 MB of weights + activations) exceeds L2",
                   "timing": "CUDA-graph replay of the library launches, per-step CUDA events",
                   "mlp": args.mlp, "pdl": args.pdl, "attn": args.attn,
                   "split_batch": (f"two concurrent halves of {(B + 1) // 2} and {B // 2} "
                                   "images on two streams" if split else "off"),
                   "gemm224": ["8warp", "16warp", "pair"][hb.get_option(hb.OPT_GEMM224)]},
        "ms_per_forward": ms_per_forward,
        "timed_seconds": total_ms / 1e3,
        "tflops": gflop_per_image * images / (total_ms * 1e-3) * 1e-3,
        "attn_gemm_frac_of_bf16_peak": attn_gemm_gflop / (ms_per_forward * 1e-3) / 1e3 / tf_burst,
        "attn_gemm_frac_of_bf16_sustained": attn_gemm_gflop / (ms_per_forward * 1e-3) / 1e3
        / tf_sust,
        "gflop_per_image": gflop_per_image,
        "roofline": roofline,
        "kernels": classes,
        "by_kernel": by_kernel,
        "by_shape": shape_list,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "unroll_reroll_hbm": reroll_hbm,
        "extra_workloads": extra,
        "clocks": clock_rec,
        "gpu_launches": launches_per_forward * replays * args.steps,
        "launches_per_forward": launches_per_forward,
        "per_launch": [[n, round(fl / 1e9, 3), round(ms * 1e3, 2)]
                       for (n, ms), (_, fl) in zip(per_launch, flops)],
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--replays", type=int, default=0,
                    help="forwards per timed step (0: chosen so the timed region lasts "
                         "--timed-seconds)")
    ap.add_argument("--timed-seconds", type=float, default=1.2)
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the batch-1 latency and 2048^2 throughput measurements")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--batch", type=int, default=BATCH)
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mlp", choices=["fused", "unfused"], default="fused",
                    help="stage-0/1 MLPs as one fused kernel (default) or two GEMMs")
    ap.add_argument("--pdl", choices=["on", "off"], default="on",
                    help="programmatic dependent launch between the library's kernels")
    ap.add_argument("--attn", choices=["fused", "unfused"], default="fused",
                    help="stage-0 attention half (norm1, qkv, attention, proj) as one kernel "
                         "(default) or three")
    ap.add_argument("--split", choices=["on", "off"], default="on",
                    help="run each batch as two concurrent halves on two streams (library "
                         "default) or as one batch")
    ap.add_argument("--gemm224", choices=["default", "8warp", "16warp", "pair"],
                    default="default",
                    help="kernel of the 224-column-tile Linear layers (library default, the "
                         "eight- or sixteen-epilogue-warp CTA, or the CTA pair)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
