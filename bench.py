"""Benchmark of the ternary linear-stack decode path on B200.

Workload: the 28-layer stack of a 1.5B-class decoder's seven ternary linears
(q, k, v, o 1536x1536/256; gate, up 1536->8960; down 8960->1536), 1.31e9
ternary weights = 327,548,928 packed bytes, M = 1 token per step by default,
per-token int8 activation quantisation fused before every GEMV.  One step is
one bitnet_linear_stack launch over all 196 layers.  Weights (327.5 MB) are
larger than the 126 MB L2, so every step streams them from HBM; no L2 flush is
needed between steps.

Prints one JSON line (rank 0).  `value` is whole-job tokens/s with inputs
resident in HBM; `e2e` is the same metric through the C ABI with the step's
activations copied host->device and the outputs device->host every step.
Multi-GPU runs are independent replicas (the path has no exchange step).

``--impl reference`` times the CPU oracle (plain single-threaded C) on the
same workload instead: each step is one M=1 token through a bounded sample of
the stack's layers.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "M=1 ternary linear-stack tokens/s & packed-weight HBM GB/s; prefill int8 TOPS"
STACK_BYTES = 327_548_928
FALLBACK_HBM_GBS = 6650.0


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=1, help="tokens per step (1, 2, 4, 8)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the M = 2, 4, 8 lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the M=2048 prefill GEMM line")
    ap.add_argument("--i8-only", action="store_true",
                    help="run only the I8_S decode measurement and print its object")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the M=2048 prefill GEMMs (profiling aid) and print their object")
    ap.add_argument("--soak", type=float, default=0.5,
                    help="seconds of untimed launches before timing (clock sampling window)")
    ap.add_argument("--layers", type=int, default=28,
                    help="decoder layers in the stack (28 = the benchmark; fewer only for profiling captures)")
    return ap.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", d
    except Exception:
        return FALLBACK_HBM_GBS, "fallback", {}


def _kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemv.cu", "gemv.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "ternary_weight_i2_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic(m):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "gemv_stack_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("source_hash") == _kernel_source_hash() and str(m) in d.get("bytes_per_launch", {}):
            return float(d["bytes_per_launch"][str(m)])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons polled through NVML every
    ~2 ms from a background thread while the timed region runs."""

    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.stop_evt = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of numbers
            self.err = str(e)

    def _poll(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()

    def stop(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable: " + self.err]}
        self.stop_evt.set()
        self.t.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ GPU arm

def build_stack(m, dev, layers=28):
    """Pack the 28 layers on the GPU; return descriptors, the contiguous input
    and output buffers and their per-layer views."""
    import torch
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import synth

    packed, tws = [], []
    fl = torch.zeros(1, dtype=torch.int32, device=dev)
    for L in range(layers):
        for (name, n, k), (w, s) in zip(synth.LAYER_SHAPES, synth.layer_weights(L, 3)):
            wt = torch.from_numpy(w).to(dev)
            pk = torch.empty((n, tw2.packed_bytes(n, k) // n), dtype=torch.uint8, device=dev)
            tw2.pack_ternary(wt, pk, flags=fl)
            del wt
            packed.append(pk)
            tws.append(tw2.make_tw(pk, n, k, s))
    torch.cuda.synchronize()
    if int(fl.item()) != 0:
        raise RuntimeError("pack flagged a non-ternary weight")
    # all distinct inputs in one buffer, all outputs in another
    in_sizes = [m * k for _ in range(layers) for k in synth.LAYER_INPUT_K]
    out_sizes = [m * n for _ in range(layers) for (_, n, _) in synth.LAYER_SHAPES]
    x_host = np.empty(sum(in_sizes), np.float32)
    off = 0
    for L in range(layers):
        for a in synth.layer_inputs(L, m, 3):
            x_host[off:off + a.size] = a.ravel()
            off += a.size
    x_dev = torch.from_numpy(x_host).to(dev)
    y_dev = torch.empty(sum(out_sizes), dtype=torch.float32, device=dev)
    xs, ys, off, yoff = [], [], 0, 0
    for L in range(layers):
        views = []
        for k in synth.LAYER_INPUT_K:
            views.append(x_dev[off:off + m * k].view(m, k))
            off += m * k
        for (_, n, _), j in zip(synth.LAYER_SHAPES, synth.LAYER_INPUT_OF):
            xs.append(views[j])
            ys.append(y_dev[yoff:yoff + m * n].view(m, n))
            yoff += m * n
    return packed, tws, xs, ys, x_host, x_dev, y_dev


def time_device(call, steps, warmup, stream, profile_range=False):
    """Per-launch CUDA-event durations on `stream` and the whole-loop time.
    With profile_range the timed loop is bracketed by cudaProfilerStart/Stop,
    so that a profiler started with --profile-from-start off sees only it."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    _barrier()
    torch.cuda.synchronize()
    if profile_range:
        torch.cuda.cudart().cudaProfilerStart()
    for i in range(steps):
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if profile_range:
        torch.cuda.cudart().cudaProfilerStop()
    _barrier()
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total = starts[0].elapsed_time(ends[-1])
    return total, per


def _barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def _max_over_ranks(v):
    """The slowest rank's value (every rank gets it).  One process per GPU
    over NCCL in a bench run; the tensor lives where the backend wants it."""
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return v


def whole_job_rate(world, units_per_rank, max_ms):
    """Units per second of the whole job: every rank processes
    `units_per_rank` units per step (replicas, weak scaling), and the job's
    step time is the slowest rank's."""
    return world * units_per_rank / (max_ms * 1e-3)


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import build as tbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    tbuild.build()
    tw2.load()

    m = args.m
    packed, tws, xs, ys, x_host, x_dev, y_dev = build_stack(m, dev, args.layers)
    stack_bytes = sum(int(p.numel()) for p in packed)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    call = tw2.StackCall(xs, tws, ys)
    stream = torch.cuda.current_stream()

    # device-resident timing through a captured graph of the stack launch
    call(flags=flags)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(flags=flags)
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local)
    for _ in range(int(args.soak / 1e-4)):   # untimed soak of the same launch before timing
        graph.replay()
    clocks.start()
    total_ms, per = time_device(graph.replay, args.steps, args.warmup, stream, profile_range=True)
    clk = clocks.stop()
    if int(flags.item()) != 0:
        raise RuntimeError(f"device flags {int(flags.item())} during the timed run")
    total_ms = _max_over_ranks(total_ms)
    kern_ms = _max_over_ranks(statistics.mean(per))
    ms_step = total_ms / args.steps
    tok_s = whole_job_rate(world, m, ms_step)

    # end to end through the C ABI: H2D inputs, stack call, D2H outputs per step
    e2e = None
    if not args.no_e2e:
        x_pin = torch.from_numpy(x_host).pin_memory()
        y_pin = torch.empty(y_dev.numel(), dtype=torch.float32).pin_memory()

        def e2e_step():
            x_dev.copy_(x_pin, non_blocking=True)
            call(flags=flags)
            y_pin.copy_(y_dev, non_blocking=True)

        e_total, _ = time_device(e2e_step, max(args.steps // 2, 10), args.warmup, stream)
        e_total = _max_over_ranks(e_total)
        e_steps = max(args.steps // 2, 10)
        e2e = {"value": whole_job_rate(world, m, e_total / e_steps), "unit": "tokens/s",
               "h2d_bytes_per_step": int(x_host.nbytes), "d2h_bytes_per_step": int(y_dev.numel() * 4)}

    peak, peak_kind, peaks = _peaks()
    achieved = stack_bytes / (kern_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": _ncu_traffic(m),
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "kernel": "gemv_stack_kernel", "kernel_ms": round(kern_ms, 5),
                "algorithmic_bytes": stack_bytes}

    sweep = {}
    if not args.no_sweep and m == 1:
        for ms in (2, 4, 8):
            _, twsm, xsm, ysm, _, _, _ = build_stack_views(ms, dev, tws, args.layers)
            c2 = tw2.StackCall(xsm, twsm, ysm)
            c2(flags=flags)
            torch.cuda.synchronize()
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                c2(flags=flags)
            t2, per2 = time_device(g2.replay, 50, 5, stream)
            t2 = _max_over_ranks(t2)
            k2 = _max_over_ranks(statistics.mean(per2))
            sweep[str(ms)] = {"tokens_per_s": round(whole_job_rate(world, ms, t2 / 50), 1),
                              "weight_gbs": round(stack_bytes / (k2 * 1e-3) / 1e9, 1)}

    # the same M=1 stack with the fused epilogue on every linear: bias, layer
    # scale and residual add (ReLU on gate and up), residuals in one buffer
    epi_line = None
    if m == 1:
        r_dev = torch.randn(y_dev.numel(), dtype=torch.float32, device=dev)
        b_dev = torch.randn(y_dev.numel() // m, dtype=torch.float32, device=dev)
        g_dev = torch.rand(y_dev.numel() // m, dtype=torch.float32, device=dev) + 0.5
        epis, off = [], 0
        for i, (y, tw) in enumerate(zip(ys, tws)):
            n = y.shape[1]
            name = synth_layer_name(i)
            epis.append(tw2.make_epilogue(bias=b_dev[off:off + n], gamma=g_dev[off:off + n],
                                          residual=r_dev[off * m:(off + n) * m].view(m, n),
                                          relu=name in ("gate", "up")))
            off += n
        ce = tw2.StackCall(xs, tws, ys, epis=epis)
        ce(flags=flags)
        torch.cuda.synchronize()
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge):
            ce(flags=flags)
        te, _ = time_device(ge.replay, 50, 5, stream)
        te = _max_over_ranks(te) / 50
        epi_line = {"workload": "the M=1 stack with bias + layer scale + residual add on all %d linears "
                                "(ReLU on gate/up)" % len(tws),
                    "tokens_per_s": round(whole_job_rate(world, m, te), 1), "ms_per_step": round(te, 5),
                    "vs_plain_stack": round(ms_step / te, 4),
                    "extra_bytes_per_step": int(3 * 4 * y_dev.numel())}
        if int(flags.item()) != 0:
            raise RuntimeError(f"device flags {int(flags.item())} in the epilogue stack run")

    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(dev, stream, flags, world)
    qpack = run_quantize_pack(dev, stream, flags, world)
    i8_line = run_i8_decode(dev, stream, flags, world)
    try:
        pack_line = run_pack(dev, stream, flags, world)
    except Exception as e:   # a load-time side measurement must not cost the main line
        pack_line = {"error": str(e)[:300]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(budget_s=12.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(tok_s, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
            "data": "synthetic (seeded ternary weights and fp32 activations of the 1.5B-class decoder-layer shapes)",
            "config": {"workload": "%d-layer ternary linear stack, %d layers, M=%d decode"
                                   % (args.layers, 7 * args.layers, m),
                       "tokens_per_step_per_gpu": m, "layers": 7 * args.layers,
                       "packed_weight_bytes": stack_bytes,
                       "l2": "weights 327.5 MB > 126 MB L2 (no flush needed)",
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "timing": "CUDA graph replay of one bitnet_linear_stack launch per step"},
            "weight_gbs": round(stack_bytes * world / (ms_step * 1e-3) / 1e9, 1),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clk,
            "m_sweep": sweep,
            "prefill": prefill,
            "quantize_pack": qpack,
            "fused_epilogue_stack": epi_line,
            "i8s_decode": i8_line,
            "pack": pack_line,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def synth_layer_name(i):
    from ternary_weight_i2_b200 import synth
    return synth.LAYER_SHAPES[i % len(synth.LAYER_SHAPES)][0]


PREFILL_M = 2048
PREFILL_OPS = 2 * PREFILL_M * sum(n * k for _, n, k in
                                  [("q", 1536, 1536), ("k", 256, 1536), ("v", 256, 1536), ("o", 1536, 1536),
                                   ("gate", 8960, 1536), ("up", 8960, 1536), ("down", 1536, 8960)])


def run_prefill(dev, stream, flags, world):
    """M=2048 prefill over the seven decoder-layer shapes: int8 activations
    pre-quantised by bitnet_quant_act (timed separately), then one
    bitnet_linear_q_grouped launch (the tcgen05 GEMM over all seven layers'
    tiles) per step, graph-replayed.  Per-shape lines time each layer alone."""
    import torch
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import synth

    xs = synth.prefill_inputs(PREFILL_M)
    xq, xs_scale, x_dev = {}, {}, {}
    for k, x in xs.items():
        x_dev[k] = torch.from_numpy(x).to(dev)
        xq[k] = torch.empty((PREFILL_M, tw2.kpad(k)), dtype=torch.int8, device=dev)
        xs_scale[k] = torch.empty(PREFILL_M, dtype=torch.float32, device=dev)
    tws, ys, keep = [], [], []
    for i, (name, n, k) in enumerate(synth.LAYER_SHAPES):
        rng = np.random.default_rng(synth.seed_for(4, i))
        w = synth.ternary(rng, n, k)
        s = synth.weight_scale(rng)
        pk = torch.empty((n, tw2.packed_bytes(n, k) // n), dtype=torch.uint8, device=dev)
        tw2.pack_ternary(torch.from_numpy(w).to(dev), pk, flags=flags)
        keep.append(pk)
        tws.append((name, n, k, tw2.make_tw(pk, n, k, s)))
        ys.append(torch.empty((PREFILL_M, n), dtype=torch.float32, device=dev))

    def quant():
        for k in xs:
            tw2.quant_act(x_dev[k], xq[k], xs_scale[k], flags=flags)

    grouped = tw2.GroupedCall([xq[k] for (_, _, k, _) in tws], [xs_scale[k] for (_, _, k, _) in tws],
                              [tw for (_, _, _, tw) in tws], ys)

    def gemms():
        grouped(flags=flags)

    quant()
    gemms()
    torch.cuda.synchronize()
    gq, gg = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gq):
        quant()
    with torch.cuda.graph(gg):
        gemms()
    tq, _ = time_device(gq.replay, 20, 3, stream)
    tg, per = time_device(gg.replay, 20, 3, stream)
    tq, tg = _max_over_ranks(tq) / 20, _max_over_ranks(tg) / 20
    # the quantiser's algorithmic bytes: fp32 in, int8 rows (with pads) and
    # one fp32 scale per token out, per distinct input
    quant_bytes = sum(PREFILL_M * (4 * k + tw2.kpad(k) + 4) for k in xs)
    # the same launch with the fused epilogue on every layer (bias, layer
    # scale, residual add; ReLU on gate and up)
    epi_keep, epis = [], []
    for name, n, k, tw in tws:
        b = torch.randn(n, device=dev)
        g = torch.rand(n, device=dev) + 0.5
        r = torch.randn((PREFILL_M, n), device=dev)
        epi_keep.append((b, g, r))
        epis.append(tw2.make_epilogue(bias=b, gamma=g, residual=r, relu=name in ("gate", "up")))
    grouped_epi = tw2.GroupedCall([xq[k] for (_, _, k, _) in tws], [xs_scale[k] for (_, _, k, _) in tws],
                                  [tw for (_, _, _, tw) in tws], ys, epis=epis)
    grouped_epi(flags=flags)
    torch.cuda.synchronize()
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge):
        grouped_epi(flags=flags)
    te, _ = time_device(ge.replay, 20, 3, stream)
    te = _max_over_ranks(te) / 20
    per_shape = {}
    for (name, n, k, tw), y in zip(tws, ys):
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1):
            tw2.linear_q(xq[k], xs_scale[k], tw, y, flags=flags)
        t, _ = time_device(g1.replay, 10, 2, stream)
        per_shape[name] = {"ms": round(t / 10, 5), "tops": round(2 * PREFILL_M * n * k / (t / 10 * 1e-3) / 1e12, 1)}
    if int(flags.item()) != 0:
        raise RuntimeError(f"device flags {int(flags.item())} in the prefill run")
    _, _, peaks = _peaks()
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    peak = 2.0 * bf16          # int8 dense = 2 x bf16 dense (nominal 4.5 vs 2.25 PFLOP/s)
    tops = whole_job_rate(world, PREFILL_OPS, tg) / 1e12
    return {"workload": "M=2048 tokens x the seven decoder-layer shapes, int8 activations x ternary weights",
            "ops_per_step": PREFILL_OPS, "ms_per_step": round(tg, 5), "tops": round(tops, 1),
            "roofline": {"bound": "tensor", "achieved": round(tops / world, 1), "peak": round(peak, 1),
                         "unit": "TOPS", "frac": round(tops / world / peak, 4),
                         "peak_kind": "measured bf16 cuBLAS burst (MEASURED_PEAKS.json) x 2 (int8:bf16 dense ratio)"},
            "quant_ms_per_step": round(tq, 5),
            "quant_roofline": {"bound": "hbm", "achieved": round(quant_bytes / (tq * 1e-3) / 1e9, 1),
                               "peak": round(_peaks()[0], 1), "unit": "GB/s",
                               "frac": round(quant_bytes / (tq * 1e-3) / 1e9 / _peaks()[0], 4),
                               "bytes": quant_bytes, "kernel": "quant_kernel (a2 standalone)"},
            "per_shape": per_shape,
            "with_fused_epilogue": {"ms_per_step": round(te, 5),
                                    "tops": round(whole_job_rate(world, PREFILL_OPS, te) / 1e12, 1),
                                    "epilogue": "bias + layer scale + residual add on all seven (ReLU on gate/up)"},
            "kernel": "gemm_i2_kernel (tcgen05.mma kind::i8, weights expanded into TMEM as A, activations as B from shared memory, 128 features x 192 tokens x 128 tiles, one grouped launch)"}


def run_quantize_pack(dev, stream, flags, world):
    """Load-time absmean quantise + pack of one decoder layer's seven fp32
    weight tensors (187 MB of fp32, larger than L2), graph-replayed: two
    launches per tensor.  Algorithmic bytes: 4 B read + 1/4 B written per
    weight; the kernels read each tensor twice, the second time mostly from
    L2 (a tensor is at most 55 MB)."""
    import torch
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import synth

    ws = torch.empty(tw2.quantize_pack_workspace_bytes(), dtype=torch.uint8, device=dev)
    scales = torch.empty(len(synth.LAYER_SHAPES), dtype=torch.float32, device=dev)
    work, weights = [], 0
    for i, (name, n, k) in enumerate(synth.LAYER_SHAPES):
        g = torch.Generator(device=dev)
        g.manual_seed(synth.seed_for(5, i))
        W = torch.randn((n, k), generator=g, device=dev, dtype=torch.float32) * 0.02
        pk = torch.empty((n, tw2.packed_bytes(n, k) // n), dtype=torch.uint8, device=dev)
        work.append((W, pk, scales[i:i + 1]))
        weights += n * k

    def step():
        for W, pk, sc in work:
            tw2.quantize_pack(W, pk, sc, ws, flags=flags)

    step()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        step()
    steps = 20
    t, _ = time_device(gr.replay, steps, 3, stream)
    t = _max_over_ranks(t) / steps
    if int(flags.item()) != 0:
        raise RuntimeError(f"device flags {int(flags.item())} in the quantize_pack run")
    hbm, _, _ = _peaks()
    alg = 4.25 * weights
    gbs = alg / (t * 1e-3) / 1e9
    return {"workload": "absmean quantise + pack of one decoder layer's seven fp32 weight tensors "
                        "(%d weights, %.1f MB fp32 > L2)" % (weights, 4 * weights / 1e6),
            "ms_per_step": round(t, 5), "launches_per_step": 2 * len(work),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes_per_weight": 4.25},
            "kernels": "absmean_partial_kernel, absmean_pack_kernel"}


I8_LAYERS = 4
PACK_LAYERS = 4


def run_pack(dev, stream, flags, world):
    """Load-time pack (int8 ternary -> 2-bit codes) of four decoder layers'
    28 tensors per step (187 MB of int8, larger than L2), graph-replayed.
    Algorithmic bytes: 1 B read + 1/4 B written per weight."""
    import torch
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import synth

    g = torch.Generator(device=dev)
    g.manual_seed(synth.seed_for(7, 0))
    work, weights = [], 0
    for L in range(PACK_LAYERS):
        for name, n, k in synth.LAYER_SHAPES:
            w = torch.randint(-1, 2, (n, k), generator=g, device=dev, dtype=torch.int8)
            pk = torch.empty((n, tw2.packed_bytes(n, k) // n), dtype=torch.uint8, device=dev)
            work.append((w, pk))
            weights += n * k

    def step():
        for w, pk in work:
            tw2.pack_ternary(w, pk, flags=flags)

    step()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        step()
    steps = 10
    t, _ = time_device(gr.replay, steps, 3, stream)
    t = _max_over_ranks(t) / steps
    if int(flags.item()) != 0:
        raise RuntimeError(f"device flags {int(flags.item())} in the pack run")
    hbm, _, _ = _peaks()
    gbs = 1.25 * weights / (t * 1e-3) / 1e9
    return {"workload": "pack of %d decoder layers' %d ternary int8 tensors (%.1f MB > L2)"
                        % (PACK_LAYERS, len(work), weights / 1e6),
            "ms_per_step": round(t, 5), "launches_per_step": len(work),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes_per_weight": 1.25},
            "kernels": "pack_kernel"}


def run_i8_decode(dev, stream, flags, world):
    """I8_S decode: M=1 token through four decoder layers' seven linears with
    int8 weights, all 28 in one bitnet_linear_i8_grouped call per step
    (graph-replayed; 187 MB of weights, larger than L2).  Algorithmic bytes:
    1 B per weight."""
    import torch
    import ternary_weight_i2_b200 as tw2
    from ternary_weight_i2_b200 import synth

    g = torch.Generator(device=dev)
    g.manual_seed(synth.seed_for(6, 0))
    keep, xs_l, w8s, ys, weight_bytes = [], [], [], [], 0
    xs = {k: torch.randn((1, k), generator=g, device=dev) for k in synth.LAYER_INPUT_K}
    for L in range(I8_LAYERS):
        for name, n, k in synth.LAYER_SHAPES:
            rows = torch.randint(-127, 128, (n, tw2.i8_row_bytes(k)), generator=g, device=dev, dtype=torch.int8)
            keep.append(rows)
            w8s.append(tw2.make_i8w(rows, n, k, 0.01))
            xs_l.append(xs[k])
            ys.append(torch.empty((1, n), device=dev))
            weight_bytes += n * k
    call = tw2.I8GroupCall(xs_l, w8s, ys)
    ws = torch.empty(call.workspace_bytes, dtype=torch.uint8, device=dev)

    def step():
        call(ws, flags=flags)

    step()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        step()
    steps = 20
    t, _ = time_device(gr.replay, steps, 3, stream)
    t = _max_over_ranks(t) / steps
    if int(flags.item()) != 0:
        raise RuntimeError(f"device flags {int(flags.item())} in the I8_S run")
    hbm, _, _ = _peaks()
    gbs = weight_bytes / (t * 1e-3) / 1e9
    return {"workload": "I8_S decode, M=1, %d decoder layers x seven linears with int8 weights (%.1f MB > L2), "
                        "one grouped call" % (I8_LAYERS, weight_bytes / 1e6),
            "tokens_per_s": round(whole_job_rate(world, 1, t), 1), "ms_per_step": round(t, 5),
            "launches_per_step": len(xs) + 1,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes_per_weight": 1.0},
            "kernels": "quant_kernel per distinct input + one i8_gemv_kernel<1> over all rows"}


def build_stack_views(m, dev, tws, layers=28):
    """Inputs/outputs for another token count, reusing the packed weights."""
    import torch
    from ternary_weight_i2_b200 import synth
    xs, ys = [], []
    for L in range(layers):
        views = [torch.from_numpy(a).to(dev) for a in synth.layer_inputs(L, m, 3)]
        for (_, n, _), j in zip(synth.LAYER_SHAPES, synth.LAYER_INPUT_OF):
            xs.append(views[j])
            ys.append(torch.empty((m, n), dtype=torch.float32, device=dev))
    return None, tws, xs, ys, None, None, None


# ------------------------------------------------------------ CPU oracle arm

class OracleSample:
    """A bounded sample of the workload for the CPU oracle: decoder layer 0's
    seven linears (11.7 MB packed, 1/28 of the stack) at M = 1, packed once by
    the oracle.  One pass = one token through those seven layers."""

    def __init__(self):
        import oracle
        from ternary_weight_i2_b200 import synth
        self.oracle = oracle
        xl = synth.layer_inputs(0, 1, 3)
        self.layers = []
        self.bytes = 0
        for (name, n, k), (w, s), j in zip(synth.LAYER_SHAPES, synth.layer_weights(0, 3),
                                           synth.LAYER_INPUT_OF):
            pk, _ = oracle.pack(w)
            self.layers.append((xl[j], pk, n, k, s))
            self.bytes += pk.nbytes

    def run(self):
        t0 = time.perf_counter()
        for x, pk, n, k, s in self.layers:
            self.oracle.linear(x, pk, n, k, s)
        return time.perf_counter() - t0

    def tokens_per_s(self, secs, passes):
        # fraction of the stack per pass = self.bytes / STACK_BYTES
        return passes * (self.bytes / STACK_BYTES) / secs


def cpu_baseline(budget_s=12.0):
    smp = OracleSample()
    secs, passes = 0.0, 0
    while secs < budget_s:
        secs += smp.run()
        passes += 1
    return {"value": round(smp.tokens_per_s(secs, passes), 4), "unit": "tokens/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{passes} passes of one M=1 token through decoder layer 0's seven linears "
                      f"({smp.bytes} of {STACK_BYTES} packed bytes per pass, {secs:.1f} s single-threaded), "
                      f"scaled by packed bytes to the 196-layer stack"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.run()
    t_total = 0.0
    for _ in range(args.steps):
        t_total += smp.run()
    tok_s = smp.tokens_per_s(t_total, args.steps)
    ms_step = t_total / args.steps * 1e3 * STACK_BYTES / smp.bytes
    line = {
        "impl": "reference", "metric": METRIC, "value": round(tok_s, 4), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": {"workload": "28-layer ternary linear stack, 196 layers, M=1 decode",
                   "tokens_per_step_per_gpu": 1},
        "cpu_baseline": {"value": round(tok_s, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: one M=1 token through decoder layer 0's seven linears "
                                   f"({smp.bytes} packed bytes, 1/28 of the stack) on the plain C oracle, "
                                   f"single-threaded; tokens/s scaled by packed bytes to the full stack"},
        "e2e": {"value": round(tok_s, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    elif args.prefill_only or args.i8_only:
        import torch
        import ternary_weight_i2_b200 as tw2
        from ternary_weight_i2_b200 import build as tbuild
        tbuild.build()
        tw2.load()
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        flags = torch.zeros(1, dtype=torch.int32, device=dev)
        run = run_prefill if args.prefill_only else run_i8_decode
        print(json.dumps(run(dev, torch.cuda.current_stream(), flags, 1)))
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
