#!/usr/bin/env python
"""Benchmark of the NF4 scoring pass (the AQLoRA setup pass) on B200.

One step = one pass of the whole path over a model's weights, resident in HBM:
fused NF4 quantize + nibble pack + double quantization + per-layer reconstruction error
for every layer (aqnf4_layer_error), then the top-K selection under the byte budget
(aqnf4_select_topk).  With N ranks the layers are split by LPT and the scores are
all-gathered before the selection.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead, on a
bounded sample of the same workload, on this machine's host cores.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NF4 quantize+score GB/s (fp16 weights read) and % of HBM roofline; dequant GB/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SRCS = [os.path.join(ROOT, "quantized_lora_setup_b200", "csrc", f)
               for f in ("quant_score.cu", "device.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_quant_score_7b.md")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="7b", choices=["tiny", "1.4b", "7b", "14b"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dequant", action="store_true")
    ap.add_argument("--no-dequant-sweep", action="store_true",
                    help="skip the dequantize sweep (packed 1 MB .. 4 GB and the named shapes)")
    ap.add_argument("--no-nf4-linear", action="store_true",
                    help="skip the fused NF4-dequant GEMM measurement")
    ap.add_argument("--only-nf4-linear", action="store_true",
                    help="time only the fused NF4-dequant GEMM (shape: --gemm-shape)")
    ap.add_argument("--gemm-shape", default="4096,11008,4096",
                    help="M,N,K of --only-nf4-linear")
    ap.add_argument("--gemm-reps", type=int, default=20)
    ap.add_argument("--no-dq-score", action="store_true",
                    help="skip the step scored against the double-quantized constants")
    ap.add_argument("--extra-workloads", default="14b,1.4b",
                    help="comma-separated workloads also timed (1 GPU only; '' to skip)")
    ap.add_argument("--max-layers", type=int, default=0,
                    help="use only the first N layers (small cases for profiling)")
    ap.add_argument("--protocol", action="store_true",
                    help="also run the source pages' timing protocol: two identical arms of "
                         ">= 2 s each (noise floor); the CPU baseline is also timed on one "
                         "thread")
    ap.add_argument("--sessions", type=int, default=1,
                    help="run this many whole sessions (separate processes, each with "
                         "--protocol) and report their median and spread (1 GPU only)")
    return ap.parse_args()


L2_BYTES = 126 << 20


def host_threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 64))


def workload_desc(wl) -> str:
    shapes = sorted({(s.rows, s.cols) for s in wl.layers})
    sh = ", ".join(f"{r}x{c}" for r, c in shapes)
    dts = sorted({str(s.dtype).replace("torch.", "") for s in wl.layers})
    return (f"{wl.name}-shaped: {len(wl.layers)} linear layers ({sh}), {'/'.join(dts)}, "
            f"{wl.numel / 1e9:.3f}e9 weights, synthetic seeded")


def algorithmic_bytes(n: int) -> int:
    """Bytes the fused pass must move for an n-element layer: read the 16-bit weights,
    write packed nibbles, 8-bit DQ codes and fp32 DQ scales."""
    nb = (n + 63) // 64
    return 2 * n + (n + 1) // 2 + nb + 4 * ((nb + 255) // 256)


# ------------------------------------------------------------------ CPU oracle leg


def oracle_pass(sample):
    """The oracle's version of one step on a list of (bits, dtype) layer samples."""
    import oracle

    def one(item):
        b, dt = item
        _, absmax, _ = oracle.quantize(b, dt)
        oracle.double_quant(absmax)
        oracle.layer_error(b, dt)
        return b.size

    with ThreadPoolExecutor(max_workers=len(sample)) as ex:
        return sum(ex.map(one, sample))


def build_oracle_sample(wl, threads, per_thread_elems, layer_tensors=None):
    """One equal-size slice per thread: the first elements of the workload's first
    `threads` layers (equal sizes keep the threads busy for the same time)."""
    from quantized_lora_setup_b200 import synth
    import oracle
    sample = []
    nl = min(threads, len(wl.layers))
    per_thread_elems = min([per_thread_elems] + [wl.layers[i].numel for i in range(nl)])
    for i in range(nl):
        spec = wl.layers[i]
        if layer_tensors is not None:
            w = layer_tensors[i].reshape(-1)[: min(spec.numel, per_thread_elems)].cpu()
        else:
            w = synth.layer_host(spec, wl.seed, i).reshape(-1)[: min(spec.numel, per_thread_elems)]
        dt = oracle.BF16 if str(w.dtype) == "torch.bfloat16" else oracle.F16
        n = (w.numel() // 16384) * 16384 or w.numel()
        sample.append((synth.bits_u16(w[:n]), dt))
    return sample


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from quantized_lora_setup_b200 import synth
    wl = synth.workload(args.workload)
    threads = host_threads()
    # ~75 ns per element per thread for quantize + DQ + error in the oracle: size each step so
    # the whole run (warm-up + steps) stays near two minutes.
    per_step_s = max(0.2, 120.0 / max(1, args.steps + args.warmup))
    per_thread = max(16384, int(per_step_s / 75e-9) // 16384 * 16384)
    sample = build_oracle_sample(wl, threads, per_thread)
    elems = sum(b.size for b, _ in sample)
    for _ in range(args.warmup):
        oracle_pass(sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(sample)
    dt = time.perf_counter() - t0
    value = 2 * elems * args.steps / dt / 1e9
    desc = (f"{len(sample)} slices of {sample[0][0].size} elements (the first elements of the "
            f"first {len(sample)} layers), {elems} weights per step, one thread per slice")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload_desc(wl), "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": len(sample), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Polls NVML every 10 ms (SM clock, max SM clock, clock-event reasons) in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:  # CUDA and NVML may number the GPUs differently: match by UUID
                uuid = str(torch.cuda.get_device_properties(index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than fail the bench
            self.nv, self.err = None, str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            self._stop.wait(0.01)

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ native arm


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic():
    """Per-launch DRAM bytes of k_quant_score from the committed ncu summary, if it was
    taken on the current kernel sources (their sha256 is recorded beside the number)."""
    try:
        text = open(TRAFFIC_FILE).read()
        h = hashlib.sha256()
        for f in KERNEL_SRCS:
            with open(f, "rb") as fh:
                h.update(fh.read())
        src = h.hexdigest()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        line = line.strip().lstrip("-").strip()
        if ":" in line and line.startswith(("traffic_bytes_per_launch", "source_sha256")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("` ")
    if vals.get("source_sha256") != src:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def run_native(args):
    import torch
    import torch.distributed as dist

    from quantized_lora_setup_b200 import aqnf4, synth
    from quantized_lora_setup_b200.shard import ScoreGather, lpt_partition

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    aqnf4.library()

    wl = synth.workload(args.workload)
    if args.max_layers > 0:
        wl = synth.Workload(wl.name + f"[:{args.max_layers}]", wl.layers[: args.max_layers],
                            wl.budgets, wl.k_cap, wl.seed)
    L = len(wl.layers)
    parts = lpt_partition([s.numel for s in wl.layers], world)
    mine = parts[rank]
    weights = [synth.layer_device(wl.layers[i], wl.seed, i, dev) for i in mine]
    stor = [aqnf4.NF4Storage(w.numel(), dev) for w in weights]
    descs = aqnf4.make_layers([{"w": w, "packed": s.packed, "codes8": s.codes8,
                                "scales": s.scales} for w, s in zip(weights, stor)])
    ws = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=dev)
    se = torch.empty(max(1, len(mine)), dtype=torch.float64, device=dev)
    sw = torch.empty_like(se)
    rel = torch.empty(max(1, len(mine)), dtype=torch.float32, device=dev)
    cost = torch.tensor([aqnf4.aqnf4_cost_bytes(s.numel) for s in wl.layers], dtype=torch.int64,
                        device=dev)
    sel = torch.empty(L, dtype=torch.int32, device=dev)
    kout = torch.empty(1, dtype=torch.int32, device=dev)
    budget = wl.budgets[0]
    gather = ScoreGather(parts, rank, L, dev) if world > 1 else None
    stream = torch.cuda.current_stream(dev)

    def step(ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        if mine:
            aqnf4.aqnf4_layer_error(descs, ws, se, sw, rel, None, stream)
        if ev_b is not None:
            ev_b.record(stream)
        scores = gather(rel) if gather is not None else rel
        aqnf4.aqnf4_select_topk(scores, cost, budget, wl.k_cap, sel, kout, stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    launches0 = aqnf4.aqnf4_launch_count()
    clocks.start()
    t_start.record(stream)
    for i in range(K):
        step(*ev[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    launches = aqnf4.aqnf4_launch_count() - launches0
    barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    agg = torch.tensor([elapsed_ms, float(launches)], dtype=torch.float64, device=dev)
    if world > 1:
        mx = agg[:1].clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        tot = agg[1:].clone()
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
        elapsed_ms, launches = float(mx.item()), int(tot.item())
    total_weight_bytes = wl.weight_bytes
    value = total_weight_bytes * K / (elapsed_ms / 1e3) / 1e9

    # roofline of the dominant kernel (this rank's fused pass; the small finalize kernel
    # that follows it is inside the same event pair, so this slightly understates it)
    my_alg = sum(algorithmic_bytes(w.numel()) for w in weights)
    kern_avg_ms = statistics.mean(kern_ms)
    achieved = my_alg / (kern_avg_ms / 1e3) / 1e9
    peak, peak_src = measured_hbm_peak()
    traffic = recorded_traffic()

    k_sel = int(kout.item())
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "layers_per_s": L * K / (elapsed_ms / 1e3),
        "config": {
            "workload": workload_desc(wl), "layers": L, "weight_bytes": total_weight_bytes,
            "budget_bytes": budget, "k_cap": wl.k_cap,
            "l2": "inputs larger than L2 (weights read once per step, no flush needed)"
            if total_weight_bytes >= 2 * L2_BYTES else
            "L2-resident: the working set is below twice the 126 MB L2 (reported as such)",
            "parallelism": f"layers split over {world} rank(s) by LPT; scores all-gathered"
            if world > 1 else "single GPU",
            "outputs": "packed NF4 + 8-bit DQ codes + fp32 DQ scales + per-layer scores",
        },
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": ("profiles/k_quant_score_7b.md: ncu dram__bytes_read.sum + "
                                        "dram__bytes_write.sum of one full-size launch, taken on "
                                        "kernel sources with the recorded sha256")
                     if traffic is not None else
                     "none: no ncu capture recorded for the current kernel sources",
                     "kernel": "k_quant_score",
                     "peak_source": f"{peak_src} hbm_gbs", "alg_bytes_per_launch": my_alg,
                     "launch_ms": kern_avg_ms},
        "clocks": clocks.summary(),
        "gpu_launches": launches,
        "selected": {"k": k_sel, "of": L},
    }

    if args.protocol:
        result["protocol"] = bench_protocol(step, dev, stream, world, total_weight_bytes,
                                            elapsed_ms / K)

    if not args.no_dequant:
        result["dequant"] = bench_dequant(dev, stream, peak)
    if not args.no_dequant and not args.no_dequant_sweep:
        result["dequant_sweep"] = bench_dequant_sweep(dev, stream, peak)

    if world == 1:
        result["select_blocks"] = bench_select_blocks(wl, se, sw, cost, budget, dev, stream)

    if world == 1:
        result["split_model"] = bench_split_model(weights, budget, wl.k_cap, dev)

    if world == 1 and not args.no_nf4_linear:
        result["nf4_linear"] = bench_nf4_linear(dev, stream)

    if world == 1 and not args.no_dq_score:
        result["dqc_score"] = bench_dq_score(weights, stor, wl, cost, budget, sel, k_sel, dev,
                                             stream, peak, steps=min(K, 100), mode="centered")
        result["dq_score"] = bench_dq_score(weights, stor, wl, cost, budget, sel, k_sel, dev,
                                            stream, peak, steps=min(K, 100))

    if not args.no_e2e:
        result["e2e"] = bench_e2e(args, weights, step, sel, kout, dev, stream, world,
                                  total_weight_bytes, L)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_threads()
        per_thread = max(16384, int(20.0 / threads / 75e-9) // 16384 * 16384)
        sample = build_oracle_sample(wl, threads, per_thread, layer_tensors=weights)
        t0 = time.perf_counter()
        elems = oracle_pass(sample)
        dt = time.perf_counter() - t0
        result["cpu_baseline"] = {
            "value": 2 * elems / dt / 1e9, "unit": UNIT, "cores": len(sample), "kind": "oracle",
            "sample": f"{len(sample)} slices of {sample[0][0].size} elements from the first "
                      f"{len(sample)} layers ({elems} weights), quantize + DQ + error, one "
                      f"thread per slice"}
        if args.protocol:  # the pages' second oracle timing: one slice on one thread
            t0 = time.perf_counter()
            one = oracle_pass(sample[:1])
            result["cpu_baseline"]["single_thread"] = 2 * one / (time.perf_counter() - t0) / 1e9

    extras = [w for w in args.extra_workloads.split(",") if w and w != args.workload]
    if world == 1 and extras:
        del weights, stor, descs, ws
        torch.cuda.empty_cache()
        result["workloads"] = {name: bench_workload(name, dev, stream, peak, steps=50)
                               for name in extras}

    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        result["summary"] = compact_summary(result)  # last: a tail of the line keeps it
        print(json.dumps(result), flush=True)
    return 0


def compact_summary(r):
    """The line's figures in a few hundred bytes: the main kernel's roofline fraction and
    layers/s, the other model shapes, the dequantize kernel (named shape and sweep points
    with the same-traffic copy floor), the fused GEMM against dequantize + cuBLAS, and the
    DQ-absmax score."""
    def rnd(x, d=4):
        return None if x is None else round(float(x), d)
    s = {"frac": rnd(r["roofline"]["frac"]), "gbs": rnd(r["value"], 1),
         "layers_per_s": rnd(r.get("layers_per_s"), 1)}
    for name, w in (r.get("workloads") or {}).items():
        s[name] = {"frac": rnd(w["roofline"]["frac"]), "gbs": rnd(w["value"], 1),
                   "layers_per_s": rnd(w.get("layers_per_s"), 1)}
    if "dequant" in r:
        d = r["dequant"]
        s["dequant"] = {"shape": d["shape"], "gbs": rnd(d["value"], 1),
                        "frac": rnd(d["roofline"]["frac"])}
    pts = {p["case"]: p for p in (r.get("dequant_sweep") or {}).get("points", [])}
    for case in ("packed_8MB", "packed_16MB", "packed_1024MB"):
        if case in pts:
            s.setdefault("dequant", {})[case] = [rnd(pts[case]["frac"], 3),
                                                 rnd(pts[case].get("copy_frac"), 3)]
    if "nf4_linear" in r:
        for k, v in r["nf4_linear"].items():
            if k.startswith("tokens_"):
                s[f"gemm_{k}"] = [rnd(v["value"], 1), rnd(v.get("dequant_then_cublas"), 1)]
    if "dq_score" in r:
        s["dq_score_frac"] = rnd(r["dq_score"]["roofline"]["frac"])
    if "dqc_score" in r:
        s["dqc_score_frac"] = rnd(r["dqc_score"]["roofline"]["frac"])
    return s


def measured_tensor_peak():
    """(dense bf16 TFLOP/s for a kernel timed in a short burst, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def run_only_nf4_linear(args):
    """One JSON line with the fused GEMM alone (for profiling a single shape)."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M, N, K = (int(v) for v in args.gemm_shape.split(","))
    out = bench_nf4_linear(dev, torch.cuda.current_stream(dev), reps=args.gemm_reps,
                           shapes=((M, N, K),), baseline=False)
    print(json.dumps({"nf4_linear": out}), flush=True)
    return 0


def bench_nf4_linear(dev, stream, reps=20,
                     shapes=((4096, 11008, 4096), (512, 11008, 4096), (128, 11008, 4096)),
                     baseline=True):
    """The forward product of an NF4 + DQ layer, y = x w_hat^T, with the dequantization fused
    into the tcgen05 GEMM (aqnf4_nf4_linear): the 7B-shaped MLP up-projection (11008 x 4096)
    at 4096, 512 and 128 tokens, bf16.  TFLOP/s against the measured bf16 peak, beside the unfused
    path (aqnf4_dequantize, then cuBLAS on the bf16 weights) for context."""
    import torch

    from quantized_lora_setup_b200 import aqnf4, synth
    peak, src = measured_tensor_peak()
    out = {"unit": "TFLOP/s", "peak": peak, "peak_source": f"{src} bf16_tflops"}
    layers = {}
    for M, N, K in shapes:
        if (N, K) not in layers:
            w = synth.normal_matrix_device(N, K, seed=7, device=dev)
            st = aqnf4.NF4Storage(N * K, dev)
            aqnf4.score_layers([w.reshape(-1)], [st], stream=stream)
            del w
            layers[(N, K)] = st
        st = layers[(N, K)]
        out["layer"] = [N, K]
        wd = torch.empty(N * K, dtype=torch.bfloat16, device=dev) if baseline else None
        g = torch.Generator(device=dev)
        g.manual_seed(M)
        x = torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

        def fused():
            aqnf4.aqnf4_nf4_linear(x, st.packed, st.codes8, st.scales, N, y, None, stream)

        def unfused():
            aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, N * K, wd, stream)
            torch.matmul(x, wd.view(N, K).t(), out=y)

        res = {}
        arms = (("fused", fused), ("dequant_then_cublas", unfused)) if baseline else (("fused", fused),)
        for name, fn in arms:
            for _ in range(3):
                fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ms = a.elapsed_time(b) / reps
            res[name] = 2.0 * M * N * K / (ms / 1e3) / 1e12
        out[f"tokens_{M}"] = {
            "value": res["fused"], "ms": 2.0 * M * N * K / res["fused"] / 1e9,
            "split_k": aqnf4.aqnf4_nf4_linear_splits(M, N, K),
            "roofline": {"bound": "tensor", "achieved": res["fused"], "peak": peak,
                         "unit": "TFLOP/s", "frac": res["fused"] / peak,
                         "kernel": "k_nf4_gemm"},
            "dequant_then_cublas": res.get("dequant_then_cublas")}
    return out


def bench_split_model(weights, budget, k_cap, dev):
    """Materialize the split model (fused pass + selection + keeping one copy per layer)
    twice: the first wall time includes the first allocation of every layer's NF4 storage,
    the second runs with torch's caching allocator warm.  Also the memory report."""
    import torch

    from quantized_lora_setup_b200 import split_model
    walls = []
    for _ in range(2):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        model = split_model.materialize(weights, budget, k_cap)
        torch.cuda.synchronize(dev)
        walls.append((time.perf_counter() - t0) * 1e3)
        rep = model.memory_report()
        del model
    return {"first_wall_ms": walls[0], "wall_ms": walls[1], "memory": rep}


def bench_select_blocks(wl, se, sw, cost, budget, dev, stream, reps=200):
    """Block-level selection (speed setting) on the step's scores, both orders: the blocks
    kept under the budget, the lowest kept block, and the kernel's time per launch."""
    import torch

    from quantized_lora_setup_b200 import aqnf4, synth
    block_of = torch.tensor(synth.block_index(wl), dtype=torch.int32, device=dev)
    B = int(block_of.max().item()) + 1
    out = {"blocks": B}
    for name, order in (("by_depth", aqnf4.AQNF4_BLOCKS_BY_DEPTH),
                        ("by_error", aqnf4.AQNF4_BLOCKS_BY_ERROR)):
        rank = torch.empty(B, dtype=torch.int32, device=dev)
        k = torch.empty(1, dtype=torch.int32, device=dev)

        def run():
            aqnf4.aqnf4_select_blocks(se, sw, block_of, cost, B, budget, order, rank, None, k,
                                      stream)
        for _ in range(3):
            run()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            run()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        kept = rank[: int(k.item())].tolist()
        out[name] = {"kept": kept, "lowest_kept_block": min(kept) if kept else None,
                     "us_per_launch": t0.elapsed_time(t1) * 1e3 / reps}
    return out


def bench_dq_score(weights, stor, wl, cost, budget, sel_plain, k_plain, dev, stream, peak, steps,
                   mode="absmax"):
    """The same scoring step with every layer scored against its double-quantized constants
    (mode "absmax": AQNF4_SCORE_DQ_ABSMAX; "centered": AQNF4_SCORE_DQ_CENTERED, the
    mean-centred format): GB/s of weights read, the fused kernel's roofline fraction, and
    whether the kept set under the budget differs from the plain score's."""
    import torch

    from quantized_lora_setup_b200 import aqnf4
    flag = {"absmax": aqnf4.AQNF4_SCORE_DQ_ABSMAX, "centered": aqnf4.AQNF4_SCORE_DQ_CENTERED}[mode]
    descs = aqnf4.make_layers([{"w": w, "packed": s.packed, "codes8": s.codes8,
                                "scales": s.scales, "flags": flag}
                               for w, s in zip(weights, stor)])
    L = len(weights)
    ws = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=dev)
    se = torch.empty(L, dtype=torch.float64, device=dev)
    sw = torch.empty_like(se)
    rel = torch.empty(L, dtype=torch.float32, device=dev)
    sel = torch.empty(L, dtype=torch.int32, device=dev)
    kout = torch.empty(1, dtype=torch.int32, device=dev)

    def step(ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        aqnf4.aqnf4_layer_error(descs, ws, se, sw, rel, None, stream)
        if ev_b is not None:
            ev_b.record(stream)
        aqnf4.aqnf4_select_topk(rel, cost, budget, wl.k_cap, sel, kout, stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(*ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / steps
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    alg = sum(algorithmic_bytes(w.numel()) for w in weights)
    k = int(kout.item())
    kept = sorted(sel[:k].tolist())
    kept_plain = sorted(sel_plain[:k_plain].tolist())
    return {"value": wl.weight_bytes / (ms / 1e3) / 1e9, "unit": UNIT, "ms_per_step": ms,
            "layers_per_s": len(weights) / (ms / 1e3),
            "steps": steps,
            "roofline": {"bound": "hbm", "achieved": alg / (kern_ms / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": alg / (kern_ms / 1e3) / 1e9 / peak,
                         "kernel": "k_quant_score (%s)" % ("AQNF4_SCORE_DQ_ABSMAX"
                                                           if mode == "absmax" else
                                                           "AQNF4_SCORE_DQ_CENTERED")},
            "selected": {"k": k, "of": L, "same_set_as_plain_score": kept == kept_plain}}


def bench_workload(name, dev, stream, peak, steps):
    """The same scoring step on another model shape (1 GPU): GB/s of weights read, the fused
    kernel's roofline fraction, and the selection at every budget of that workload."""
    import torch

    from quantized_lora_setup_b200 import aqnf4, synth
    wl = synth.workload(name)
    weights = [synth.layer_device(s, wl.seed, i, dev) for i, s in enumerate(wl.layers)]
    stor = [aqnf4.NF4Storage(w.numel(), dev) for w in weights]
    descs = aqnf4.make_layers([{"w": w, "packed": s.packed, "codes8": s.codes8,
                                "scales": s.scales} for w, s in zip(weights, stor)])
    ws = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=dev)
    L = len(weights)
    se = torch.empty(L, dtype=torch.float64, device=dev)
    sw = torch.empty_like(se)
    rel = torch.empty(L, dtype=torch.float32, device=dev)
    cost = torch.tensor([aqnf4.aqnf4_cost_bytes(s.numel) for s in wl.layers], dtype=torch.int64,
                        device=dev)
    sel = torch.empty(L, dtype=torch.int32, device=dev)
    kout = torch.empty(1, dtype=torch.int32, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        aqnf4.aqnf4_layer_error(descs, ws, se, sw, rel, None, stream)
        if e is not None:
            e[1].record(stream)
        aqnf4.aqnf4_select_topk(rel, cost, wl.budgets[0], wl.k_cap, sel, kout, stream)

    for _ in range(3):
        step()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for e in evs:
        step(e)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    kern_ms = statistics.mean(x.elapsed_time(y) for x, y in evs)
    alg = sum(algorithmic_bytes(w.numel()) for w in weights)
    kept = {}
    for budget in wl.budgets:
        aqnf4.aqnf4_select_topk(rel, cost, budget, wl.k_cap, sel, kout, stream)
        kept[str(budget)] = int(kout.item())
    achieved = alg / (kern_ms / 1e3) / 1e9
    dts = sorted({str(s.dtype).replace("torch.", "") for s in wl.layers})
    return {"workload": workload_desc(wl), "dtype_in": "/".join(dts), "steps": steps,
            "ms_per_step": ms, "value": wl.weight_bytes / (ms / 1e3) / 1e9, "unit": UNIT,
            "layers_per_s": L / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "kernel": "k_quant_score",
                         "launch_ms": kern_ms, "alg_bytes_per_launch": alg},
            "kept_per_budget": kept}


def bench_dequant(dev, stream, peak):
    """Standalone NF4+DQ -> bf16 dequantization of a 28672x8192 matrix; four distinct
    inputs rotate so the 117 MB packed input cannot stay in the 126 MB L2."""
    import torch

    from quantized_lora_setup_b200 import aqnf4, synth
    rows, cols = synth.DEQUANT_SHAPES[-1]
    n = rows * cols
    inputs = []
    for s in range(4):
        w = synth.normal_matrix_device(rows, cols, seed=1000 + s, device=dev)
        st = aqnf4.NF4Storage(n, dev)
        aqnf4.score_layers([w], [st])
        del w
        inputs.append(st)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    for st in inputs:
        aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, n, out, stream)
    reps = 40
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for i in range(reps):
        st = inputs[i % 4]
        aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, n, out, stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / reps
    alg = dequant_alg_bytes(n)
    gbs = alg / (ms / 1e3) / 1e9
    return {"shape": f"{rows}x{cols}", "ms_per_launch": ms, "value": gbs, "unit": "GB/s",
            "out_gbs": 2 * n / (ms / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": None, "kernel": "k_dequant",
                         "alg_bytes_per_launch": alg}}


def dequant_alg_bytes(n):
    """Bytes one dequantize of n elements must move: packed codes, 8-bit constants and DQ
    scales in, 16-bit values out."""
    nb = (n + 63) // 64
    return n // 2 + nb + 4 * ((nb + 255) // 256) + 2 * n


def bench_dequant_sweep(dev, stream, peak, reps=9):
    """NF4 + DQ -> bf16 over packed sizes 1 MB .. 4 GB (x2) and the named matrix shapes,
    each stored from an N(0, 0.02) bf16 matrix by the scoring pass.  Before every launch L2
    is flushed: a 256 MB write, then a read of another 256 MB so that the written lines
    are back in DRAM before the timed launch starts.  Each launch is timed alone with
    events on the launching stream and the median is reported, so every size is measured
    from DRAM with a clean L2."""
    import torch

    from quantized_lora_setup_b200 import aqnf4, synth
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    cases = [("packed_%dMB" % (1 << e), 4096, (2 << 20 << e) // 4096) for e in range(13)]
    cases += [("%dx%d" % rc, rc[1], rc[0]) for rc in (synth.DEQUANT_SHAPES[0],
                                                      synth.DEQUANT_SHAPES[-1])]
    points = []
    for name, cols, rows in cases:
        n = rows * cols
        w = synth.normal_matrix_device(rows, cols, seed=77, device=dev)
        st = aqnf4.NF4Storage(n, dev)
        aqnf4.score_layers([w.reshape(-1)], [st], stream=stream)
        del w
        out = torch.empty(n, dtype=torch.bfloat16, device=dev)
        aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, n, out, stream)
        times = []
        for _ in range(reps):
            with torch.cuda.stream(stream):
                flush.fill_(1)
                clean.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            aqnf4.aqnf4_dequantize(st.packed, st.codes8, st.scales, None, n, out, stream)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        ms = sorted(times)[reps // 2]
        alg = dequant_alg_bytes(n)
        gbs = alg / (ms / 1e3) / 1e9
        # the memory floor at this size: a device copy moving the same bytes (alg / 2 read,
        # alg / 2 written), timed the same way from a flushed L2
        src = torch.empty(alg // 2, dtype=torch.uint8, device=dev)
        dst = torch.empty_like(src)
        ctimes = []
        for _ in range(reps):
            with torch.cuda.stream(stream):
                flush.fill_(1)
                clean.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            with torch.cuda.stream(stream):
                dst.copy_(src)
            b.record(stream)
            b.synchronize()
            ctimes.append(a.elapsed_time(b))
        cms = sorted(ctimes)[reps // 2]
        points.append({"case": name, "packed_bytes": n // 2, "elements": n,
                       "us": ms * 1e3, "value": gbs, "frac": gbs / peak,
                       "copy_us": cms * 1e3, "copy_frac": alg / (cms / 1e3) / 1e9 / peak})
        del st, out, src, dst
    torch.cuda.empty_cache()
    return {"unit": "GB/s", "peak": peak, "kernel": "k_dequant", "dtype_out": "bfloat16",
            "l2": "flushed before every launch (256 MB write, then 256 MB read); median of %d"
                  % reps,
            "copy_reference": "copy_frac: a device copy of the same byte count (half read, "
                              "half written), same flush and timing: the floor at that size",
            "points": points}


def bench_e2e(args, weights, step, sel, kout, dev, stream, world, total_weight_bytes, L):
    """The same step through the public API with the weights starting in pinned host
    memory: every step copies them in, runs the pass and reads the selection back."""
    import torch
    import torch.distributed as dist

    host = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in weights]
    for h, w in zip(host, weights):
        h.copy_(w)
    steps = max(1, min(args.steps, 5))
    res_k = torch.empty(1, dtype=torch.int32, pin_memory=True)
    res_sel = torch.empty(L, dtype=torch.int32, pin_memory=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a.record(stream)
    for _ in range(steps):
        for h, w in zip(host, weights):
            w.copy_(h, non_blocking=True)
        step()
        res_k.copy_(kout, non_blocking=True)
        res_sel.copy_(sel, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    h2d = sum(w.numel() * w.element_size() for w in weights)
    return {"value": total_weight_bytes * steps / (ms / 1e3) / 1e9, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4 + 4 * L, "steps": steps}


def fixed_duration_chunks(run_chunk, max_over_ranks, min_ms):
    """Run chunks until their summed time reaches min_ms.  Each chunk's time is the maximum
    over ranks (max_over_ranks is a collective), so every rank sees the same sum and stops
    after the same number of chunks.  Returns (chunks, summed ms)."""
    chunks, total = 0, 0.0
    while total < min_ms:
        total += max_over_ranks(run_chunk())
        chunks += 1
    return chunks, total


def bench_protocol(step, dev, stream, world, total_weight_bytes, ms_per_step,
                   min_seconds=2.0):
    """The source pages' timing rules for the scoring step: the same step is run as two
    arms, "a" and "b", each back to back for at least `min_seconds` of device time (a fixed
    duration, not a fixed count), timed with CUDA events in chunks of about 0.25 s.  With
    several ranks each chunk's time is the maximum over ranks, so every rank takes the same
    number of chunks.  The relative gap between the arms is the noise floor."""
    import torch
    import torch.distributed as dist

    chunk = max(1, int(250.0 / max(ms_per_step, 1e-3)))

    def run_chunk():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(chunk):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b)

    def max_over_ranks(ms):
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    arms = {}
    for arm in ("a", "b"):
        chunks, total_ms = fixed_duration_chunks(run_chunk, max_over_ranks, min_seconds * 1e3)
        steps = chunks * chunk
        arms[arm] = {"steps": steps, "seconds": total_ms / 1e3,
                     "value": total_weight_bytes * steps / (total_ms / 1e3) / 1e9}
    va, vb = arms["a"]["value"], arms["b"]["value"]
    return {"min_seconds_per_arm": min_seconds, "unit": UNIT, "arms": arms,
            "noise_floor": abs(va - vb) / ((va + vb) / 2)}


def session_child_argv(argv):
    """The command line of one session: this one without --sessions, with --protocol."""
    child, i = [], 0
    while i < len(argv):
        if argv[i] == "--sessions":
            i += 2
            continue
        if not argv[i].startswith("--sessions="):
            child.append(argv[i])
        i += 1
    if "--protocol" not in child:
        child.append("--protocol")
    return child


def run_sessions(args):
    """Whole sessions as separate processes (each with --protocol); prints the median
    session's line with the per-session values, their median and their spread."""
    import subprocess

    child = session_child_argv(sys.argv[1:])
    lines = []
    for _ in range(args.sessions):
        out = subprocess.run([sys.executable, os.path.abspath(__file__)] + child,
                             capture_output=True, text=True)
        if out.returncode != 0:
            sys.stderr.write(out.stdout[-2000:] + out.stderr[-4000:])
            return out.returncode
        lines.append(json.loads(out.stdout.strip().splitlines()[-1]))
    vals = [d["value"] for d in lines]
    med = statistics.median(vals)
    pick = min(range(len(lines)), key=lambda j: abs(vals[j] - med))
    arm_vals = [d["protocol"]["arms"][a]["value"] for d in lines for a in ("a", "b")]
    res = dict(lines[pick])
    res["sessions"] = {
        "n": len(lines), "values": vals, "median": med,
        "spread": (max(vals) - min(vals)) / med,
        "protocol_arm_values": arm_vals,
        "protocol_arm_median": statistics.median(arm_vals),
        "protocol_arm_spread": (max(arm_vals) - min(arm_vals)) / statistics.median(arm_vals),
        "noise_floors": [d["protocol"]["noise_floor"] for d in lines]}
    print(json.dumps(res), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.sessions > 1:
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            raise SystemExit("--sessions runs separate single-GPU processes; not under torchrun")
        return run_sessions(args)
    if args.only_nf4_linear:
        return run_only_nf4_linear(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
