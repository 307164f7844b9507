#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 linear layer (NVFP4, rank 32, GELU) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload fc1_nvfp4]

A step is one pass of the whole layer over one batch: the activation kernel
(smooth + quantise + pack + down projection) and the 4-bit GEMM kernel (with
the low-rank up projection, GELU and bf16 store), for the headline layer
M=4608 tokens, K=3072, N=12288, r=32 (``--workload`` picks another; the
2048-px DiT block runs its four linears back to back, fc2 fed with fc1's
output).  Inputs are seeded synthetic data already resident in HBM; L2 is
flushed (a 256 MB write and a 256 MB read, outside the timed events) before
every step.  Under torchrun each rank runs its own replica of
the layer (the layer is token-parallel; no collective is on the data path),
and the slowest rank's device time is reported.

--impl reference times the CPU oracle (plain numpy) on the host cores on a
bounded row sample per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+rank-32 linear effective TFLOPS at M4608 K3072 N12288; % of FP4 TC roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fc1_nvfp4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-scheme-error", action="store_true",
                    help="skip the (untimed) quantisation-error report")
    ap.add_argument("--overhead-repeats", type=int, default=0,
                    help="also time the same single-layer workload at r = 0, alternating with it this "
                         "many times (each of --steps steps), and report the low-rank branch's "
                         "overhead t(r) / t(0) - 1 as median and range")
    ap.add_argument("--chain", action="store_true",
                    help="multi-layer workloads: run each fc1 -> fc2 pair with fc2's activation side fused "
                         "into fc1's GEMM epilogue (svdq_w4a4_gemm_lowrank_up_chain)")
    ap.add_argument("--int4-f16", action="store_true",
                    help="INT4 workloads: kernel 2 as one fp16 GEMM of the dequantised operands "
                         "(SVDQ_INT4_F16) instead of int8 MMAs")
    ap.add_argument("--qkv-epilogue", action="store_true",
                    help="NVFP4 qkv layers: kernel 2 with the fused Q/K RMS norm + rotary epilogue "
                         "(svdq_w4a4_gemm_lowrank_up_qkv; a seeded 2-D position table)")
    ap.add_argument("--l2-warm", action="store_true",
                    help="layer workloads: no L2 flush between steps (steps back to back; the "
                         "layers' inputs and outputs together exceed the 126 MB L2)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "bit_diffusion_transformer_w4a4_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(f"{kernel}/{workload}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        loaded = [float(r[1]) for r in rows if float(r[3]) > 300.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows)}


def layer_bytes(layer) -> int:
    """Algorithmic HBM bytes of one layer pass: X read; activation codes and
    scales written and read back; the packed weight codes and scales, L1, L2
    read; T written and read; Y written."""
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    M, K, N, r, G = layer.M, layer.K, layer.N, layer.r, layer.G
    sb = 2 if layer.variant == W.INT4 else 1          # bf16 or E4M3 scale bytes
    return (M * K * 2 + 2 * (M * K // 2) + 2 * (M * K // G) * sb + N * K // 2 + (N * K // G) * sb
            + K * r * 2 + r * N * 2 + 2 * M * r * 4 + M * N * 2)


def layer_desc(layer, f16: bool = False, qkv: bool = False) -> str:
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    return (f"{layer.name} M{layer.M} K{layer.K} N{layer.N} r{layer.r}{' GELU' if layer.gelu else ''} "
            f"{W.VARIANT_NAME[layer.variant]}{' fp16-operand GEMM' if f16 else ''}"
            f"{' + QK-norm + RoPE epilogue' if qkv else ''}")


def cpu_baseline(layer, pw, x_bits, nrows: int, one_core: bool = True):
    """The oracle, as it stands, on a row sample of the same workload: on all
    host threads its BLAS uses, and (``one_core``) again limited to one."""
    import numpy as np
    from oracle import forward as O
    rows = np.arange(nrows)
    flops = 2.0 * nrows * layer.K * layer.N + 2.0 * nrows * layer.r * (layer.K + layer.N)
    t = time.perf_counter()
    O.linear_forward(x_bits, pw, rows=rows)
    dt = time.perf_counter() - t
    out = {"value": flops / dt / 1e12, "unit": "TFLOPS", "kind": "oracle",
           "sample": f"{nrows} of {layer.M} token rows of {layer.name} (numpy fp64), {dt:.2f} s"}
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        out["cores"] = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        if one_core:
            n1 = max(8, nrows // 8)
            with threadpool_limits(limits=1):
                t = time.perf_counter()
                O.linear_forward(x_bits, pw, rows=np.arange(n1))
                d1 = time.perf_counter() - t
            f1 = flops * n1 / nrows
            out["value_1core"] = f1 / d1 / 1e12
            out["sample_1core"] = f"{n1} rows on 1 thread, {d1:.2f} s"
    except Exception:
        out["cores"] = os.cpu_count()
    return out


def run_reference(args, layers):
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    layer = layers[0]
    pw = W.synthetic_packed(layer)
    x = W.activations(layer)
    nrows = 64
    for _ in range(min(args.warmup, 3)):
        cpu_baseline(layer, pw, x, nrows, one_core=False)
    times, t_start = [], time.perf_counter()
    for _ in range(args.steps):
        r = cpu_baseline(layer, pw, x, nrows, one_core=False)
        times.append(r)
        if time.perf_counter() - t_start > 120.0:
            break
    flops = 2.0 * nrows * layer.K * layer.N + 2.0 * nrows * layer.r * (layer.K + layer.N)
    tflops = statistics.median(t["value"] for t in times)
    ms = flops / (tflops * 1e12) * 1e3
    line = {"metric": metric_name(args.workload, layers), "value": tflops, "unit": "TFLOPS",
            "n_gpus": args.gpus, "steps": len(times), "warmup": min(args.warmup, 3), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": layer_desc(layer), "step_sample_rows": nrows},
            "cpu_baseline": {k: times[-1][k] for k in ("unit", "cores", "kind", "sample")}
            | {"value": tflops},
            "e2e": {"value": tflops, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def scheme_error(layer, f16: bool = False) -> dict:
    """The method's own quantisation error on this layer, reported (not a
    gate): weights prepared by the library's GPU preparation from the
    layer's seeded full-precision W (calibration on its X, randomized SVD of
    rank r, residual quantisation), the layer run through the library, and
    the result compared with the dense fp32 product X W (relative Frobenius
    norm).  For NVFP4 also with the per-tensor weight scale, and the
    fraction of weight groups whose E4M3 scale is subnormal or zero without
    it."""
    import numpy as np
    import torch
    from bit_diffusion_transformer_w4a4_b200 import svdq
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    M, K, N, r, G = layer.M, layer.K, layer.N, layer.r, layer.G
    x_bits = W.activations(layer)
    w = W.weight(layer)
    xd = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    wd = torch.from_numpy(W.to_bf16_bits(w).view(np.int16)).cuda().view(torch.bfloat16)
    lam = torch.empty(K, dtype=torch.float32, device="cuda")
    svdq.prep_calibrate(xd, M, wd, K, N, lam)
    L1 = torch.zeros((K, max(r, 1)), dtype=torch.int16, device="cuda")
    L2 = torch.zeros((max(r, 1), N), dtype=torch.int16, device="cuda")
    if r > 0:
        omega = torch.from_numpy(np.random.default_rng([layer.config_id, 77]).standard_normal(
            (N, r + 16)).astype(np.float32)).cuda()
        svdq.prep_lowrank(wd, lam, K, N, r, omega, r + 16, 2, L1, L2)
    torch.backends.cuda.matmul.allow_tf32 = False
    ref = xd.float() @ wd.float()
    out = {"reference": "dense fp32 X W (tf32 off)", "weights": "seeded full-precision W, prepared on the GPU"}
    sb = 2 if layer.variant == W.INT4 else 1
    for ts in ([False, True] if layer.variant == W.NVFP4 else [False]):
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty(N * (K // G) * sb, dtype=torch.uint8, device="cuda")
        e = svdq.prep_residual_quantize(layer.variant, wd, lam, L1 if r else None, L2 if r else None, K, N,
                                        r, codes, scales, tensor_scale=ts)
        torch.cuda.synchronize()
        sc = scales.cpu().numpy()
        pw = W.PackedWeights(layer.variant, K, N, r, lam.cpu().numpy(),
                             L1.cpu().numpy().view(np.uint16)[:, :r], L2.cpu().numpy().view(np.uint16)[:r],
                             codes.cpu().numpy(),
                             sc.view(np.uint16).reshape(N, -1) if sb == 2 else sc.reshape(N, -1),
                             gelu=False, w_scale_exp=e)
        h = svdq.SVDQWeights(pw, M, int4_f16=f16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        h.linear_forward(xd, y, M)
        torch.cuda.synchronize()
        h.close()
        rel = float(torch.linalg.norm(y.float() - ref) / torch.linalg.norm(ref))
        out["rel_fro_tensor_scale" if ts else "rel_fro"] = rel
        if layer.variant == W.NVFP4 and not ts:
            exp0 = (sc & 0x78) == 0
            out["w_scale_subnormal_frac"] = float(np.mean(exp0 & (sc != 0)))
            out["w_scale_zero_frac"] = float(np.mean(sc == 0))
        if ts:
            out["w_scale_exp"] = e
    return out


def lowrank_overhead(d, steps: int, repeats: int, flush) -> dict:
    """t(r) / t(r = 0) - 1 for one layer: the same shapes, format and inputs
    with the low-rank branch removed, both timed `repeats` times alternately
    (each a mean over `steps` flushed steps, CUDA events at step boundaries)."""
    import dataclasses
    import statistics
    import torch
    from bit_diffusion_transformer_w4a4_b200 import svdq
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    layer = d["layer"]
    l0 = dataclasses.replace(layer, r=0)
    pw0 = W.synthetic_packed(l0)
    h0 = svdq.SVDQWeights(pw0, l0.M, int4_f16=d["f16"])
    c0, s0, t0 = h0.alloc_act(l0.M)
    y0 = torch.empty_like(d["y"])
    stream = torch.cuda.current_stream()

    def timed(h, codes, scales, t, y):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            flush()
            ev[i][0].record(stream)
            h.quantize_act_lowrank_down(d["x"], layer.M, codes, scales, t)
            h.w4a4_gemm_lowrank_up(codes, scales, t, layer.M, y)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.mean(e[0].elapsed_time(e[1]) for e in ev)

    timed(h0, c0, s0, t0, y0)
    tr, t0s = [], []
    for _ in range(repeats):
        tr.append(timed(d["h"], d["codes"], d["scales"], d["t"], d["y"]))
        t0s.append(timed(h0, c0, s0, t0, y0))
    h0.close()
    ov = [a / b - 1.0 for a, b in zip(tr, t0s)]
    return {"r": layer.r, "median": statistics.median(ov), "min": min(ov), "max": max(ov),
            "repeats": repeats, "steps_each": steps, "ms_r": tr, "ms_r0": t0s}


def metric_name(workload: str, layers) -> str:
    if workload == "fc1_nvfp4":
        return METRIC
    flops = sum(l.flops() for l in layers)
    return f"W4A4+low-rank linear effective TFLOPS, {workload} ({len(layers)} layer(s), {flops / 1e9:.0f} GFLOP per step)"


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank values across the process group (the
    slowest rank defines a multi-GPU step); identity on one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, flops_per_rank: float, ms_step: float) -> float:
    """Whole-job TFLOPS: every rank processes its own batch (weak scaling),
    timed by the slowest rank."""
    return world * flops_per_rank / (ms_step * 1e-3) / 1e12


def run_ours(args, layers):
    import numpy as np
    import torch
    import torch.distributed as dist
    from bit_diffusion_transformer_w4a4_b200 import svdq
    from bit_diffusion_transformer_w4a4_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    # one handle and one set of buffers per layer; in the DiT block fc2 reads
    # fc1's output (the MLP pair chained), the other layers their own inputs
    names = [l.name for l in layers]
    L = []
    for i, layer in enumerate(layers):
        f16 = bool(args.int4_f16) and layer.variant == W.INT4
        pw = W.synthetic_packed(layer, seed=rank)
        x_bits = W.activations(layer, seed=rank)
        qkv = bool(args.qkv_epilogue) and layer.name.endswith("qkv") and layer.variant == W.NVFP4
        rope = None
        if qkv:
            gq, gk, rope_h = W.qkv_epilogue_inputs(layer.M, rank)
            h = svdq.SVDQWeights(pw, layer.M, qkv_norm=(gq, gk, 1e-6))
            rope = torch.from_numpy(rope_h).cuda()
        else:
            h = svdq.SVDQWeights(pw, layer.M, int4_f16=f16)
        chained = layer.name.endswith("fc2") and any(n.endswith("fc1") for n in names[:i])
        if chained:
            x = L[names.index(names[i - 1])]["y"]
        else:
            x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.empty((layer.M, layer.N), dtype=torch.bfloat16, device="cuda")
        codes, scales, t = h.alloc_act(layer.M)
        L.append(dict(layer=layer, pw=pw, x_bits=x_bits, h=h, x=x, y=y, codes=codes, scales=scales,
                      t=t, f16=f16, chained=chained, rope=rope))
    # L2 flush before every step, outside the timed events: a 256 MB write,
    # then a 256 MB read of another buffer, so that L2 holds neither the inputs
    # nor dirty lines whose write-back would land inside the next step
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush():
        if args.l2_warm:
            return
        flush_w.zero_()
        flush_r.sum()

    # the step as a list of kernel launches (name, call); with --chain an
    # fc1 -> fc2 pair is fc1's activation kernel, the fused GEMM and fc2's GEMM
    fused = set()
    if args.chain:
        for i, d in enumerate(L):
            if d["chained"] and L[i - 1]["layer"].variant == W.NVFP4 and d["layer"].variant == W.NVFP4:
                fused.add(i - 1)
    launches = []
    for i, d in enumerate(L):
        pre = d["layer"].name + "." if len(L) > 1 else ""
        if i - 1 in fused:      # fc2 of a fused pair: its activation side came from fc1's GEMM
            launches.append((pre + "w4a4_gemm_lowrank_up", lambda d=d: d["h"].w4a4_gemm_lowrank_up(
                d["codes"], d["scales"], d["t"], d["layer"].M, d["y"])))
            continue
        launches.append((pre + "quantize_act_lowrank_down", lambda d=d: d["h"].quantize_act_lowrank_down(
            d["x"], d["layer"].M, d["codes"], d["scales"], d["t"])))
        if i in fused:
            d2 = L[i + 1]
            launches.append((pre + "w4a4_gemm_lowrank_up_chain", lambda d=d, d2=d2: svdq.gemm_lowrank_up_chain(
                d["h"], d["codes"], d["scales"], d["t"], d["layer"].M, None, d2["h"], d2["codes"], d2["scales"],
                d2["t"])))
        elif d["rope"] is not None:
            launches.append((pre + "w4a4_gemm_lowrank_up_qkv", lambda d=d: d["h"].w4a4_gemm_lowrank_up_qkv(
                d["codes"], d["scales"], d["t"], d["layer"].M, d["rope"], d["y"])))
        else:
            launches.append((pre + "w4a4_gemm_lowrank_up", lambda d=d: d["h"].w4a4_gemm_lowrank_up(
                d["codes"], d["scales"], d["t"], d["layer"].M, d["y"])))

    def run_layers(evs=None):
        for i, (_, call) in enumerate(launches):
            call()
            if evs is not None:
                evs[i + 1].record(stream)

    for _ in range(args.warmup):
        flush()
        run_layers()
    torch.cuda.synchronize()
    for d in L:
        st = d["h"].device_status()
        if st != 0:
            raise RuntimeError(f"device status {svdq.STATUS.get(st)} after warm-up")

    # timed pass 1: whole steps, events only at step boundaries (consecutive
    # kernels overlap through programmatic dependent launch)
    clocks = ClockSampler(local)
    clocks.start()
    ev_step = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    for i in range(args.steps):
        flush()
        ev_step[i][0].record(stream)
        run_layers()
        ev_step[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks.mark(False)
    # timed pass 2: the same steps with an event after every kernel, for the
    # per-kernel durations (the events keep consecutive kernels apart)
    nk = len(launches)
    ev_k = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        ev_k[i][0].record(stream)
        run_layers(ev_k[i])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    for d in L:
        st = d["h"].device_status()
        if st != 0:
            raise RuntimeError(f"device status {svdq.STATUS.get(st)} in the timed region")
    ms_step = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_step)
    per_k = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev_k) for j in range(nk)]
    ms_sum = sum(per_k)
    vals = max_over_ranks([ms_step, ms_sum] + per_k, "cuda")
    ms_step, ms_sum, per_k = vals[0], vals[1], vals[2:]

    flops = sum(d["layer"].flops() for d in L)
    value = job_throughput(world, flops, ms_step)

    # end to end through the host entry point (pinned buffers, copies timed):
    # every layer takes its input from host memory and returns its output there
    e2e_steps = max(3, min(args.steps, 20))
    hx = [torch.from_numpy(d["x_bits"].view(np.int16)).pin_memory() for d in L]
    hy = [torch.empty((d["layer"].M, d["layer"].N), dtype=torch.int16).pin_memory() for d in L]

    def host_step():
        for d, xh, yh in zip(L, hx, hy):
            if d["rope"] is None:
                d["h"].linear_forward_host(xh, yh, d["layer"].M)
                continue
            # the QKV-epilogue layer has no host-buffer entry point: the same
            # copies around the device entry point
            d["x"].view(torch.int16).copy_(xh, non_blocking=True)
            d["h"].linear_forward_qkv(d["x"], d["rope"], d["y"], d["layer"].M)
            yh.copy_(d["y"].view(torch.int16), non_blocking=True)

    for _ in range(2):
        host_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        host_step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / e2e_steps
    (ms_e2e,) = max_over_ranks([ms_e2e], "cuda")
    for d in L:
        if d["h"].device_status() != 0:
            raise RuntimeError("device status error in the end-to-end loop")

    pk, pk_src = peaks()
    # dominant kernel: the 4-bit GEMM of the layer with the most work.  NVFP4
    # runs on the FP4 tensor path (dense peak = measured bf16 burst x 4, the
    # 9 : 2.25 PF nominal ratio); INT4 on the int8 path (x 2), or with fp16
    # operands on the 16-bit path (the measured bf16 burst itself)
    di = max(range(len(L)), key=lambda i: L[i]["layer"].flops())
    dl, f16 = L[di]["layer"], L[di]["f16"]
    M, K, N, r = dl.M, dl.K, dl.N, dl.r
    nvfp4 = dl.variant == W.NVFP4
    names_k = [n for n, _ in launches]
    pre_d = dl.name + "." if len(L) > 1 else ""
    kname = pre_d + ("w4a4_gemm_lowrank_up_chain" if di in fused else "w4a4_gemm_lowrank_up")
    ms_kg = per_k[names_k.index(kname)]
    kg_flops = 2.0 * M * K * N + 2.0 * M * N * r
    achieved = kg_flops / (ms_kg * 1e-3) / 1e12
    ratio = 4.0 if nvfp4 else (1.0 if f16 else 2.0)
    peak = pk["bf16_tflops"] * ratio
    if nvfp4:
        peak_src = f"{pk_src} bf16 burst {pk['bf16_tflops']} TFLOP/s x 4 (FP4:BF16 nominal 9:2.25)"
    elif f16:
        peak_src = f"{pk_src} bf16 burst {pk['bf16_tflops']} TFLOP/s (fp16 = bf16 rate)"
    else:
        peak_src = f"{pk_src} bf16 burst {pk['bf16_tflops']} TFLOP/s x 2 (INT8:BF16 nominal 4.5:2.25)"
    # the nominal dense 4-bit / 8-bit tensor rate at the sampled SM clock
    # (2 x 128 x 256 x 64 per SM per 128 cycles for FP4; half that for INT8)
    sm_mhz = clk.get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
    nominal = 148 * 2 * 128 * 256 * 64 / 128 * sm_mhz * 1e6 / 1e12 / (1.0 if nvfp4 else 2.0)
    traffic_key = args.workload + ("/int4_f16" if f16 else "")
    wl = " + ".join(layer_desc(d["layer"], d["f16"], d["rope"] is not None) for d in L)
    kernels = {n: per_k[i] for i, n in enumerate(names_k)}
    line = {
        "metric": metric_name(args.workload, [d["layer"] for d in L]), "value": value, "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4" if nvfp4 else ("int4 (fp16 operands)" if f16 else "int4"), "data": "synthetic",
        "config": {"workload": wl,
                   "l2": ("not flushed: steps back to back (inputs and outputs exceed the 126 MB L2)"
                          if args.l2_warm else
                          "flushed before every step (256 MB write, then 256 MB read; outside the timed events)"),
                   "parallelism": f"replicas x{world}", "tokens_per_step": L[0]["layer"].M * world,
                   "chained": [d["layer"].name for d in L if d["chained"]],
                   "fused_pairs": [L[i]["layer"].name + "->" + L[i + 1]["layer"].name for i in sorted(fused)],
                   "qkv_epilogue": [d["layer"].name for d in L if d["rope"] is not None],
                   "timing": "ms_per_step: events at step boundaries only (kernels overlap through "
                             "programmatic dependent launch); kernels_ms: a second timed pass with an "
                             "event after every kernel"},
        "tokens_per_s": world * L[0]["layer"].M / (ms_step * 1e-3),
        "frac_of_fp4_roofline": None,
        "kernels_ms": kernels,
        "kernels_sum_ms": ms_sum,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic("w4a4_gemm_lowrank_up", traffic_key),
                     "peak_source": peak_src, "kernel": kname,
                     "nominal_peak": nominal, "frac_of_nominal": achieved / nominal,
                     "nominal_source": f"{'FP4' if nvfp4 else 'INT8'} dense tcgen05 rate at {sm_mhz:.0f} MHz "
                                       "(128x256x64 per SM per 128 cycles)"},
        "e2e": {"value": job_throughput(world, flops, ms_e2e), "unit": "TFLOPS",
                "h2d_bytes_per_step": sum(d["layer"].M * d["layer"].K * 2 for d in L),
                "d2h_bytes_per_step": sum(d["layer"].M * d["layer"].N * 2 for d in L)},
        # the qkv-epilogue call launches the rotary-table copy and the GEMM
        "gpu_launches": sum(2 if n.endswith("_qkv") else 1 for n, _ in launches) * args.steps,
        "clocks": clk,
        "kernel_source_hash": kernel_source_hash(),
    }
    # whole-step roofline: the slower of 4-bit compute and the step's HBM bytes
    bytes_alg = sum(layer_bytes(d["layer"]) for d in L)
    t_star = max(flops / (peak * 1e12), bytes_alg / (pk["hbm_gbs"] * 1e9))
    line["frac_of_fp4_roofline"] = t_star / (ms_step * 1e-3)
    line["frac_of_nominal_roofline"] = max(flops / (nominal * 1e12),
                                           bytes_alg / (pk["hbm_gbs"] * 1e9)) / (ms_step * 1e-3)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(L[0]["layer"], L[0]["pw"], L[0]["x_bits"], 1024)
    if rank == 0 and world == 1 and not args.no_scheme_error:
        line["scheme_error"] = {d["layer"].name: scheme_error(d["layer"], d["f16"]) for d in L}
    if args.overhead_repeats > 0 and len(L) == 1 and world == 1:
        line["lowrank_overhead"] = lowrank_overhead(L[0], args.steps, args.overhead_repeats, flush)
    if rank == 0:
        print(json.dumps(line), flush=True)
    for d in L:
        d["h"].close()
    if world > 1:
        dist.destroy_process_group()


def run_awq(args, layer):
    """The AWQ W4A16 modulation linear: one call per step, HBM-bound on the
    4-bit weight stream."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from bit_diffusion_transformer_w4a4_b200 import svdq
    from bit_diffusion_transformer_w4a4_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    M, K, N = layer.M, layer.K, layer.N
    if args.impl == "reference":
        if rank == 0:
            from oracle import awq as A
            p = W.synthetic_awq(layer)
            xb = W.awq_activations(layer)
            for _ in range(min(args.warmup, 3)):
                A.forward(xb, p)
            ts = []
            for _ in range(min(args.steps, 20)):
                t = time.perf_counter()
                A.forward(xb, p)
                ts.append(time.perf_counter() - t)
            ms = statistics.median(ts) * 1e3
            v = (layer.weight_bytes() + M * K * 2 + M * N * 2) / (ms * 1e-3) / 1e9
            print(json.dumps({"metric": f"AWQ W4A16 linear weight-stream GB/s at M{M} K{K} N{N}", "value": v,
                              "unit": "GB/s", "n_gpus": args.gpus, "steps": len(ts), "warmup": min(args.warmup, 3),
                              "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                              "dtype": "f64", "data": "synthetic", "impl": "reference",
                              "config": {"workload": f"{layer.name} M{M} K{K} N{N} awq_w4a16_g64"},
                              "cpu_baseline": {"value": v, "unit": "GB/s", "kind": "oracle",
                                               "cores": os.cpu_count(), "sample": "the whole call"},
                              "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    p = W.synthetic_awq(layer, seed=rank)
    xb = W.awq_activations(layer, seed=rank)
    h = svdq.AWQWeights(p, M)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        if not args.l2_warm:
            flush_w.zero_(); flush_r.sum()
        h.forward(x, y, M)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        if not args.l2_warm:
            flush_w.zero_(); flush_r.sum()
        evs[i][0].record(stream)
        h.forward(x, y, M)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    (ms,) = max_over_ranks([ms], "cuda")
    nbytes = layer.weight_bytes() + M * K * 2 + M * N * 2 + K * 4 + (N * 2 if p.bias is not None else 0)
    gbs = world * nbytes / (ms * 1e-3) / 1e9
    xh = torch.from_numpy(xb.view(np.int16)).pin_memory()
    yh = torch.empty((M, N), dtype=torch.int16).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    xd = torch.empty_like(x)
    n_e2e = max(3, min(args.steps, 50))
    e0.record(stream)
    for _ in range(n_e2e):
        xd.view(torch.int16).copy_(xh, non_blocking=True)
        h.forward(xd, y, M)
        yh.copy_(y.view(torch.int16), non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / n_e2e
    (ms_e2e,) = max_over_ranks([ms_e2e], "cuda")
    pk, pk_src = peaks()
    line = {"metric": f"AWQ W4A16 linear weight-stream GB/s at M{M} K{K} N{N}", "value": gbs, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x int4",
            "data": "synthetic",
            "config": {"workload": f"{layer.name} M{M} K{K} N{N} awq_w4a16_g64",
                       "l2": ("not flushed: steps back to back (inputs and outputs exceed the 126 MB L2)"
                          if args.l2_warm else
                          "flushed before every step (256 MB write, then 256 MB read; outside the timed events)"),
                       "parallelism": f"replicas x{world}"},
            "tokens_per_s": world * M / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "traffic": recorded_traffic("awq_w4a16_forward", args.workload),
                         "peak_source": f"{pk_src} copy bandwidth", "kernel": "kawq_kernel",
                         "bytes_per_launch": nbytes},
            "e2e": {"value": world * nbytes / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2},
            "gpu_launches": args.steps, "clocks": clk, "kernel_source_hash": kernel_source_hash()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import awq as A
        t = time.perf_counter()
        A.forward(xb, p)
        dt = time.perf_counter() - t
        line["cpu_baseline"] = {"value": nbytes / dt / 1e9, "unit": "GB/s", "kind": "oracle",
                                "cores": os.cpu_count(), "sample": f"the whole call (numpy fp64), {dt:.2f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    if args.workload in W.awq_workloads():
        run_awq(args, W.awq_workloads()[args.workload])
        return
    layers = W.workloads()[args.workload]
    if args.impl == "reference":
        run_reference(args, layers)
    else:
        run_ours(args, layers)


if __name__ == "__main__":
    main()
