"""Benchmark of the B200 FP8 x FP4 MoE expert layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference] [--workload ID]

A step is one moe_forward (routing + gather, GEMM1 + SwiGLU + requant, GEMM2,
combine) over one batch of seeded synthetic inputs already resident in HBM.
The default workload is the decode case (T=8, E=384, top-6, H=7168, I=3072);
``--workload`` picks another row of the workload table.  With N > 1 (torchrun,
one process per GPU) every rank runs an independent replica of the layer (the
single-GPU layer has no exchange step) and the value is the whole job's
throughput.  Prints one JSON line on rank 0.

``--impl reference`` times the CPU oracle on the host cores instead (a bounded
sample of the same workload per step), as the comparison arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "MoE layer µs & TFLOP/s (E=384,k=6,H=7168,I=3072); % of HBM/TC roofline"
# B200 specification figures, reported beside the measured-peak fractions:
# HBM3e 8 TB/s, dense FP8 4.5 PFLOP/s (the FP8 x FP4 block-scaled MMA rate)
SPEC_HBM_GBPS = 8000.0
SPEC_FP8_TFLOPS = 4500.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--workload", type=int, default=1)
    p.add_argument("--also", default=None,
                   help="comma-separated workload ids measured after the headline one in the same run "
                        "(default: 2,3,4 when the headline is the decode workload; '' for none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-tokens", type=int, default=8, help="tokens in the oracle's timed sample")
    p.add_argument("--experts", type=int, default=0,
                   help="override E (a smaller resident weight set for profiler captures)")
    p.add_argument("--tokens", type=int, default=0, help="override T (with --experts: same rows per expert)")
    p.add_argument("--layout", default="packets", choices=["packets", "rowmajor"],
                   help="weight layout: tile packets, or row-major bodies with separate scale blocks")
    p.add_argument("--format", default="mx", choices=["mx", "nvfp4"],
                   help="mx: FP8 activations x FP4 weights, UE8M0 per 32; nvfp4: E2M1 x E2M1, UE4M3 per 16")
    p.add_argument("--shared-expert", type=int, default=0, metavar="T",
                   help="time the BF16 shared expert (moe_shared_forward) on T tokens instead of the layer")
    p.add_argument("--shared-dims", default="7168,2048", help="SH,SI of the shared expert")
    p.add_argument("--ep", action="store_true",
                   help="expert parallelism: rank r of N holds experts [r E/N, (r+1) E/N) and T tokens of its own; "
                        "NCCL all-to-alls around the library's dispatch and combine")
    p.add_argument("--fp8-peak", action="store_true",
                   help="measure cuBLAS FP8 8192^3 matmul throughput (MX block-scaled and per-tensor scaled), "
                        "burst and sustained")
    return p.parse_args()


SPEC_BF16_TFLOPS = 2250.0


def run_shared(args, rank, world, local_rank):
    """The BF16 shared expert alone: T tokens through moe_shared_forward, inputs
    resident in HBM. Its weights (88 MB at SH=7168, SI=2048) fit in L2, so L2
    is flushed (a 256 MB write) before every timed call and CUDA events on the
    launch stream bracket each call; the same K calls back to back without
    the flush are reported beside it. For context, the same computation as
    torch operators (cuBLAS GEMMs + elementwise activation), timed the same
    two ways."""
    import moe_expert_layer_08_b200 as moe
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    T = args.shared_expert
    SH, SI = (int(v) for v in args.shared_dims.split(","))
    x, l1, l2 = W.gen_shared(T, SH, SI, 1, device)
    ws = moe.shared_workspace(T, SH, SI, device)
    out = torch.empty((T, SH), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        barrier()
        start.record(stream)
        for _ in range(args.steps):
            fn()
        stop.record(stream)
        barrier()
        return max_over_ranks(start.elapsed_time(stop) / args.steps, device)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # twice the 126 MB L2

    def timed_flushed(fn):
        for _ in range(args.warmup):
            flush.fill_(1)
            fn()
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i, (a, b) in enumerate(ev):
            flush.fill_(i & 0xFF)
            a.record(stream)
            fn()
            b.record(stream)
        barrier()
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, device)

    def timed_graph(fn):
        """K calls captured in one CUDA graph (the two kernels of consecutive
        calls keep their programmatic overlap), replayed W times untimed and
        once timed: back-to-back calls without the host's per-call enqueue
        cost, which at small T is above the device time. None when capture
        fails."""
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(args.steps):
                    fn()
        except Exception:  # noqa: BLE001 -- reported as unmeasured
            return None
        for _ in range(args.warmup):
            g.replay()
        barrier()
        start.record(stream)
        g.replay()
        stop.record(stream)
        barrier()
        del g
        return max_over_ranks(start.elapsed_time(stop) / args.steps, device)

    call = lambda: moe.shared_forward(x, l1, l2, out=out, workspace=ws)
    with ClockSampler(device.index) as clocks:
        ms = timed_flushed(call)
    ms_resident = timed(call)
    ms_graph = timed_graph(call)
    st = moe.check_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {moe.STATUS.get(st, st)}")

    def torch_ops():
        g, u = torch.nn.functional.linear(x, l1).chunk(2, dim=-1)
        h = (torch.nn.functional.silu(g.float()) * u.float()).to(torch.bfloat16)
        return torch.nn.functional.linear(h, l2)

    torch_ms = timed_flushed(torch_ops)
    torch_ms_resident = timed(torch_ops)
    torch_ms_graph = timed_graph(torch_ops)
    if rank != 0:
        return
    pk = peaks()
    flops = 2.0 * T * 3 * SH * SI
    tf = flops / (ms * 1e-3) / 1e12
    wbytes = 3 * SH * SI * 2
    line = {
        "metric": f"BF16 shared expert TFLOP/s (SH={SH}, SI={SI})", "value": world * tf, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic",
        "dtype": "bf16 (fp32 accumulate)",
        "config": {"workload": f"shared_expert_T{T}", "T": T, "SH": SH, "SI": SI, "activation": "swiglu",
                   "parallelism": f"replicas x{world}",
                   "l2": "flushed before every timed call (256 MB write), events around each call"},
        "us_per_call": ms * 1e3,
        "us_per_call_l2_resident": ms_resident * 1e3,
        "us_per_call_l2_resident_graph": None if ms_graph is None else ms_graph * 1e3,
        "roofline": shared_roofline(flops, wbytes, ms, pk),
        "torch_ops_us": torch_ms * 1e3,
        "torch_ops_us_l2_resident": torch_ms_resident * 1e3,
        "torch_ops_us_l2_resident_graph": None if torch_ms_graph is None else torch_ms_graph * 1e3,
        "gpu_launches": args.steps * 2,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def shared_roofline(flops, wbytes, ms, pk):
    """The binding roofline of one shared-expert call: the tensor pipe
    (FLOPs at the sustained bf16 peak) or HBM (the 3·SH·SI bf16 weights read
    once at the measured copy bandwidth), whichever takes longer; the other
    figure beside it."""
    tf = flops / (ms * 1e-3) / 1e12
    gbps = wbytes / (ms * 1e-3) / 1e9
    tensor = {"achieved": tf, "peak": pk["bf16_sustained"], "unit": "TFLOP/s", "frac": tf / pk["bf16_sustained"],
              "peak_source": pk["source"] + " sustained bf16", "frac_of_burst": tf / pk["bf16"],
              "spec": {"peak": SPEC_BF16_TFLOPS, "frac": tf / SPEC_BF16_TFLOPS}}
    hbm = {"achieved": gbps, "peak": pk["hbm"], "unit": "GB/s", "frac": gbps / pk["hbm"],
           "peak_source": pk["source"] + " copy bandwidth", "algorithmic_bytes": wbytes}
    hbm_bound = wbytes / (pk["hbm"] * 1e9) > flops / (pk["bf16_sustained"] * 1e12)
    main, other = (hbm, tensor) if hbm_bound else (tensor, hbm)
    return {"kernel": "shared_gemm_kernel (GEMM1 + GEMM2)", "bound": "hbm" if hbm_bound else "tensor", **main,
            "other": {"bound": "tensor" if hbm_bound else "hbm", **other}, "traffic": None}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def cublas_fp8():
    """The measured cuBLAS FP8 matmul figures committed beside the ncu
    summaries (`--fp8-peak` writes them), or None: context for the FP8 tensor
    roofline, whose denominator stays 2 x the measured bf16 peak."""
    path = os.path.join(ROOT, "profiles", "cublas_fp8_matmul_8192.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    return {arm: dict(burst=float(d[arm]["burst_tflops"]), sustained=float(d[arm]["sustained_tflops"]))
            for arm in ("mx_blockwise_1x32", "per_tensor") if arm in d}


def expert_bytes(w, fmt="mx"):
    """FP4 + scale bytes of one expert's L1 and L2: 0.5 + 1/32 byte per weight
    (UE8M0 per 32), or 0.5 + 1/16 (NVFP4, UE4M3 per 16)."""
    num, den = (17, 32) if fmt == "mx" else (9, 16)
    return 2 * w.I * w.H * num // den, w.H * w.I * num // den


class ClockSampler:
    """Samples SM clock and throttle reasons (read-only NVML queries) from a
    background thread every 5 ms while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.sm, self.smax, self.reasons = [], [], set()
        self.ok = False

    def _run(self):
        import pynvml
        try:  # the NVML handle of the CUDA device, matched by PCI address
            p = torch.cuda.get_device_properties(self.index)
            h = pynvml.nvmlDeviceGetHandleByPciBusId(
                f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0")
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        self.smax.append(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        while not self._stop.is_set():
            self.sm.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
            self._stop.wait(0.005)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.ok = True
        except Exception:
            return self
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        # the timed region starts once sampling runs (NVML's handle lookup can
        # take longer than a short region)
        t0 = time.time()
        while not self.sm and time.time() - t0 < 2.0:
            time.sleep(0.001)
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join(timeout=5)

    def summary(self):
        if not self.sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": max(self.smax) if self.smax else None,
                "reasons": sorted(self.reasons), "samples": len(self.sm)}


def kernel_source_hash() -> str:
    import hashlib
    files = ["gemm.cu", "moe_common.cuh", "moe_internal.h"]
    src = b"".join(open(os.path.join(ROOT, "moe_expert_layer_08_b200", "csrc", f), "rb").read() for f in files)
    return hashlib.sha256(src).hexdigest()


def measured_traffic(w, touched, gemm1: bool, fmt="mx"):
    """DRAM bytes per launch of the dominant GEMM from the committed ncu
    capture (scaled by touched experts, which the traffic is proportional
    to), or None when the kernel changed since or another variant runs."""
    regime = "decode" if w.T * w.k <= 8 * w.E else "prefill"
    path = os.path.join(ROOT, "profiles", f"gemm_{regime}_traffic.json")
    if not os.path.exists(path) or fmt != "mx":
        return None
    d = json.load(open(path))
    if d.get("kernel_source_sha256") != kernel_source_hash():
        return None
    return touched * d["gemm1_bytes_per_touched_expert" if gemm1 else "gemm2_bytes_per_touched_expert"]


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job is as slow as its slowest
    replica); identity without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def build_layer(w, device, layout="packets", fmt="mx"):
    """Seeded bf16 draws quantised and laid out by the CUDA library, resident in
    HBM: tile packets (l1_t, l2_t) or row-major bodies + scale blocks (rm);
    fmt "nvfp4": NVFP4 activations and packets."""
    import moe_expert_layer_08_b200 as moe
    x = W.gen_x(w, device)
    idx, tw = W.gen_routing(w, device)
    u8 = dict(dtype=torch.uint8, device=device)
    if fmt == "nvfp4":
        xq, xs = moe.quantize_nvfp4(x)
        n1, n2 = moe.transformed_weight_bytes_nvfp4(w.E, w.H, w.I)
        l1_t, l2_t = torch.empty(n1, **u8), torch.empty(n2, **u8)
        p1, p2 = n1 // w.E, n2 // w.E
        for e in range(w.E):
            a, b = moe.quantize_nvfp4(W.gen_l1(w, e, device))
            c, d = moe.quantize_nvfp4(W.gen_l2(w, e, device))
            moe.transform_weights_nvfp4(a[None], b[None], c[None], d[None],
                                        out=(l1_t[e * p1:(e + 1) * p1], l2_t[e * p2:(e + 1) * p2]))
        torch.cuda.synchronize()
        return dict(x=x, xq=xq, xs=xs, idx=idx, tw=tw, l1_t=l1_t, l2_t=l2_t, rm=None)
    xq, xs = moe.quantize_fp8(x)
    if layout == "packets":
        n1, n2 = moe.transformed_weight_bytes(w.E, w.H, w.I)
        l1_t, l2_t = torch.empty(n1, **u8), torch.empty(n2, **u8)
        p1, p2 = n1 // w.E, n2 // w.E
    else:
        r1, r2 = torch.empty((w.E, 2 * w.I, w.H // 2), **u8), torch.empty((w.E, w.H, w.I // 2), **u8)
        m1, m2 = moe.transformed_scale_bytes(w.E, w.H, w.I)
        s1, s2 = torch.empty(m1, **u8), torch.empty(m2, **u8)
        q1, q2 = m1 // w.E, m2 // w.E
    for e in range(w.E):
        a, b = moe.quantize_fp4(W.gen_l1(w, e, device))
        c, d = moe.quantize_fp4(W.gen_l2(w, e, device))
        if layout == "packets":
            moe.transform_weights(a[None], b[None], c[None], d[None],
                                  out=(l1_t[e * p1:(e + 1) * p1], l2_t[e * p2:(e + 1) * p2]))
        else:
            r1[e], r2[e] = a, c
            moe.transform_scales(b[None], d[None], out=(s1[e * q1:(e + 1) * q1], s2[e * q2:(e + 1) * q2]))
    torch.cuda.synchronize()
    g = dict(x=x, xq=xq, xs=xs, idx=idx, tw=tw)
    if layout == "packets":
        g.update(l1_t=l1_t, l2_t=l2_t, rm=None)
    else:
        g.update(l1_t=None, l2_t=None, rm=moe.RowMajorWeights(r1, s1, r2, s2))
    return g


def oracle_sample(w, ntok, device, fmt="mx"):
    """Host inputs of the oracle for the first ``ntok`` tokens (oracle-quantised)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    x = W.gen_x(w, device)
    idx, tw = W.gen_routing(w, device)
    idx, tw = idx.cpu().numpy(), tw.cpu().numpy()
    tokens = np.arange(min(ntok, w.T), dtype=np.int32)
    qx, qw = (oracle.quantize_nvfp4, oracle.quantize_nvfp4) if fmt == "nvfp4" else \
        (oracle.quantize_e4m3, oracle.quantize_e2m1)
    xq, xs = qx(x.float().cpu().numpy())
    need = sorted(set(int(e) for e in idx[tokens].ravel()))

    def quant(item):
        e, a, b = item
        return e, qw(a) + qw(b)

    with ThreadPoolExecutor(max(1, min(len(need), os.cpu_count() or 1))) as pool:
        futs = [pool.submit(quant, (e, W.gen_l1(w, e, device).float().cpu().numpy(),
                                    W.gen_l2(w, e, device).float().cpu().numpy())) for e in need]
        experts = dict(f.result() for f in futs)
    return dict(xq=xq, xs=xs, idx=idx, tw=tw, experts=experts, tokens=tokens, fmt=fmt)


def time_oracle(w, s, steps):
    import oracle
    threads = min(len(s["tokens"]), oracle.num_threads(0))
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.forward(s["xq"], s["xs"], s["idx"], s["tw"], s["experts"], w.E, w.H, w.I,
                       tokens=s["tokens"], threads=threads, fmt=s["fmt"])
        times.append(time.perf_counter() - t0)
    flops = 2 * len(s["tokens"]) * w.k * 3 * w.H * w.I
    return flops, times, threads


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    device = "cuda" if torch.cuda.is_available() else "cpu"
    s = oracle_sample(w, args.cpu_tokens, device, args.format)
    flops, times, threads = time_oracle(w, s, args.warmup + args.steps)
    t = float(np.mean(times[args.warmup:])) if args.steps > 0 else float(np.mean(times))
    value = flops / t / 1e12
    sample = f"first {len(s['tokens'])} of {w.T} tokens (all {w.k} experts each) per step"
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, args, world, len(W.touched_experts(torch.from_numpy(s["idx"]), w.E)),
                                  expert_bytes(w, args.format)),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_fp8_peak(args):
    """Library FP8 reference figures for the tensor roofline, 8192^3 E4M3 x
    E4M3 matmuls with bf16 output: MX block scaling (UE8M0 per 32 along K,
    F.scaled_mm -> cuBLAS) and per-tensor scales (torch._scaled_mm), each as
    the best of 10 timed calls (burst) and back to back for ~4 s
    (sustained)."""
    import torch.nn.functional as F
    device = torch.device("cuda", 0)
    n = 8192
    g = torch.Generator(device=device).manual_seed(0)
    a = torch.randn((n, n), device=device, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn((n, n), device=device, generator=g).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=device)
    # scale 2^0 everywhere: the swizzled image of a constant is the constant
    sf = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=device).view(torch.float8_e8m0fnu)
    blk, swz = F.ScalingType.BlockWise1x32, F.SwizzleType.SWIZZLE_32_4_4
    arms = {
        "mx_blockwise_1x32": lambda: F.scaled_mm(a, b, sf, blk, sf, blk, swizzle_a=swz, swizzle_b=swz,
                                                 output_dtype=torch.bfloat16),
        "per_tensor": lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
    }
    flops = 2.0 * n ** 3
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = {"metric": "cuBLAS FP8 E4M3 8192^3 matmul, bf16 out", "unit": "TFLOP/s"}
    for name, mm in arms.items():
        try:
            mm()
            torch.cuda.synchronize()
        except (RuntimeError, TypeError, ValueError) as e:
            out[name] = {"unavailable": str(e).splitlines()[0][:200]}
            continue
        for _ in range(5):
            mm()
        best = 0.0
        for _ in range(10):
            s0.record()
            mm()
            s1.record()
            torch.cuda.synchronize()
            best = max(best, flops / (s0.elapsed_time(s1) * 1e-3) / 1e12)
        with ClockSampler(device.index) as clocks:
            reps, t_end = 0, time.time() + 4.0
            s0.record()
            while time.time() < t_end:
                for _ in range(20):
                    mm()
                reps += 20
                torch.cuda.synchronize()
            s1.record()
            torch.cuda.synchronize()
        out[name] = {"burst": best, "sustained": flops * reps / (s0.elapsed_time(s1) * 1e-3) / 1e12,
                     "clocks": clocks.summary()}
    print(json.dumps(out), flush=True)


def run_ep(args, w, rank, world, local_rank):
    """Expert-parallel steps (moe_expert_layer_08_b200.ep): every rank routes
    its own T tokens over all E experts and holds E / N of them; a step is
    the dispatch, the count all-gather and row all-to-alls, the layer over the
    received rows, the all-to-all back and the combine.  Timed like the main
    arm (barrier + CUDA events around K steps, max over ranks); the step
    includes its one host synchronisation (the split sizes)."""
    import moe_expert_layer_08_b200 as moe
    from moe_expert_layer_08_b200 import build as mbuild
    from moe_expert_layer_08_b200.ep import ExpertParallelLayer
    if rank == 0:
        mbuild.build()
    if world > 1:
        torch.distributed.barrier()
    if w.E % world:
        raise SystemExit(f"E = {w.E} is not a multiple of {world} ranks")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    e_loc = w.E // world
    mine = W.custom(f"{w.name}_rank{rank}", T=w.T, E=w.E, k=w.k, H=w.H, I=w.I, seed=w.seed + 7919 * rank,
                    routing=w.routing, zipf_s=w.zipf_s)
    x = W.gen_x(mine, device)
    idx, tw = W.gen_routing(mine, device)
    xq, xs = moe.quantize_fp8(x)
    n1, n2 = moe.transformed_weight_bytes(w.E, w.H, w.I)
    p1, p2 = n1 // w.E, n2 // w.E
    l1_t = torch.empty(e_loc * p1, dtype=torch.uint8, device=device)
    l2_t = torch.empty(e_loc * p2, dtype=torch.uint8, device=device)
    for i, e in enumerate(range(rank * e_loc, (rank + 1) * e_loc)):   # the experts' draws depend on w.seed only
        a, b = moe.quantize_fp4(W.gen_l1(w, e, device))
        c, d = moe.quantize_fp4(W.gen_l2(w, e, device))
        moe.transform_weights(a[None], b[None], c[None], d[None],
                              out=(l1_t[i * p1:(i + 1) * p1], l2_t[i * p2:(i + 1) * p2]))
    torch.cuda.synchronize(device)
    layer = ExpertParallelLayer(l1_t, l2_t, w.E, w.k, w.H, w.I, T_max=w.T)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        layer(xq, xs, idx, tw, out=out)

    for _ in range(args.warmup):
        step()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clocks:
        barrier()
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        barrier()
    ms = max_over_ranks(start.elapsed_time(stop) / args.steps, device)
    st = layer.check()  # the dispatch's error word, then the expert layer's
    if st != 0:
        raise RuntimeError(f"device error: {moe.STATUS.get(st, st)}")
    # kernels of this library per step: routing (one block up to 1024 rows,
    # else four kernels) + pack, the layer over the received rows, the combine
    route = 1 if w.T * w.k <= 1024 else 4
    launches = route + 1 + moe.forward_kernel_launches(layer.last_n_recv, e_loc, 1, w.H, w.I) + 1
    if rank == 0:
        line = {
            "metric": METRIC, "value": world * w.flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "data": "synthetic", "dtype": "fp8xfp4 (fp32 accumulate)",
            "config": {"workload": w.name, **{k: getattr(w, k) for k in ("T", "E", "k", "H", "I", "routing")},
                       "tokens_per_rank": w.T, "experts_per_rank": e_loc, "parallelism": f"ep{world}",
                       "exchange": "NCCL all_gather (counts) + all_to_all_single (rows out, outputs back)"
                       if world > 1 else "none (one rank)"},
            "us_per_layer": ms * 1e3,
            "gpu_launches": args.steps * launches,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)


def run_shared_reference(args, rank):
    """The oracle's shared expert on the host cores, on the first
    ``--cpu-tokens`` of the T tokens per step (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    T = args.shared_expert
    SH, SI = (int(v) for v in args.shared_dims.split(","))
    x, l1, l2 = W.gen_shared(T, SH, SI, 1, "cuda" if torch.cuda.is_available() else "cpu")
    u16 = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16)
    xb, l1b, l2b = u16(x), u16(l1), u16(l2)
    n = min(args.cpu_tokens, T)
    tok = np.arange(n, dtype=np.int32)
    times = []
    for _ in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.shared_forward(xb, l1b, l2b, tokens=tok)
        times.append(time.perf_counter() - t0)
    t = float(np.mean(times[args.warmup:])) if args.steps > 0 else float(np.mean(times))
    value = 2.0 * n * 3 * SH * SI / t / 1e12
    threads = min(oracle.num_threads(), n)
    line = {
        "metric": f"BF16 shared expert TFLOP/s (SH={SH}, SI={SI})", "impl": "reference", "value": value,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"shared_expert_T{T}", "T": T, "SH": SH, "SI": SI, "activation": "swiglu"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {n} of {T} tokens per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, args, world, touched=None, b12=None):
    """The `config` object of a bench line (the same keys in both arms)."""
    cfg = {"workload": w.name, **{k: getattr(w, k) for k in ("T", "E", "k", "H", "I", "seed", "routing")},
           "parallelism": f"replicas x{world}", "weight_layout": args.layout}
    if touched is not None:
        cfg["l2"] = ("inputs larger than L2 (touched expert weights per step >> 126 MB)"
                     if touched * sum(b12) > 256e6 else "inputs fit in L2 (not flushed)")
    return cfg


def time_layer(args, w, device, world):
    """Seeded inputs and weights of workload w resident in HBM, W warm-up
    layer calls, then K calls back to back timed with CUDA events on the launch
    stream (barrier + synchronize on both sides), then the same K calls again
    with an event between kernels for the per-kernel times."""
    import moe_expert_layer_08_b200 as moe
    g = build_layer(w, device, args.layout, args.format)
    layer = moe.MoELayer(g["l1_t"], g["l2_t"], w.E, w.k, w.H, w.I, T_max=w.T, device=device, weights=g["rm"],
                         fmt=args.format)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.NUM_STAGE_EVENTS)]
          for _ in range(args.steps)]

    def step(events=None):
        layer(g["xq"], g["xs"], g["idx"], g["tw"], out=out, events=events, stream=stream)

    for _ in range(args.warmup):
        step()
    st = moe.check_device_error(layer.workspace)
    if st != 0:
        raise RuntimeError(f"device error after warm-up: {moe.STATUS.get(st, st)}")

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clocks:
        # the timed region: K layer calls back to back, nothing else enqueued
        barrier()
        start.record(stream)
        for i in range(args.steps):
            step()
        stop.record(stream)
        barrier()
        total_ms = start.elapsed_time(stop)
        # per-kernel durations: the same K calls again with an event between
        # kernels (an event breaks the programmatic overlap of consecutive
        # kernels, so this pass is a little slower and is not the headline)
        barrier()
        start.record(stream)
        for i in range(args.steps):
            step(ev[i])
        stop.record(stream)
        barrier()
        staged_ms = start.elapsed_time(stop) / args.steps
    st = moe.check_device_error(layer.workspace)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {moe.STATUS.get(st, st)}")
    stage_ms = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(moe.NUM_STAGE_EVENTS - 1)] for e in ev])
    ms = max_over_ranks(total_ms / args.steps, device)
    return dict(g=g, layer=layer, out=out, stream=stream, ms=ms, staged_ms=staged_ms, stage_ms=stage_ms,
                clocks=clocks.summary(), barrier=barrier)


def layer_figures(args, w, r, world):
    """Throughput, per-kernel times and rooflines of one timed workload."""
    import moe_expert_layer_08_b200 as moe
    g, ms, stage_ms = r["g"], r["ms"], r["stage_ms"]
    # roofline of the dominant kernel (GEMM1 or GEMM2), timed by the stage events
    touched = len(W.touched_experts(g["idx"].cpu(), w.E))
    b1, b2 = expert_bytes(w, args.format)
    g1_ms, g2_ms = float(stage_ms[:, 1].mean()), float(stage_ms[:, 2].mean())
    pk = peaks()
    if g1_ms >= g2_ms:
        kname, kms, kbytes = "moe_gemm_kernel<gemm1>", g1_ms, touched * b1
    else:
        kname, kms, kbytes = "moe_gemm_kernel<gemm2>", g2_ms, touched * b2
    achieved = kbytes / (kms * 1e-3) / 1e9
    traffic = measured_traffic(w, touched, g1_ms >= g2_ms, args.format)
    roofline = {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "peak_source": pk["source"], "algorithmic_bytes": kbytes,
                "traffic": traffic, "spec": {"peak": SPEC_HBM_GBPS, "frac": achieved / SPEC_HBM_GBPS}}
    # tensor peaks: FP8 = 2 x measured bf16, FP4 (NVFP4) = 4 x (the nominal
    # dense ratios); the block-scaled FP8 x FP4 MMA runs at the FP8 rate
    ratio = 2.0 if args.format == "mx" else 4.0
    spec_tc = SPEC_FP8_TFLOPS * ratio / 2.0
    # the binding roofline of the dominant kernel: its algorithmic FLOPs at the
    # sustained tensor peak (the power-capped regime of a long run; burst and
    # spec beside it, and "clocks" shows the regime the timed region ran in)
    # against its algorithmic bytes at the measured HBM bandwidth, whichever
    # takes longer; the other fraction is reported beside it
    kflops = 2.0 * w.T * w.k * (2 * w.I if g1_ms >= g2_ms else w.H) * (w.H if g1_ms >= g2_ms else w.I)
    peak_s, peak_b = ratio * pk["bf16_sustained"], ratio * pk["bf16"]
    tflops = kflops / (kms * 1e-3) / 1e12
    tensor_frac = {"achieved": tflops, "peak": peak_s, "unit": "TFLOP/s", "frac": tflops / peak_s,
                   "frac_of_burst": tflops / peak_b, "algorithmic_flops": kflops}
    if kflops / (peak_s * 1e12) <= kbytes / (pk["hbm"] * 1e9):
        roofline["tensor"] = tensor_frac
    else:
        roofline = {"kernel": kname, "bound": "tensor", "achieved": tflops, "peak": peak_s, "unit": "TFLOP/s",
                    "frac": tflops / peak_s,
                    "peak_source": pk["source"] + f" sustained ({ratio:g} x bf16_tflops_sustained)",
                    "frac_of_burst": tflops / peak_b,
                    "burst_peak": peak_b,
                    "spec": {"peak": spec_tc, "frac": tflops / spec_tc},
                    "algorithmic_flops": kflops,
                    "traffic": traffic, "hbm": {"achieved_GBps": achieved, "frac": achieved / pk["hbm"]}}
        if cublas_fp8() and args.format == "mx":
            roofline["cublas_fp8"] = {arm: {"sustained": c["sustained"], "frac": tflops / c["sustained"],
                                            "burst": c["burst"], "frac_of_burst": tflops / c["burst"]}
                                      for arm, c in cublas_fp8().items()}
    x_bytes = w.T * w.H * 33 // 32 if args.format == "mx" else w.T * w.H * 9 // 16
    layer_bytes = touched * (b1 + b2) + x_bytes + w.T * w.k * 12 + w.T * w.H * 2
    tflops_layer = w.flops / (ms * 1e-3) / 1e12
    layer_tc = {"sustained": tflops_layer / (ratio * pk["bf16_sustained"]),
                "burst": tflops_layer / (ratio * pk["bf16"]),
                "spec": tflops_layer / spec_tc}
    if cublas_fp8() and args.format == "mx":
        layer_tc["cublas_fp8_sustained"] = {arm: tflops_layer / c["sustained"] for arm, c in cublas_fp8().items()}
    return {
        "value": world * tflops_layer, "ms_per_step": ms, "touched": touched, "b12": (b1, b2),
        "us_per_layer": ms * 1e3,
        "effective_GBps": layer_bytes / (ms * 1e-3) / 1e9,
        "hbm_frac_layer": layer_bytes / (ms * 1e-3) / 1e9 / pk["hbm"],
        "touched_experts": touched,
        "stage_us": {"route_gather": float(stage_ms[:, 0].mean() * 1e3), "gemm1": g1_ms * 1e3,
                     "gemm2": g2_ms * 1e3, "combine": float(stage_ms[:, 3].mean() * 1e3)},
        "stage_timing": {"how": "second pass of the same K steps with a CUDA event on the launch stream "
                                "between kernels; the roofline's kernel duration comes from it",
                         "us_per_layer": r["staged_ms"] * 1e3},
        "roofline": roofline,
        "layer_frac_of_tensor_peak": layer_tc,
        "layer_frac_of_hbm_spec": layer_bytes / (ms * 1e-3) / 1e9 / SPEC_HBM_GBPS,
        "gpu_launches": args.steps * moe.forward_kernel_launches(w.T, w.E, w.k, w.H, w.I),
        "clocks": r["clocks"],
    }


def run_b200(args, w, rank, world, local_rank):
    import moe_expert_layer_08_b200 as moe
    from moe_expert_layer_08_b200 import build as mbuild
    if rank == 0:
        mbuild.build()
    if world > 1:
        torch.distributed.barrier()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if args.format == "nvfp4" and args.layout != "packets":
        raise SystemExit("the NVFP4 variant takes packet weights")
    r = time_layer(args, w, device, world)
    g, layer, out, stream, barrier = r["g"], r["layer"], r["out"], r["stream"], r["barrier"]

    # end to end through the public API: pinned host inputs -> device -> layer -> host output,
    # every step's copies inside the timed region. The step's four inputs sit in
    # one pinned staging buffer (256-byte aligned sections) and move in one
    # host-to-device copy; the layer reads views of the device copy. As a
    # serving loop would, the copies run on two copy streams beside the layer's
    # stream with double-buffered device inputs and outputs: step i+1's inputs
    # arrive while step i computes, and step i's output leaves while step i+1
    # computes (events order each buffer's reuse).
    srcs = [g["xq"], g["xs"], g["idx"], g["tw"]]
    sizes = [t.numel() * t.element_size() for t in srcs]
    offs, o = [], 0
    for n in sizes:
        offs.append(o)
        o += (n + 255) // 256 * 256
    h_in = torch.empty(o, dtype=torch.uint8).pin_memory()
    d_in = [torch.empty(o, dtype=torch.uint8, device=device) for _ in range(2)]

    def section(buf, i):
        t = srcs[i]
        return buf[offs[i]:offs[i] + sizes[i]].view(t.dtype).view(t.shape)

    for i, t in enumerate(srcs):
        section(h_in, i).copy_(t.cpu())
    views = [[section(d_in[b], i) for i in range(4)] for b in range(2)]
    outs = [out, torch.empty_like(out)]
    h_out = [torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = o  # the staging buffer, padding included
    d2h = h_out[0].numel() * h_out[0].element_size()
    s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]   # the layer finished with buffer b
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output of buffer b on the host

    def issue_h2d(b):
        s_h2d.wait_event(ev_done[b])  # the layer two steps back has read this buffer
        with torch.cuda.stream(s_h2d):
            d_in[b].copy_(h_in, non_blocking=True)
        ev_in[b].record(s_h2d)

    def e2e_steps(n):
        for b in range(2):
            ev_done[b].record(stream)
            ev_out[b].record(s_d2h)
        s_h2d.wait_stream(stream)
        issue_h2d(0)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                issue_h2d(b ^ 1)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # the host copy of this buffer's last output is done
            layer(*views[b], out=outs[b], stream=stream)
            ev_done[b].record(stream)
            s_d2h.wait_event(ev_done[b])
            with torch.cuda.stream(s_d2h):
                h_out[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_d2h)
        stream.wait_stream(s_d2h)

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps(args.warmup)
    barrier()
    start.record(stream)
    e2e_steps(args.steps)
    stop.record(stream)
    barrier()
    e2e_ms = max_over_ranks(start.elapsed_time(stop) / args.steps, device)
    st = moe.check_device_error(layer.workspace)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {moe.STATUS.get(st, st)}")

    if rank != 0:
        return
    f = layer_figures(args, w, r, world)
    line = {
        "metric": METRIC, "value": f["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": f["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "data": "synthetic",
        "dtype": "fp8xfp4 (fp32 accumulate)" if args.format == "mx" else "nvfp4 e2m1xe2m1 (fp32 accumulate)",
        "config": workload_config(w, args, world, f["touched"], f["b12"]),
        **{k: f[k] for k in ("us_per_layer", "effective_GBps", "hbm_frac_layer", "touched_experts", "stage_us",
                             "stage_timing", "roofline", "layer_frac_of_tensor_peak", "layer_frac_of_hbm_spec")},
        "e2e": {"value": world * w.flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": f["gpu_launches"],
        "clocks": f["clocks"],
    }
    if not args.no_cpu_baseline:
        s = oracle_sample(w, args.cpu_tokens, device, args.format)
        cflops, times, threads = time_oracle(w, s, 1)
        line["cpu_baseline"] = {"value": cflops / times[0] / 1e12, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "seconds": times[0],
                                "sample": f"first {len(s['tokens'])} of {w.T} tokens, all {w.k} experts each"}
    # The other workloads of the table, measured in the same run (one GPU
    # only): the same K timed calls after W warm-up calls each, with their own
    # clocks.  No end-to-end pass and no oracle timing for these (the
    # headline workload above carries both).
    extra = [int(x) for x in args.also.split(",") if x.strip()] if args.also else []
    if world == 1 and extra and not (args.experts or args.tokens):
        del r, g, layer, out, outs, h_in, d_in, h_out, views
        torch.cuda.empty_cache()
        line["workloads"] = {}
        for wid in extra:
            wx = W.WORKLOADS[wid]
            rx = time_layer(args, wx, device, world)
            fx = layer_figures(args, wx, rx, world)
            line["workloads"][wx.name] = {
                "config": workload_config(wx, args, world, fx["touched"], fx["b12"]),
                "tflops": fx["value"], "us_per_layer": fx["us_per_layer"],
                **{k: fx[k] for k in ("effective_GBps", "hbm_frac_layer", "touched_experts", "stage_us",
                                      "roofline", "layer_frac_of_tensor_peak", "gpu_launches", "clocks")},
                "not_measured_here": "e2e and the oracle's cpu_baseline (headline workload only)",
            }
            del rx
            torch.cuda.empty_cache()
        line["gpu_launches"] += sum(v["gpu_launches"] for v in line["workloads"].values())
        line["gpu_launches_note"] = "headline timed region plus the timed regions of `workloads`"
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if args.impl == "b200" else "gloo",
                                             timeout=datetime.timedelta(seconds=120))
    if args.also is None:
        args.also = "2,3,4" if args.workload == 1 and not (args.experts or args.tokens) and \
            args.format == "mx" and args.layout == "packets" else ""
    w = W.WORKLOADS[args.workload]
    if args.experts or args.tokens:
        E, T = args.experts or w.E, args.tokens or w.T
        w = W.custom(f"{w.name}_T{T}_E{E}", T=T, E=E, k=w.k, H=w.H, I=w.I, seed=w.seed,
                     routing=w.routing, zipf_s=w.zipf_s)
    try:
        if args.fp8_peak:
            run_fp8_peak(args)
        elif args.ep and args.impl == "b200":
            run_ep(args, w, rank, world, local_rank)
        elif args.shared_expert and args.impl == "reference":
            run_shared_reference(args, rank)
        elif args.shared_expert:
            run_shared(args, rank, world, local_rank)
        elif args.impl == "reference":
            run_reference(args, w, rank, world)
        else:
            run_b200(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
