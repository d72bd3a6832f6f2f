"""Benchmark of MXAttention's MXFP4 PNQ forward attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 720p] [--impl ours|reference]

One step = the whole hot path on one synthetic batch: Hadamard rotation +
MXFP4 quantization of Q and K, MXFP4 quantization of V along keys, and the
fused online-softmax attention with PNQ (three kernel launches).  The metric
is attention TFLOPS = 4 * B * H * N^2 * d / step time, on the 720p
video-DiT-shaped workload (B1 H40 N75600 d128, bf16) by default.

* ``value``: device time of K steps (CUDA events on the launching stream,
  inputs resident in HBM; the 2.3 GB of inputs exceed the 126 MB L2, so no
  flush is needed), max over ranks.
* ``e2e``: the same metric through the public host-buffer call
  ``mxattn_forward_host`` on pinned host buffers: the host->device copies of
  Q, K, V and the device->host copy of O are inside the timed region,
  pipelined by chunks of heads against the kernels.
* ``roofline``: the attention kernel alone (events around its launch inside
  the timed steps) against the dense FP4 tensor peak.
* ``cpu_baseline``: the CPU oracle timed on a bounded sample of the workload.

Multi-GPU (torchrun): the path partitions into independent attention
problems; every rank runs its own batch element (weak scaling), with no
collective on the data path; the host only reduces the timings.

``--impl reference`` times the CPU oracle alone on a bounded sample of the
same workload (the reference arm of this repository).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXFP4 PNQ attention TFLOPS at N=75.6k,H=40,d=128; % of B200 FP4 tensor peak"
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="720p")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-probe", action="store_true",
                    help="skip the dense FP4 MMA probe (the same-run peak beside the roofline's)")
    ap.add_argument("--format", default="mxfp4", choices=["mxfp4", "nvfp4"],
                    help="element format: the method's MXFP4, or the NVFP4 comparison format")
    ap.add_argument("--key-tile", type=int, default=128, choices=[64, 128],
                    help="keys per online-softmax step (the attention kernel's key tile)")
    ap.add_argument("--causal", action="store_true",
                    help="causal self-attention; TFLOPS count the visible (query, key) pairs, N(N+1)/2 per head")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 6650.0, "fallback"


def kernel_name(key_tile: int) -> str:
    return "mxattn_fwd_wide_kernel" if key_tile == 128 else "mxattn_fwd_kernel"


def kernel_source_hash(key_tile: int = 128) -> str:
    """Hash of the sources of the attention kernel for the key tile (and of the shared headers)."""
    h = hashlib.sha256()
    for name in ("attn_wide.cu" if key_tile == 128 else "attn.cu", "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "mxfp4_bit_attention_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, key_tile: int = 128):
    """DRAM bytes per attention launch from the committed ncu summary of the kernel for the key
    tile, if it was taken on that kernel's current source (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    rec = rec.get(kernel_name(key_tile), {})
    if rec.get("kernel_source_hash") != kernel_source_hash(key_tile):
        return None
    per = rec.get("per_workload", {}).get(workload)
    return None if per is None else float(per)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus: int):
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import datetime

    import torch
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return rank, world, dist


def reduce_max(x: float, dist, device: str = "cuda") -> float:
    """Max of a per-rank timing over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Batch element `rank` of a B = world batch: the workload's shape with its own seeded inputs.
    The ranks' problems are independent, so no data moves between GPUs."""
    from mxfp4_bit_attention_b200 import inputs
    return inputs.Workload(w.name, 1, w.H, w.N, w.d, w.dtype, w.seed + 1000 * rank)


def attention_flops(w, causal: bool) -> float:
    """The two contractions of one problem: 4 d flops per visible (query, key) pair, N^2 pairs per
    head, or N(N+1)/2 under causal masking."""
    pairs = w.N * (w.N + 1) / 2 if causal else float(w.N) * w.N
    return 4.0 * w.B * w.H * pairs * w.d


def whole_job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Throughput of the whole job: every rank's flops over the slowest rank's step time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def barrier(dist):
    import torch
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()


# ------------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ------------------------------------------------------------------------------------------------
def cpu_oracle_sample(w, target_seconds: float, causal: bool = False):
    """Time the oracle on one head's rotation/quantization plus attention for as many
    query rows as fit the time budget.  Returns (tflops, seconds, description, cores)."""
    import oracle
    from mxfp4_bit_attention_b200 import inputs
    g = inputs.generate(w, heads=[0])
    q, k, v = (inputs.as_fp32(g[n], w.dtype)[0] for n in "qkv")
    cores = oracle.num_threads()
    s = float(np.float32(w.d ** -0.5))
    t0 = time.perf_counter()
    _, kd, vd = oracle.prepare_head(q[:1], k, v)
    prep = time.perf_counter() - t0
    # calibrate on one row per oracle thread, then run the bounded sample
    probe = np.arange(cores, dtype=np.int64) * max(1, w.N // cores)
    t1 = time.perf_counter()
    qd, _, _ = oracle.prepare_head(q[probe], k[:32], v[:32])
    oracle.attention_rows(qd, kd, vd, s, w.key_tile, tau=8.0)
    per_row = max(time.perf_counter() - t1, 1e-4) / len(probe)
    nrows = int(max(cores, min(w.N, (target_seconds - prep) / per_row)))
    sel = np.linspace(0, w.N - 1, nrows).astype(np.int64)
    t2 = time.perf_counter()
    qd, _, _ = oracle.prepare_head(q[sel], k[:32], v[:32])
    oracle.attention_rows(qd, kd, vd, s, w.key_tile, tau=8.0, qpos=sel if causal else None)
    att = time.perf_counter() - t2
    # work: Q/K/V quantization of one head is not attention flops; the metric counts the
    # attention contractions of the sampled rows, timed together with one head's operand prep
    keys = float(np.sum(np.minimum(sel + 1, w.N))) if causal else float(nrows) * w.N
    flops = 4.0 * keys * w.d
    total = prep + att
    desc = (f"head 0 of {w.name}: rotation+MXFP4 of K and V ({w.N}x{w.d}) and PNQ attention for {nrows} of "
            f"{w.N} query rows{' (causal)' if causal else ''}; TFLOPS = 4*(visible query-key pairs)*d / "
            f"(prep + attention time)")
    return flops / total / 1e12, total, desc, cores


def relaunch_ranks(n_gpus: int) -> int:
    """`bench.py --gpus N` started without torchrun: start N ranks of this same command under
    torch.distributed.run on this node (127.0.0.1, a free port) and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd).returncode


# ------------------------------------------------------------------------------------------------
def main():
    args = parse()
    if args.gpus > 1 and "RANK" not in os.environ:
        sys.exit(relaunch_ranks(args.gpus))
    from mxfp4_bit_attention_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    bf16_peak, hbm_peak, peak_kind = peaks()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        times = []
        val = None
        desc = cores = None
        for _ in range(args.warmup + args.steps):
            val, t, desc, cores = cpu_oracle_sample(w, max(1.0, args.cpu_sample_seconds / max(1, args.steps)),
                                                    args.causal)
            times.append(t)
        times = times[args.warmup:]
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS",
                "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)),
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                                                "input_dtype": w.dtype, "causal": args.causal},
                "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc},
                "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    from mxfp4_bit_attention_b200 import binding
    rank, world, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load()

    # inputs: batch element `rank` of a B = world batch (independent problems)
    g = inputs.generate(rank_workload(w, rank))
    shape = (1, w.H, w.N, w.d)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host_tensor(a):
        t = torch.from_numpy(a)
        if w.dtype == "bf16":
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.reshape(shape).pin_memory()

    hq, hk, hv = (host_tensor(g[n]) for n in "qkv")
    del g
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    if args.format == "nvfp4":
        args.key_tile = 64  # the NVFP4 comparison format runs with 64-key tiles
    opts = binding.Opts(causal=args.causal, key_tile=args.key_tile,
                        format=binding.FMT_NVFP4 if args.format == "nvfp4" else binding.FMT_MXFP4)
    scale = float(np.float32(w.d ** -0.5))
    ws = binding.new_workspace(1, w.H, w.N, w.d, opts, dev)
    out = torch.empty(shape, dtype=tdt, device=dev)
    sizes = binding.operand_sizes(1, w.H, w.N, w.d, opts.format)
    # the packed operands live inside the workspace; carve the same views for the split calls
    ops = {}
    off = 256
    for key in ("q_codes", "q_scales", "k_codes", "k_scales", "v_codes", "v_scales"):
        ops[key] = ws[off:off + sizes[key]]
        off = (off + sizes[key] + 255) // 256 * 256
    stream = torch.cuda.current_stream()

    def step(ev_mid=None, ev_att_end=None):
        binding.mxattn_hadamard_quant_qk(q, k, opts, out=ops)
        binding.mxattn_quant_v(v, opts, out=ops)
        if ev_mid is not None:
            ev_mid.record(stream)
        binding.mxattn_attention_mxfp4(ops, 1, w.H, w.N, w.d, scale, out, opts, workspace=ws)
        if ev_att_end is not None:
            ev_att_end.record(stream)

    for _ in range(args.warmup):
        step()
    barrier(dist)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with Clocks(dev.index) as clk:
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step(mids[i], ends[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    total_ms = t_begin.elapsed_time(t_end)
    attn_ms = statistics.mean(m.elapsed_time(e) for m, e in zip(mids, ends))
    quant_ms = statistics.mean(s.elapsed_time(m) for s, m in zip(starts, mids))
    status = binding.mxattn_get_device_error(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")
    total_ms = reduce_max(total_ms, dist)
    attn_ms_max = reduce_max(attn_ms, dist)
    ms_per_step = total_ms / args.steps
    flops = attention_flops(w, args.causal)  # per rank (B = 1 per rank)
    value = whole_job_tflops(world, flops, ms_per_step)
    clocks = clk.summary()

    # e2e through the public host-buffer entry point (mxattn_forward_host): every step copies Q, K, V
    # from pinned host memory and O back, pipelined by chunks of heads against the kernels
    e2e = None
    if not args.no_e2e:
        hout = torch.empty(shape, dtype=tdt).pin_memory()
        host_bytes = binding.load().mxattn_workspace_bytes_host(
            1, w.H, w.N, w.d, ctypes.byref(binding._copts(opts, binding._dtype_code(q))))
        ws_host = torch.zeros(host_bytes, dtype=torch.uint8, device=dev)
        for _ in range(max(1, args.warmup)):
            binding.mxattn_forward_host(hq, hk, hv, scale, opts, out=hout, workspace=ws_host)
        barrier(dist)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            binding.mxattn_forward_host(hq, hk, hv, scale, opts, out=hout, workspace=ws_host)
        e1.record(stream)
        torch.cuda.synchronize()
        if binding.mxattn_get_device_error(ws_host) != 0:
            raise RuntimeError("device status set during the end-to-end steps")
        e2e_ms = reduce_max(e0.elapsed_time(e1), dist) / args.steps
        in_bytes = 3 * q.numel() * q.element_size()
        e2e = {"value": whole_job_tflops(world, flops, e2e_ms), "unit": "TFLOPS", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out.numel() * out.element_size(),
               "call": "mxattn_forward_host"}
        del ws_host

    # The dense FP4 tensor-core peak measured on this GPU in this run (mxattn_fp4_mma_probe: one CTA
    # per SM issuing back-to-back M128 x N256 x K64 kind::mxf4 MMAs), after the timed regions.
    probe_tflops = None
    if not args.no_probe:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        iters, n = 100000, 256
        binding.mxattn_fp4_mma_probe(sms, 2000, n, stream)
        times = []
        for _ in range(3):
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(stream)
            binding.mxattn_fp4_mma_probe(sms, iters, n, stream)
            p1.record(stream)
            torch.cuda.synchronize()
            times.append(p0.elapsed_time(p1))
        probe_tflops = sms * iters * 2 * 128 * n * 64 / (sorted(times)[1] * 1e-3) / 1e12

    fp4_peak = bf16_peak * FP4_PER_BF16
    achieved = flops / (attn_ms_max * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak,
                # the recorded DRAM bytes are those of the full-attention MXFP4 kernel
                "traffic": recorded_traffic(w.name, args.key_tile) if (args.format == "mxfp4" and not args.causal)
                else None,
                "kernel": kernel_name(args.key_tile), "ms_per_launch": attn_ms_max,
                "peak_source": f"{peak_kind} bf16 {bf16_peak:.1f} TFLOP/s x nominal FP4/BF16 ratio {FP4_PER_BF16:g}",
                "frac_of_spec_9pf": achieved / 9000.0,
                "probe_fp4_tflops": probe_tflops,
                "frac_of_probe": None if probe_tflops is None else achieved / probe_tflops,
                "quantizers_ms": quant_ms,
                "quantizers_hbm_gbs": (3 * q.numel() * (q.element_size() + 0.5 + 1 / 32)) / (quant_ms * 1e-3) / 1e9}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, t, desc, cores = cpu_oracle_sample(w, args.cpu_sample_seconds, args.causal)
        cpu = {"value": val, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc, "seconds": t}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "fp4(e2m1)+fp32 accumulate, bf16 in/out", "data": "synthetic",
                "config": {"workload": w.name, "B": world, "H": w.H, "N": w.N, "d": w.d, "input_dtype": w.dtype,
                           "key_tile": args.key_tile, "pnq": True, "rotate": True, "causal": args.causal,
                           "format": args.format,
                           "scale_rule": "UOS Qmax=7.25" if args.format == "mxfp4" else "E4M3(amax/6) per 16",
                           "rescale_tau": opts.rescale_tau, "parallelism": f"independent problems x{world}",
                           "l2": "inputs (2.3 GB) larger than L2 (126 MB); no flush"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": 3 * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
