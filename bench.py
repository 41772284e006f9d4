#!/usr/bin/env python
"""Parallax decode benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen|large|long|ragged|tiny]
    python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm
    python bench.py --prefill [--prefill-shape B,Hq,Hkv,L,D]   # the causal training-shape forward
    python bench.py --kv-mode paged|block_sparse --workload large   # paged / block-sparse decode

A step is one Parallax decode pass (split-KV kernel + merge kernel) over one
batch of synthetic input resident in HBM. The headline value is KV-read
bandwidth (algorithmic K and V bytes of the valid keys per step / step time),
reported next to microseconds per step and the in-run R = 0 softmax decode on
the same pipeline and buffers. Multi-GPU runs are independent replicas (the
decode has no cross-GPU exchange), one process per GPU under torchrun.

Timing: CUDA events on the launching stream after W untimed steps, barrier +
synchronize on both sides, max over ranks. Workloads smaller than the L2
rotate over enough K/V copies to exceed twice the L2, so every step reads HBM.
Small workloads are replayed from CUDA graphs (the pages' bench replays
graphs too: parallax-kernel 0.1.0 README, "Benchmark").
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from parameterized_local_linear_b200 import inputs, replicas  # noqa: E402

METRIC = "decode µs/step and KV-read GB/s (% of HBM peak) vs in-run R=0 softmax decode"
PREFILL_METRIC = "prefill forward TFLOP/s (algorithmic, causal) vs in-run softmax attention"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# Qwen-3-0.6B attention heads (16 query, 8 kv, D = 128) at a 4096-token context
PREFILL_DEFAULT_SHAPE = "4,16,8,4096,128"
DEFAULT_STEPS = {"tiny": 20000, "qwen": 100000, "large": 200, "long": 200, "ragged": 200}
DEFAULT_WARMUP = {"tiny": 2000, "qwen": 5000, "large": 5, "long": 5, "ragged": 5}
# the sources that decide what each decode kernel does (hashed against its ncu summary)
_CSRC = os.path.join(ROOT, "parameterized_local_linear_b200", "csrc")
KERNEL_SRCS = {
    "tc": [os.path.join(_CSRC, f) for f in ("kernel_tc.cuh", "partition.cuh", "common.cuh",
                                            "ptx.cuh")],
    "cluster": [os.path.join(_CSRC, f) for f in ("kernel_cluster.cuh", "kernel_tc.cuh",
                                                 "common.cuh", "ptx.cuh")],
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", "--config", choices=sorted(inputs.WORKLOADS), default="large")
    ap.add_argument("--num-splits", "--splits", type=int, default=0)
    ap.add_argument("--out-dtype", choices=["bf16", "f32"], default="bf16",
                    help="decode output: bf16, or the fp32 debug output")
    ap.add_argument("--seed", type=int, default=None, help="override the workload's seed")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (for profiling a smaller copy)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="bound of the CPU oracle baseline sample (seconds)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-companion", action="store_true",
                    help="skip the Qwen B=1 step measured beside a larger workload")
    ap.add_argument("--kv-mode", choices=["contiguous", "paged", "block_sparse"],
                    default="contiguous", help="where the decode reads its keys from")
    ap.add_argument("--page-size", type=int, default=256)
    ap.add_argument("--density", type=float, default=0.5,
                    help="block-sparse: fraction of each sequence's 64-key blocks attended")
    ap.add_argument("--prefill", action="store_true",
                    help="time the causal training-shape forward instead of the decode")
    ap.add_argument("--prefill-shape", default=PREFILL_DEFAULT_SHAPE,
                    help="B,Hq,Hkv,L,D of the prefill forward")
    ap.add_argument("--varlen", action="store_true",
                    help="prefill: B packed sequences of seeded lengths U{1..L} instead")
    a = ap.parse_args()
    if a.prefill:
        a.steps = a.steps if a.steps is not None else 50
        a.warmup = a.warmup if a.warmup is not None else 5
    a.steps = a.steps if a.steps is not None else DEFAULT_STEPS[a.workload]
    a.warmup = a.warmup if a.warmup is not None else DEFAULT_WARMUP[a.workload]
    return a


# ------------------------------------------------------------------ helpers --

def kv_bytes(x) -> int:
    """Algorithmic K+V bytes of one step: 2 tensors x valid keys x Hkv x D x itemsize."""
    n = int(x["seqlens"].to(torch.int64).clamp(0, x["k"].shape[2]).sum())
    _, Hkv, _, D = x["k"].shape
    return 2 * n * Hkv * D * x["k"].element_size()


def qro_bytes(x) -> int:
    """q and r reads plus the bf16 output write of one step."""
    return 3 * x["q"].numel() * x["q"].element_size()


def workload_desc(w: inputs.Workload) -> str:
    lens = {"full": f"L={w.Lmax}", "uniform": f"L~U[1,{w.Lmax}]"}.get(
        w.lengths if isinstance(w.lengths, str) else "", f"L={list(w.lengths)}")
    return (f"{w.name}: Parallax decode B={w.B} Hq={w.Hq} Hkv={w.Hkv} D={w.D} {lens} "
            f"Lmax={w.Lmax} {str(w.dtype).replace('torch.', '')} seed={w.seed}")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    """Dense bf16 tensor peak: the burst figure (a kernel timed on its own)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def measured_bf16_sustained():
    """Dense bf16 tensor peak held for seconds under the power cap, or None."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return None


# ncu summaries whose traffic line the bench reports, per (workload, kernel):
# (file, batch rows the capture ran). A capture on fewer rows than the
# workload is scaled by the rows processed (every row of these workloads has
# the same length, so the kernel's traffic grows in proportion).
PROFILE_FOR = {("qwen", "cluster"): ("parallax_cluster_kernel_qwen.md", 1),
               ("large", "tc"): ("parallax_tc_kernel_large_B64.md", 64)}


def source_hash(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SRCS[kernel]:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(w, kernel):
    """Per-launch DRAM traffic (read + write) of the workload's dominant
    kernel from its committed ncu summary, if that was taken on the current
    kernel source; scaled to the workload's batch when captured on fewer
    rows. None otherwise."""
    name = w.name.split("-")[0]
    if (name, kernel) not in PROFILE_FOR or w.name != name:
        return None
    fname, rows = PROFILE_FOR[(name, kernel)]
    try:
        text = open(os.path.join(ROOT, "profiles", fname)).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_traffic = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not m_hash or not m_traffic or m_hash.group(1) != source_hash(kernel):
        return None
    return int(m_traffic.group(1)) * w.B // rows


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while the
    timed region runs (reads only; changes no setting)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.period, self._stop = [], period_s, threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if str(uuid) in u:
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "err", "nvml unavailable")}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = sorted(v for k, v in self.REASONS.items() if bits & k)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


class Dist:
    def __init__(self, gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if gpus != self.world:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={self.world}: launch N>1 with torchrun")
        self.pg = None

    def init_gpu(self):
        torch.cuda.set_device(self.local)
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local))
            self.pg = dist

    def barrier(self):
        replicas.barrier()

    def max(self, x: float) -> float:
        return replicas.max_over_ranks(x)

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------ CPU oracle ----

def oracle_rows_for_budget(w: inputs.Workload, x_host: dict, budget_s: float):
    """Batch rows whose single oracle pass takes about budget_s (at least one)."""
    import oracle
    idx = torch.tensor([0])
    t0 = time.perf_counter()
    oracle.parallax_decode(x_host["q"][idx], x_host["r"][idx], x_host["k"][idx],
                           x_host["v"][idx], x_host["seqlens"][idx], x_host["scale"])
    one = max(1e-4, time.perf_counter() - t0)
    return list(range(max(1, min(w.B, int(budget_s / one)))))


def oracle_timed(w: inputs.Workload, x_host: dict, rows, steps: int):
    """Time `steps` passes of the fp64 oracle, as it stands, over batch rows
    `rows`. Returns (GB/s of K/V processed, threads, seconds)."""
    import oracle
    idx = torch.tensor(rows)
    sub = {k: (x_host[k][idx] if torch.is_tensor(x_host[k]) else x_host[k])
           for k in ("q", "r", "k", "v", "seqlens")}
    n = sub["seqlens"].to(torch.int64).clamp(0, w.Lmax).sum().item()
    kv = 2 * n * w.Hkv * w.D * x_host["k"].element_size()
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.parallax_decode(sub["q"], sub["r"], sub["k"], sub["v"], sub["seqlens"],
                               x_host["scale"])
    secs = time.perf_counter() - t0
    return kv * steps / secs / 1e9, oracle.num_threads(), secs


def oracle_sample(w: inputs.Workload, x_host: dict, budget_s: float):
    """The CPU baseline: the oracle on a bounded sample of the workload, about
    budget_s of CPU work. Returns (GB/s, threads, description, seconds)."""
    rows = oracle_rows_for_budget(w, x_host, budget_s / 4)
    _, _, t1 = oracle_timed(w, x_host, rows, 1)
    passes = max(1, int(budget_s / max(t1, 1e-6)))
    v, cores, secs = oracle_timed(w, x_host, rows, passes)
    desc = (f"fp64 oracle (covariance form), {passes} passes over batch rows 0..{rows[-1]} "
            f"({len(rows)} of {w.B}); {secs:.1f} s")
    return v, cores, desc, secs


def host_inputs_for_oracle(w: inputs.Workload, budget_rows: int = 64):
    """The workload's seeded inputs on the host, limited to the first rows the
    oracle can take (large workloads are drawn on the GPU and copied back)."""
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = inputs.make_inputs(w, device=dev, pad_value=None)
    rows = min(w.B, budget_rows)
    out = {k: (v[:rows].cpu() if torch.is_tensor(v) else v) for k, v in x.items()}
    del x
    if dev == "cuda":
        torch.cuda.empty_cache()
    wsub = inputs.Workload(w.name, rows, w.Hq, w.Hkv, w.D, w.Lmax, w.dtype, w.seed, "full",
                           w.r_scale, w.k_offset_std, w.scale)
    return wsub, out


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores. A step is one
    oracle pass over a bounded sample of the workload's batch rows (sized so
    that the whole run takes a few minutes); exactly K steps are timed."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = inputs.WORKLOADS[args.workload]
    wsub, xh = host_inputs_for_oracle(w)
    per_step = min(5.0, 120.0 / max(1, args.steps + args.warmup))
    rows = oracle_rows_for_budget(wsub, xh, per_step)
    if args.warmup:
        oracle_timed(wsub, xh, rows, args.warmup)
    value, cores, secs = oracle_timed(wsub, xh, rows, args.steps)
    desc = (f"fp64 oracle (covariance form); a step = one pass over batch rows 0..{rows[-1]} "
            f"({len(rows)} of {w.B}) of the workload")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / max(1, args.steps) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "parallelism": "rank 0 only (host CPU)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------- prefill forward ----

def prefill_flops(B, Hq, L, D, causal=True):
    """Algorithmic flops of the forward: q.k, r.k, e.v and (e s).v, 2 D flops
    each per (query head, row, attended key)."""
    pairs = L * (L + 1) // 2 if causal else L * L
    return 8 * D * B * Hq * pairs


def prefill_inputs(B, Hq, Hkv, L, D, device, seed=7):
    """The pages' quickstart recipe for the training shape: q, r, k, v all
    bf16 N(0, 1) (parallax-kernel 0.1.0 README, "Training (Triton)")."""
    g = torch.Generator(device=device).manual_seed(seed)
    mk = lambda H: torch.randn(B, H, L, D, device=device, dtype=torch.bfloat16, generator=g)
    return mk(Hq), mk(Hq), mk(Hkv), mk(Hkv)


def prefill_oracle_sample(shape, budget_s):
    """The fp64 oracle on the first query heads of batch row 0 (full length),
    as many as fit in about budget_s. Returns (TFLOP/s, threads, description)."""
    import oracle
    B, Hq, Hkv, L, D = shape
    G = Hq // Hkv
    q, r, k, v = prefill_inputs(1, G, 1, L, D, "cpu")
    t0 = time.perf_counter()
    oracle.parallax_prefill(q[:, :1], r[:, :1], k, v, D ** -0.5, True)
    one = max(1e-4, time.perf_counter() - t0)
    heads = max(1, min(G, int(budget_s / one)))
    reps = max(1, int(budget_s / (one * heads)))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.parallax_prefill(q[:, :heads], r[:, :heads], k, v, D ** -0.5, True)
    secs = time.perf_counter() - t0
    tf = prefill_flops(1, heads, L, D) * reps / secs / 1e12
    desc = (f"fp64 oracle prefill, {reps} passes over {heads} query head(s) of one batch row "
            f"at L={L}, D={D}; {secs:.1f} s")
    return tf, oracle.num_threads(), desc, secs


def run_prefill(args):
    """Causal training-shape forward: one step is one parallax_prefill launch
    over the whole [B, H, L, D] problem, inputs resident in HBM."""
    shape = tuple(int(t) for t in args.prefill_shape.split(","))
    B, Hq, Hkv, L, D = shape
    flops = prefill_flops(B, Hq, L, D)
    cfg = {"workload": f"prefill: Parallax causal forward B={B} Hq={Hq} Hkv={Hkv} L={L} D={D} "
                       f"bf16 N(0,1)", "global_batch": B, "seq_len": L}
    lens = None
    if args.varlen:
        g = torch.Generator().manual_seed(11)
        lens = torch.randint(1, L + 1, (B,), generator=g).tolist()
        flops = sum(8 * D * Hq * n * (n + 1) // 2 for n in lens)
        cfg["workload"] = (f"varlen prefill: {B} packed sequences, lengths U{{1..{L}}} seeded "
                           f"({sum(lens)} tokens), Hq={Hq} Hkv={Hkv} D={D} bf16 N(0,1)")
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        tf, cores, desc, secs = prefill_oracle_sample(shape, min(10.0, args.cpu_seconds))
        line = {"impl": "reference", "metric": PREFILL_METRIC, "value": tf, "unit": "TFLOP/s",
                "n_gpus": args.gpus, "steps": 1, "warmup": 0, "ms_per_step": secs * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    from parameterized_local_linear_b200 import binding
    dist = Dist(args.gpus)
    dist.init_gpu()
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load_library()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    if lens is None:
        q, r, k, v = prefill_inputs(B, Hq, Hkv, L, D, dev)
    else:  # the same draws, packed: [total, H, D]
        total = sum(lens)
        q, r, k, v = (t[0].transpose(0, 1).contiguous() for t in
                      prefill_inputs(1, Hq, Hkv, total, D, dev))
        cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32,
                          device=dev)
    out = torch.empty_like(q)
    out_f32 = out.dtype == torch.float32
    # room for the fp16 copy of V (the fp16 value products of the bf16 output)
    ws = (binding.prefill_workspace(B, L, Hkv, D, dev) if lens is None
          else binding.prefill_workspace(1, sum(lens), Hkv, D, dev))
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    in_bytes = sum(t.numel() * t.element_size() for t in (q, r, k, v, out))
    # inputs smaller than the L2: rotate over enough copies to exceed twice the L2
    nbuf = max(1, math.ceil(2 * l2 / in_bytes)) if in_bytes < 2 * l2 else 1
    sets = [(q, r, k, v)] + [tuple(t.clone() for t in (q, r, k, v)) for _ in range(nbuf - 1)]

    def call(j=0):
        qq, rr, kk, vv = sets[j % nbuf]
        if lens is None:
            binding.parallax_prefill(qq, rr, kk, vv, out=out, workspace=ws, stream=stream)
        else:
            binding.parallax_varlen_prefill(qq, rr, kk, vv, cu, max(lens), out=out, workspace=ws,
                                            stream=stream)

    def run(k_steps, events=None):
        for i in range(k_steps):
            if events:
                events[i][0].record(stream)
            call(i)
            if events:
                events[i][1].record(stream)

    def timed(fn, k_steps, w_steps, sampler=None):
        return timed_steps(dist, stream, fn, k_steps, w_steps, sampler)

    sampler = ClockSampler(dev.index)
    t_step = timed(run, args.steps, args.warmup, sampler)
    # per-launch kernel duration (events around each launch)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    run(args.steps, evs)
    torch.cuda.synchronize()
    kern_s = statistics.median(a.elapsed_time(b) for a, b in evs) / 1e3
    st = int(ws[:4].view(torch.int32).item())
    if st != 0:
        raise SystemExit(f"device status after timing: {st:#x}")

    # in-run softmax-only attention on the same q, k, v (torch SDPA, causal,
    # grouped heads): context for the tensor-core efficiency, not the target
    sdpa = None
    try:
        if lens is not None:
            raise RuntimeError("no packed-sequence SDPA in torch; see the dense line")

        def run_sdpa(k_steps):
            for i in range(k_steps):
                qq, _, kk, vv = sets[i % nbuf]
                torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True,
                                                                 enable_gqa=Hq != Hkv)
        t_sdpa = timed(run_sdpa, args.steps, args.warmup)
        sdpa = {"us_per_step": t_sdpa / args.steps * 1e6,
                "tflops": flops / 2 * args.steps / t_sdpa / 1e12,
                "note": "torch scaled_dot_product_attention, causal: 4 D flops per pair"}
    except Exception as exc:  # an SDPA backend may not take this shape
        sdpa = {"unavailable": str(exc).splitlines()[0][:200]}

    # end to end through the public API: inputs from pinned host memory each step
    hq, hr, hk, hv = (t.cpu().pin_memory() for t in (q, r, k, v))
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def run_e2e(k_steps):
        for _ in range(k_steps):
            for dst, src in ((q, hq), (r, hr), (k, hk), (v, hv)):
                dst.copy_(src, non_blocking=True)
            call()
            out_host.copy_(out, non_blocking=True)

    k_e2e = min(args.steps, 20)
    t_e2e = timed_plain(dist, stream, run_e2e, k_e2e, 2)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hr, hk, hv))
    d2h = out_host.numel() * out_host.element_size()

    # accuracy of this launch configuration against the fp64 oracle on one
    # sampled slice: the last (batch row, query head) of the dense problem, or
    # the last packed sequence
    accuracy = None
    if dist.rank == 0:
        import numpy as np
        import oracle
        call(0)
        torch.cuda.synchronize()
        if lens is None:
            hh, gg = Hq - 1, (Hq - 1) // (Hq // Hkv)
            sl = lambda t, i: t[B - 1:B, i:i + 1].cpu()
            want = oracle.parallax_prefill(sl(q, hh), sl(r, hh), sl(k, gg), sl(v, gg), D ** -0.5,
                                           True)
            got = out[B - 1:B, hh:hh + 1].float().cpu().double().numpy()
            sample = f"batch row {B - 1}, query head {hh}, all {L} rows"
        else:
            a0 = int(cu[-2])
            seg = lambda t: t[a0:].cpu()
            want = oracle.parallax_varlen_prefill(seg(q), seg(r), seg(k), seg(v),
                                                  [0, sum(lens) - a0], D ** -0.5, True)
            got = out[a0:].float().cpu().double().numpy()
            sample = f"the last sequence ({sum(lens) - a0} rows), all heads"
        err = float(np.max(np.abs(got - want) / np.maximum(1.0, np.abs(want))))
        accuracy = {"max_scaled_err": err, "tolerance": 1e-4 if out_f32 else 2e-2,
                    "pass": bool(np.isfinite(got).all() and err <= (1e-4 if out_f32 else 2e-2)),
                    "oracle": "fp64", "sample": sample}

    # sustained: whole calls back to back for at least one second (the power
    # cap and the clocks it settles at), one gated region; last, so that it
    # heats the GPU after the other timings
    k_sus = max(args.steps, math.ceil(1.0 / (t_step / args.steps)))
    t0 = time.perf_counter()
    run(4)
    host_call = (time.perf_counter() - t0) / 4
    torch.cuda.synchronize()
    dist.barrier()
    sus_sampler = ClockSampler(dev.index)
    t_sus = dist.max(gated_region(stream, lambda: run(k_sus), host_call * k_sus, sus_sampler))
    torch.cuda.synchronize()
    dist.barrier()
    sus_clocks = sus_sampler.summary()

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        tf, cores, desc, _ = prefill_oracle_sample(shape, min(10.0, args.cpu_seconds))
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    peak, peak_src = measured_bf16_peak()
    sustained = measured_bf16_sustained()
    N = dist.world
    achieved = flops / kern_s / 1e12
    clocks = sampler.summary()
    line = {
        "metric": PREFILL_METRIC, "value": N * flops * args.steps / t_step / 1e12,
        "unit": "TFLOP/s", "n_gpus": N, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_step / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        # bf16 scores; bf16 output: value products on fp16 weights and V (the
        # exact bf16 hi + lo pair on tiles outside fp16's range)
        "vs_baseline": None, "dtype": "bf16+f16", "data": "synthetic",
        "config": dict(cfg, parallelism=f"replicas x{N}" if N > 1 else "single GPU",
                       l2=(f"rotate {nbuf} input copies ({nbuf * in_bytes / 1e6:.0f} MB > 2x L2)"
                           if nbuf > 1 else f"inputs ({in_bytes / 1e6:.0f} MB) larger than L2")),
        "softmax_sdpa": sdpa,
        "sustained": {"steps": k_sus, "seconds": t_sus, "us_per_step": t_sus / k_sus * 1e6,
                      "value": N * flops * k_sus / t_sus / 1e12, "unit": "TFLOP/s",
                      "frac_of_sustained_peak": (flops * k_sus / t_sus / 1e12 / sustained
                                                 if sustained else None),
                      "clocks": {k2: sus_clocks[k2] for k2 in ("sm_mhz", "sm_max_mhz", "reasons",
                                                               "samples")},
                      "method": "whole calls over at least one second, one gated region"},
        "accuracy": accuracy,
        "clocks": {k2: clocks[k2] for k2 in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
        "e2e": {"value": N * flops * k_e2e / t_e2e / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": t_e2e / k_e2e * 1e6},
        # per step: the fp16 copy of V, then the prefill kernel
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "frac_of_sustained": achieved / sustained if sustained else None,
                     "kernel": "parallax_prefill_kernel",
                     "kernel_us_covers": "the fp16 copy of V and the prefill kernel",
                     "peak_source": peak_src + " (burst)",
                     "kernel_us": kern_s * 1e6, "algorithmic_flops_per_launch": flops,
                     "tensor_flops_issued_per_launch": flops},
        "cpu_baseline": cpu,
    }
    if dist.rank == 0:
        print(json.dumps(line))
    dist.close()
    return 0


# -------------------------------------------------- paged / block-sparse ----

def run_kv_variant(args):
    """Decode steps over a paged cache or a block-sparse key selection. The
    value is the KV-read bandwidth of the keys actually attended; the R = 0
    path on the same inputs runs in alternating blocks beside it."""
    if args.impl == "reference":
        return run_kv_variant_reference(args)
    from parameterized_local_linear_b200 import binding
    dist = Dist(args.gpus)
    dist.init_gpu()
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load_library()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    w = inputs.WORKLOADS[args.workload]
    if args.batch is not None:
        w = inputs.Workload(w.name + f"-B{args.batch}", args.batch, w.Hq, w.Hkv, w.D, w.Lmax,
                            w.dtype, w.seed, w.lengths, w.r_scale, w.k_offset_std, w.scale)
    esz = 2
    if args.kv_mode == "paged":
        x = inputs.make_paged(w, args.page_size, dev)
        lens = x["seqlens"].to(torch.int64).clamp(0, w.Lmax)
        keys = int(lens.sum())
        plan_len = x["table"].shape[1] * args.page_size
        desc = f"paged: page_size {args.page_size}, pages scattered by a seeded permutation"
    else:
        x = inputs.make_block_sparse(w, args.density, dev)
        lens = x["seqlens"].to(torch.int64).clamp(0, w.Lmax).cpu()
        ids, cnt = x["block_ids"].cpu(), x["num_blocks"].cpu()
        keys = 0
        for b in range(w.B):
            blk = ids[b, :int(cnt[b])].to(torch.int64)
            keys += int((lens[b] - 64 * blk).clamp(0, 64).sum())
        plan_len = 64 * x["block_ids"].shape[1]
        desc = f"block-sparse: {args.density:.2f} of each sequence's 64-key blocks, seeded"
    step_kv = 2 * keys * w.Hkv * w.D * esz
    ws = binding.Workspace(w.B, w.Hq, w.Hkv, w.D, plan_len, args.num_splits, device=dev)
    out = torch.empty((w.B, w.Hq, w.D), device=dev, dtype=torch.bfloat16)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    pool_bytes = 2 * x["k"].numel() * esz
    # a pool smaller than the L2: rotate over enough copies of K and V to
    # exceed twice the L2, replayed from CUDA graphs (as the contiguous bench)
    nbuf = max(1, math.ceil(2 * l2 / pool_bytes)) if pool_bytes < 2 * l2 else 1
    kvs = [(x["k"], x["v"])] + [(x["k"].clone(), x["v"].clone()) for _ in range(nbuf - 1)]

    def step(probe, j=0):
        kk, vv = kvs[j % nbuf]
        if args.kv_mode == "paged":
            binding.parallax_decode_paged(x["q"], x["r"], kk, vv, x["table"],
                                          x["seqlens"], scale=x["scale"], out=out, workspace=ws,
                                          num_splits=args.num_splits, probe=probe, stream=stream)
        else:
            binding.parallax_decode_block_sparse(x["q"], x["r"], kk, vv, x["block_ids"],
                                                 x["num_blocks"], x["seqlens"], scale=x["scale"],
                                                 out=out, workspace=ws, num_splits=args.num_splits,
                                                 probe=probe, stream=stream)

    graphs = {}
    if nbuf > 1:
        for probe in (True, False):
            for j in range(nbuf):
                step(probe, j)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for j in range(nbuf):
                    step(probe, j)
            graphs[probe] = g

    def run(k_steps, probe=True):
        if nbuf > 1:
            for _ in range(max(1, k_steps // nbuf)):
                graphs[probe].replay()
            return
        for i in range(k_steps):
            step(probe, i)

    def timed(fn, k_steps, w_steps, sampler=None):
        return timed_steps(dist, stream, fn, k_steps, w_steps, sampler)

    if nbuf > 1:  # whole graph chains only
        args.steps = max(nbuf, args.steps // nbuf * nbuf)
    sampler = ClockSampler(dev.index)
    t = timed(run, args.steps, args.warmup, sampler)
    per = {True: [], False: []}
    blk = max(1, min(args.steps, 20)) if nbuf == 1 else nbuf * max(1, 800 // nbuf)
    for _ in range(5):
        for probe in (True, False):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run(blk, probe)
            b.record(stream)
            b.synchronize()
            per[probe].append(a.elapsed_time(b) / 1e3 / blk)
    t_p, t_s = dist.max(statistics.median(per[True])), dist.max(statistics.median(per[False]))
    rc, bits = ws.status()
    if rc != 0:
        raise SystemExit(f"device status after timing: {binding.parallax_status_string(rc)}")
    # end to end: q, r and lengths packed in one pinned host block copied in,
    # the output copied back, every step (small pools through parallax_copy,
    # large ones by DMA, as in the contiguous bench); the step reads device
    # views of the copied block
    names = ("q", "r", "seqlens")
    offs, nb = [], 0
    for k in names:
        offs.append(nb)
        nb += (x[k].numel() * x[k].element_size() + 255) // 256 * 256
    host_block = torch.zeros(nb, dtype=torch.uint8)
    dev_block = torch.zeros(nb, dtype=torch.uint8, device=dev)
    for k, o in zip(names, offs):
        n_ = x[k].numel() * x[k].element_size()
        host_block[o:o + n_].copy_(x[k].cpu().contiguous().view(-1).view(torch.uint8))
        x[k] = dev_block[o:o + n_].view(x[k].dtype).view(x[k].shape)
    host_block = host_block.pin_memory()
    dev_block.copy_(host_block)  # the views that now stand for q, r and the lengths hold them
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    k_e2e = min(args.steps, 50)

    def decode_with(xx, kk, vv, dst):
        if args.kv_mode == "paged":
            binding.parallax_decode_paged(xx["q"], xx["r"], kk, vv, xx["table"], xx["seqlens"],
                                          scale=xx["scale"], out=dst, workspace=ws,
                                          num_splits=args.num_splits, stream=stream)
        else:
            binding.parallax_decode_block_sparse(xx["q"], xx["r"], kk, vv, xx["block_ids"],
                                                 xx["num_blocks"], xx["seqlens"],
                                                 scale=xx["scale"], out=dst, workspace=ws,
                                                 num_splits=args.num_splits, stream=stream)

    if nbuf > 1:
        # small pools: per step its own input block and output buffer, the
        # input copy on a side stream ahead of the decode and the output copy
        # on another behind it (parallax_copy), replayed from a CUDA graph, as
        # in the contiguous bench
        transfer = ("parallax_copy (kernel over mapped pinned host memory) on two side streams, "
                    "each step's input and output copies overlapping its neighbours' decodes")
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        sets = []
        for _ in range(nbuf):
            blk = torch.zeros(nb, dtype=torch.uint8, device=dev)
            views = {k: blk[o:o + x[k].numel() * x[k].element_size()].view(x[k].dtype)
                     .view(x[k].shape) for k, o in zip(names, offs)}
            sets.append((blk, {**x, **views}, torch.empty_like(out),
                         torch.empty(out.shape, dtype=out.dtype).pin_memory()))
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_dec = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]

        def chain():
            fork = torch.cuda.Event()
            fork.record(stream)
            s_in.wait_event(fork)
            s_out.wait_event(fork)
            for i in range(nbuf):
                blk, xx, dout, hout = sets[i]
                binding.parallax_copy(blk, host_block, stream=s_in)
                ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                decode_with(xx, kvs[i][0], kvs[i][1], dout)
                ev_dec[i].record(stream)
                s_out.wait_event(ev_dec[i])
                binding.parallax_copy(hout, dout, stream=s_out)
                ev_out[i].record(s_out)
            for i in range(nbuf):
                stream.wait_event(ev_out[i])

        chain()
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            chain()
        k_e2e = max(nbuf, k_e2e // nbuf * nbuf)

        def run_e2e(k_steps, start_event=None):
            for _ in range(k_steps // nbuf):
                g_e2e.replay()
    else:
        # large pools: DMA copies on two copy streams, double-buffered (each
        # step's input copy overlaps the previous step's decode, its output
        # copy the next one's), as in the contiguous bench
        transfer = ("cudaMemcpyAsync (DMA) on two copy streams, double-buffered: each step's "
                    "input copy overlaps the previous step's decode, its output copy the next one's")
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        slots = []
        for _ in range(2):
            blk = torch.zeros(nb, dtype=torch.uint8, device=dev)
            views = {k: blk[o:o + x[k].numel() * x[k].element_size()].view(x[k].dtype)
                     .view(x[k].shape) for k, o in zip(names, offs)}
            slots.append({"blk": blk, "x": {**x, **views}, "out": torch.empty_like(out),
                          "out_host": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                          "in_ready": torch.cuda.Event(), "decoded": torch.cuda.Event(),
                          "out_done": torch.cuda.Event()})

        def run_e2e(k_steps, start_event=None):
            if start_event is not None:
                s_in.wait_event(start_event)
            for i in range(k_steps):
                sl = slots[i % 2]
                if i >= 2:
                    s_in.wait_event(sl["decoded"])
                with torch.cuda.stream(s_in):
                    sl["blk"].copy_(host_block, non_blocking=True)
                sl["in_ready"].record(s_in)
                stream.wait_event(sl["in_ready"])
                if i >= 2:
                    stream.wait_event(sl["out_done"])
                decode_with(sl["x"], x["k"], x["v"], sl["out"])
                sl["decoded"].record(stream)
                s_out.wait_event(sl["decoded"])
                with torch.cuda.stream(s_out):
                    sl["out_host"].copy_(sl["out"], non_blocking=True)
                sl["out_done"].record(s_out)
            for sl in slots[:min(k_steps, 2)]:
                stream.wait_event(sl["out_done"])

    run_e2e(2)
    torch.cuda.synchronize()
    dist.barrier()
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    run_e2e(k_e2e, ee0)
    ee1.record(stream)
    ee1.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    t_e2e = dist.max(ee0.elapsed_time(ee1) / 1e3)
    # CPU baseline: the oracle (it gathers the same keys into a dense cache) on
    # the first batch rows, as many as fit in the budget (rank 0, N = 1 only)
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = kv_variant_oracle_sample(args, w, x, min(10.0, args.cpu_seconds))
    hbm_peak, peak_src = measured_peaks()
    N = dist.world
    gbs = replicas.whole_job_rate(args.steps * step_kv, t, N) / 1e9
    clocks = sampler.summary()
    step_bytes = step_kv + qro_bytes(x)
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": N, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w) + f"; {desc}", "global_batch": w.B * N,
                   "seq_len": w.Lmax, "parallelism": f"replicas x{N}" if N > 1 else "single GPU",
                   "attended_keys_per_step": keys * w.Hkv, "num_splits": args.num_splits,
                   "l2": (f"rotate {nbuf} K/V pool copies ({nbuf * pool_bytes / 1e6:.0f} MB "
                          f"> 2x L2), CUDA graphs" if nbuf > 1
                          else f"pool ({pool_bytes / 1e9:.1f} GB) larger than L2")},
        "us_per_step": t / args.steps * 1e6,
        "kv_gbs_frac_of_hbm_peak": gbs / N / hbm_peak,
        "softmax_r0": {"us_per_step": t_s * 1e6, "parallax_us_per_step_same_blocks": t_p * 1e6,
                       "parallax_over_softmax_latency": t_p / t_s,
                       "method": f"5 alternating blocks of {blk} steps each, medians"},
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
        "e2e": {"value": N * k_e2e * step_kv / t_e2e / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": nb,
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
                "us_per_step": t_e2e / k_e2e * 1e6, "transfer": transfer},
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "hbm", "achieved": step_bytes / (t / args.steps) / 1e9,
                     "peak": hbm_peak, "unit": "GB/s",
                     "frac": step_bytes / (t / args.steps) / 1e9 / hbm_peak, "traffic": None,
                     "kernel": "whole step (split-KV + merge)", "peak_source": peak_src,
                     "algorithmic_bytes_per_step": step_bytes},
        "cpu_baseline": cpu,
    }
    if dist.rank == 0:
        print(json.dumps(line))
    dist.close()
    return 0


def run_kv_variant_reference(args):
    """The reference arm of the paged / block-sparse lines: the fp64 oracle
    (gathering the same keys) on the first batch rows of the same seeded
    workload, on the host (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    w = inputs.WORKLOADS[args.workload]
    rows = min(w.B, 16)  # the inputs of the first rows only, drawn on the host
    wsub = inputs.Workload(w.name, rows, w.Hq, w.Hkv, w.D, w.Lmax, w.dtype, w.seed, w.lengths,
                           w.r_scale, w.k_offset_std, w.scale)
    x = (inputs.make_paged(wsub, args.page_size, "cpu") if args.kv_mode == "paged"
         else inputs.make_block_sparse(wsub, args.density, "cpu"))
    per_step = min(5.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        kv_variant_oracle_sample(args, wsub, x, per_step)
    vals, t0 = [], time.perf_counter()
    for _ in range(args.steps):
        vals.append(kv_variant_oracle_sample(args, wsub, x, per_step))
    secs = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / max(1, args.steps) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w) + f"; {args.kv_mode}",
                       "parallelism": "rank 0 only (host CPU)"},
            "cpu_baseline": dict(vals[-1], value=value),
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def kv_variant_oracle_sample(args, w, x, budget_s):
    """The fp64 oracle on the first batch rows of a paged or block-sparse
    step: time one row, then as many rows as fit in budget_s. GB/s of the K/V
    the rows attend."""
    import oracle
    scale, esz = x["scale"], 2

    def rows_input(n_rows):
        idx = slice(0, n_rows)
        q, r, lens = x["q"][idx].cpu(), x["r"][idx].cpu(), x["seqlens"][idx].cpu()
        if args.kv_mode == "paged":
            table = x["table"][idx].cpu()
            used = torch.unique(table)  # only the pages these rows use, renumbered
            remap = torch.full((int(used.max()) + 1,), -1, dtype=torch.int64)
            remap[used] = torch.arange(used.numel())
            dev_used = used.to(x["k"].device)
            kp, vp = x["k"][dev_used].cpu(), x["v"][dev_used].cpu()
            keys = int(lens.to(torch.int64).clamp(0, w.Lmax).sum())
            call = lambda: oracle.parallax_decode_paged(q, r, kp, vp, remap[table.long()].numpy(),
                                                        lens, scale)
        else:
            ids, cnt = x["block_ids"][idx].cpu(), x["num_blocks"][idx].cpu()
            k, v = x["k"][idx].cpu(), x["v"][idx].cpu()
            keys = sum(int((lens[b].long() - 64 * ids[b, :int(cnt[b])].long()).clamp(0, 64).sum())
                       for b in range(n_rows))
            call = lambda: oracle.parallax_decode_block_sparse(q, r, k, v, ids, cnt, lens, scale)
        return call, 2 * keys * w.Hkv * w.D * esz

    call, _ = rows_input(1)
    t0 = time.perf_counter()
    call()
    one = max(1e-3, time.perf_counter() - t0)
    n_rows = max(1, min(w.B, int(budget_s / one), 16))
    call, kv = rows_input(n_rows)
    t0 = time.perf_counter()
    call()
    secs = time.perf_counter() - t0
    return {"value": kv / secs / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"fp64 oracle ({args.kv_mode}: the same keys gathered into a dense cache), "
                      f"one pass over batch rows 0..{n_rows - 1} ({n_rows} of {w.B}); {secs:.1f} s"}


# ------------------------------------------------------------- GPU timing ----

class DecodeRig:
    """One decode workload resident on the device: its K/V copies (rotated
    when smaller than twice the L2), output, workspace and split count, and
    runners for the Parallax and R = 0 steps."""

    def __init__(self, w, dev, stream, out_dtype, num_splits):
        from parameterized_local_linear_b200 import binding
        self.binding, self.w, self.dev, self.stream = binding, w, dev, stream
        self.x = inputs.make_inputs(w, device=dev, pad_value=None)
        self.step_kv = kv_bytes(self.x)
        self.l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.nbuf = 1
        if w.kv_bytes_full() < 2 * self.l2:
            self.nbuf = max(2, math.ceil(2 * self.l2 / w.kv_bytes_full()))
            self.l2_note = (f"rotate {self.nbuf} K/V copies "
                            f"({self.nbuf * w.kv_bytes_full() / 1e6:.0f} MB > 2x L2)")
        else:
            self.l2_note = f"inputs ({w.kv_bytes_full() / 1e9:.1f} GB of K/V) larger than L2"
        x = self.x
        self.bufs = [x] + [{k: (v.clone() if torch.is_tensor(v) else v) for k, v in x.items()}
                           for _ in range(self.nbuf - 1)]
        self.out = torch.empty((w.B, w.Hq, w.D), device=dev, dtype=out_dtype)
        # num_splits = 0: the library's own schedule (a cluster per item for few
        # items, else split-KV partitions + merge); > 0 forces that many partitions
        self.num_splits = num_splits
        self.plan = (binding.parallax_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax, w.dtype,
                                                  out_dtype) if num_splits == 0
                     else {"grid_ctas": num_splits, "cluster_ctas": 0})
        self.P = (num_splits if num_splits > 0 else
                  binding.parallax_default_splits(w.B, w.Hq, w.Hkv, w.Lmax, w.dtype))
        self.ws = binding.Workspace(w.B, w.Hq, w.Hkv, w.D, w.Lmax, self.P, device=dev)
        self.use_graphs = self.nbuf > 1
        self.runners = {True: self._make_runner(True), False: self._make_runner(False)}

    def step(self, b, probe=True, out=None):
        bd = self.binding
        out = self.out if out is None else out
        if probe:
            bd.parallax_decode(b["q"], b["r"], b["k"], b["v"], b["seqlens"], scale=b["scale"],
                               out=out, num_splits=self.num_splits, workspace=self.ws,
                               stream=self.stream)
        else:
            bd.parallax_softmax_decode(b["q"], b["k"], b["v"], b["seqlens"], scale=b["scale"],
                                       out=out, num_splits=self.num_splits,
                                       workspace=self.ws, stream=self.stream)

    def _make_runner(self, probe):
        """run(k) enqueues exactly k steps. Graph-replayed workloads replay
        whole chains of `chain` steps (a multiple of the rotation) and one
        graph of the remainder; run.prepare(k) captures what run(k) replays,
        so that no capture falls inside a timed region."""
        bufs, nbuf = self.bufs, self.nbuf
        if not self.use_graphs:
            def run(k):
                for i in range(k):
                    self.step(bufs[i % nbuf], probe)
            run.prepare = lambda k: None
            return run
        for b in bufs:  # warm the launch path outside capture
            self.step(b, probe)
        torch.cuda.synchronize()
        graphs = {}
        chain = nbuf * max(1, 256 // nbuf)

        def graph(n):
            if n not in graphs:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self.stream):
                    for i in range(n):
                        self.step(bufs[i % nbuf], probe)
                graphs[n] = g
            return graphs[n]

        def prepare(k):
            if k >= chain:
                graph(chain)
            if k % chain:
                graph(k % chain)

        def run(k):
            prepare(k)
            for _ in range(k // chain):
                graphs[chain].replay()
            if k % chain:
                graphs[k % chain].replay()
        run.prepare = prepare
        return run

    def host_seconds_per_step(self, probe=True, k=None):
        """Host time to enqueue one step (the gate in front of a timed region
        must outlast the enqueueing of the steps behind it)."""
        run = self.runners[probe]
        k = k or (256 if self.use_graphs else 4)
        run.prepare(k)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        run(k)
        dt = time.perf_counter() - t0
        torch.cuda.synchronize()
        return dt / k


def timed_plain(dist, stream, fn, k_steps, w_steps):
    """W untimed steps, then K steps between two events, enqueued as the host
    goes (the end-to-end loop: host launch gaps and copies are part of it)."""
    fn(w_steps)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    fn(k_steps)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(e0.elapsed_time(e1) / 1e3)


def timed_steps(dist, stream, fn, k_steps, w_steps, sampler=None):
    """W untimed steps, then exactly K steps timed by gated_region (queued
    behind a sleep kernel), barrier and synchronize on both sides, max over
    ranks."""
    fn(w_steps)
    torch.cuda.synchronize()
    n = max(1, min(k_steps, 4))
    t0 = time.perf_counter()
    fn(n)  # the host's enqueue time per step sizes the gate
    host = (time.perf_counter() - t0) / n
    torch.cuda.synchronize()
    dist.barrier()
    t = gated_region(stream, lambda: fn(k_steps), host * k_steps, sampler)
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(t)


def gated_region(stream, enqueue, host_s, sampler=None):
    """Time the launches `enqueue()` issues with CUDA events on `stream`, with
    the launches queued before the region starts: a sleep kernel holds the
    stream (torch.cuda._sleep, a fixed cycle count) while the host enqueues,
    so that host launch gaps do not land in the timed region. Returns
    seconds between the events."""
    gate_s = min(0.25, max(0.002, 1.5 * host_s))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(gate_s * 2.0e9))  # cycles at up to 2 GHz
    e0.record(stream)
    enqueue()
    e1.record(stream)
    if sampler:
        sampler.__enter__()
    e1.synchronize()
    if sampler:
        sampler.__exit__(None, None, None)
    return e0.elapsed_time(e1) / 1e3


def same_block_medians(rig, rounds, blk):
    """The R = 0 comparator: blocks of Parallax and softmax steps alternate,
    so both see the same power and clock state (B200 runs at its power cap
    while streaming HBM); each block is a gated region of whole steps."""
    per = {True: [], False: []}
    host = {p: rig.host_seconds_per_step(p) for p in (True, False)}
    for p in (True, False):
        rig.runners[p].prepare(blk)
        rig.runners[p](min(blk, 2 * rig.nbuf))
    torch.cuda.synchronize()
    for _ in range(rounds):
        for probe in (True, False):
            run = rig.runners[probe]
            per[probe].append(gated_region(rig.stream, lambda: run(blk), host[probe] * blk) / blk)
    return statistics.median(per[True]), statistics.median(per[False]), per


def qwen_companion(dev, stream, dist):
    """The latency-bound Qwen-3 decode step (B = 1, 16.8 MB of K/V) measured
    beside the default workload: same-block medians of Parallax and R = 0,
    and the pages' q05/q50/q95 statistic over trials."""
    w = inputs.WORKLOADS["qwen"]
    rig = DecodeRig(w, dev, stream, torch.bfloat16, 0)
    blk = rig.nbuf * max(1, 800 // rig.nbuf)
    t_p, t_s, _ = same_block_medians(rig, 8, blk)
    per_trial = []
    run = rig.runners[True]
    n_trial = rig.nbuf * max(1, 50 // rig.nbuf)
    host = rig.host_seconds_per_step(True)
    for _ in range(20):
        per_trial.append(gated_region(stream, lambda: run(n_trial), host * n_trial) / n_trial)
    per_trial.sort()
    out = {"workload": workload_desc(w), "plan": rig.plan, "l2": rig.l2_note,
           "us_per_step_same_blocks": dist.max(t_p) * 1e6,
           "softmax_r0_us_per_step": dist.max(t_s) * 1e6,
           "parallax_over_softmax_latency": t_p / t_s,
           "kv_gbs_same_blocks": rig.step_kv / dist.max(t_p) / 1e9,
           "latency_us": {"q05": per_trial[1] * 1e6, "q50": statistics.median(per_trial) * 1e6,
                          "q95": per_trial[-2] * 1e6},
           "method": f"8 alternating gated blocks of {blk} graph-replayed steps (medians); "
                     f"20 trials of {n_trial} steps for the quantiles"}
    rc, _ = rig.ws.status()
    if rc != 0:
        raise SystemExit(f"device status after the qwen step: {rig.binding.parallax_status_string(rc)}")
    del rig
    torch.cuda.empty_cache()
    return out


def main():
    args = parse_args()
    if args.prefill:
        return run_prefill(args)
    if args.kv_mode != "contiguous":
        return run_kv_variant(args)
    if args.impl == "reference":
        return run_reference(args)

    from parameterized_local_linear_b200 import binding

    dist = Dist(args.gpus)
    dist.init_gpu()
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load_library()
    w = inputs.WORKLOADS[args.workload]
    if args.batch is not None or args.seed is not None:
        w = inputs.Workload(w.name + (f"-B{args.batch}" if args.batch is not None else ""),
                            args.batch if args.batch is not None else w.B, w.Hq, w.Hkv, w.D,
                            w.Lmax, w.dtype, args.seed if args.seed is not None else w.seed,
                            w.lengths, w.r_scale, w.k_offset_std, w.scale)
    stream = torch.cuda.Stream(device=dev)  # graphs can not be captured on the legacy stream
    torch.cuda.set_stream(stream)

    out_dtype = torch.float32 if args.out_dtype == "f32" else torch.bfloat16
    rig = DecodeRig(w, dev, stream, out_dtype, args.num_splits)
    x, bufs, nbuf, out, ws, P = rig.x, rig.bufs, rig.nbuf, rig.out, rig.ws, rig.P
    step, step_kv, use_graphs = rig.step, rig.step_kv, rig.use_graphs
    run_plx, run_soft = rig.runners[True], rig.runners[False]

    # ---- the timed region: exactly K steps after W warm-up steps ----
    run_plx.prepare(args.steps)
    run_plx(args.warmup)
    host_s = rig.host_seconds_per_step(True) * args.steps
    torch.cuda.synchronize()
    dist.barrier()
    sampler = ClockSampler(dev.index)
    t_plx = dist.max(gated_region(stream, lambda: run_plx(args.steps), host_s, sampler))
    torch.cuda.synchronize()
    dist.barrier()

    # ---- sustained: whole steps over at least one second ----
    per_step = t_plx / args.steps
    chain = nbuf * max(1, 256 // nbuf) if use_graphs else 1
    k_sus = max(args.steps, math.ceil(1.0 / per_step / chain) * chain)
    run_plx.prepare(k_sus)
    sus_sampler = ClockSampler(dev.index)
    torch.cuda.synchronize()
    dist.barrier()
    t_sus = dist.max(gated_region(stream, lambda: run_plx(k_sus),
                                  rig.host_seconds_per_step(True) * k_sus, sus_sampler))
    sus_clocks = sus_sampler.summary()

    blk = nbuf * max(1, 800 // nbuf) if use_graphs else 10
    rounds = 8 if use_graphs else 5
    t_plx_blk, t_soft_blk, _ = same_block_medians(rig, rounds, blk)
    t_soft = dist.max(t_soft_blk)
    t_plx_blk = dist.max(t_plx_blk)
    rc, bits = ws.status()
    if rc != 0:
        raise SystemExit(f"device status after timing: {binding.parallax_status_string(rc)}")

    # ---- per-launch duration of the dominant kernel, live ----
    # The split-KV kernel alone (phase 1) on the partition path; on the
    # cluster path the step is that one kernel. Back-to-back launches (each
    # waits for the previous one's end, so the period is one launch's
    # duration). Launch-bound sizes replay them from a CUDA graph; large ones
    # are timed with events around each launch.
    cluster = rig.plan["cluster_ctas"] > 0

    def phase1(b):
        if cluster:
            step(b)
            return
        binding.parallax_decode_phase(1, True, b["q"], b["r"], b["k"], b["v"], b["seqlens"],
                                      out, ws, scale=b["scale"], num_splits=P, stream=stream)

    if use_graphs:
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, stream=stream):
            for b in bufs:
                phase1(b)
        reps = max(1, min(args.steps, 20000) // nbuf)
        for _ in range(3):
            g1.replay()
        torch.cuda.synchronize()

        def enqueue_p1():
            for _ in range(reps):
                g1.replay()
        main_s = gated_region(stream, enqueue_p1, 1e-5 * reps) / (reps * nbuf)
        main_launches = reps * nbuf
    else:
        nprof = min(args.steps, 50)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nprof)]
        for i, (a, b) in enumerate(evs):
            a.record(stream)
            phase1(bufs[i % nbuf])
            b.record(stream)
        torch.cuda.synchronize()
        main_s = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
        main_launches = nprof
    step(bufs[0])  # leave a complete result behind

    # ---- end to end through the public API with host buffers ----
    # A step's inputs (q, r and the lengths) sit in one pinned host block and
    # go over in one copy, into one device block whose views the call takes;
    # the output comes back every step.
    def packed_views(tensors, device):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 255) // 256 * 256
        block = torch.empty(n, dtype=torch.uint8, device=device)
        views = [block[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                 for o, t in zip(offs, tensors)]
        return block, views

    host_block, host_views = packed_views([x["q"], x["r"], x["seqlens"]], "cpu")
    for hv, t in zip(host_views, (x["q"], x["r"], x["seqlens"])):
        hv.copy_(t.cpu())
    host_block = host_block.pin_memory()
    h2d = host_block.numel()
    k_e2e = min(args.steps, 2000 if use_graphs else args.steps)

    if use_graphs:
        # Small per-step transfers (graph-replayed workloads) go through
        # parallax_copy (a kernel over the mapped pinned blocks: ~3 us each on
        # the GPU timeline against ~8 us for a DMA copy of a few KB). Each
        # step of a chain has its own input block and output buffer; its input
        # copy runs on a side stream ahead of its decode and its output copy on
        # another behind it, so the copies of neighbouring steps overlap the
        # decode (the steps are independent batches, as in a serving loop).
        # The chain is replayed from a CUDA graph as the device-resident steps
        # are; every step's two copies are inside the timed region.
        transfer = ("parallax_copy (kernel over mapped pinned host memory) on two side streams, "
                    "each step's input and output copies overlapping its neighbours' decodes")
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        dev_sets = []
        for b in bufs:
            dev_blk, (dq, dr, dsl) = packed_views([x["q"], x["r"], x["seqlens"]], dev)
            dev_sets.append((dev_blk, {**b, "q": dq, "r": dr, "seqlens": dsl}, torch.empty_like(out),
                             torch.empty(out.shape, dtype=out.dtype).pin_memory()))
        out_host = dev_sets[0][3]
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_dec = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]

        def chain():
            fork = torch.cuda.Event()
            fork.record(stream)
            s_in.wait_event(fork)
            s_out.wait_event(fork)
            for i in range(nbuf):
                dev_blk, b, dout, hout = dev_sets[i]
                binding.parallax_copy(dev_blk, host_block, stream=s_in)
                ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                step(b, out=dout)
                ev_dec[i].record(stream)
                s_out.wait_event(ev_dec[i])
                binding.parallax_copy(hout, dout, stream=s_out)
                ev_out[i].record(s_out)
            for i in range(nbuf):  # the chain ends with every output home
                stream.wait_event(ev_out[i])

        chain()
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            chain()
        k_e2e = max(nbuf, k_e2e // nbuf * nbuf)

        def run_e2e(k, start_event=None):
            for _ in range(k // nbuf):
                g_e2e.replay()
    else:
        # Large transfers: DMA copies on two copy streams, double-buffered:
        # step i's input copy overlaps step i-1's decode and its output copy
        # step i+1's (the steps are independent batches, as in a serving loop
        # that uploads the next batch while the current one runs).
        transfer = ("cudaMemcpyAsync (DMA) on two copy streams, double-buffered: each step's "
                    "input copy overlaps the previous step's decode, its output copy the next one's")
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        slots = []
        for _ in range(2):
            dev_blk, (dq, dr, dsl) = packed_views([x["q"], x["r"], x["seqlens"]], dev)
            slots.append({"blk": dev_blk, "b": {**bufs[0], "q": dq, "r": dr, "seqlens": dsl},
                          "out": torch.empty_like(out),
                          "out_host": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                          "in_ready": torch.cuda.Event(), "decoded": torch.cuda.Event(),
                          "out_done": torch.cuda.Event()})
        out_host = slots[0]["out_host"]

        def run_e2e(k, start_event=None):
            if start_event is not None:
                s_in.wait_event(start_event)
            for i in range(k):
                sl = slots[i % 2]
                if i >= 2:
                    s_in.wait_event(sl["decoded"])  # decode i-2 has read this input block
                with torch.cuda.stream(s_in):
                    sl["blk"].copy_(host_block, non_blocking=True)
                sl["in_ready"].record(s_in)
                stream.wait_event(sl["in_ready"])
                if i >= 2:
                    stream.wait_event(sl["out_done"])  # output i-2 has left this block
                step(sl["b"], out=sl["out"])
                sl["decoded"].record(stream)
                s_out.wait_event(sl["decoded"])
                with torch.cuda.stream(s_out):
                    sl["out_host"].copy_(sl["out"], non_blocking=True)
                sl["out_done"].record(s_out)
            for sl in slots[:min(k, 2)]:
                stream.wait_event(sl["out_done"])  # the region ends with the last output home

    # the end-to-end loop is timed as a user runs it: launches and copies
    # enqueued as the host goes, no gate in front
    run_e2e(min(args.warmup, 50))
    torch.cuda.synchronize()
    dist.barrier()
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    run_e2e(k_e2e, ee0)
    ee1.record(stream)
    ee1.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    t_e2e = dist.max(ee0.elapsed_time(ee1) / 1e3)
    step(bufs[0])  # leave the resident buffers' result behind
    d2h = out_host.numel() * out_host.element_size()

    # ---- latency distribution, the pages' method: q50 (q05, q95) over trials ----
    q_stats = None
    if use_graphs:
        per_trial = []
        n_trial = nbuf * max(1, 50 // nbuf)
        host_t = rig.host_seconds_per_step(True) * n_trial
        for _ in range(20):
            per_trial.append(gated_region(stream, lambda: run_plx(n_trial), host_t) / n_trial * 1e6)
        per_trial.sort()
        q_stats = {"q05": per_trial[1], "q50": statistics.median(per_trial), "q95": per_trial[-2],
                   "unit": "us", "method": f"20 trials of {n_trial} graph-replayed steps"}

    # ---- CPU oracle baseline and accuracy (rank 0, N = 1 only) ----
    cpu, accuracy = None, None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        xh = {k: (v[: min(w.B, 64)].cpu() if torch.is_tensor(v) else v) for k, v in x.items()}
        wsub = inputs.Workload(w.name, min(w.B, 64), w.Hq, w.Hkv, w.D, w.Lmax, w.dtype, w.seed,
                               "full", w.r_scale, w.k_offset_std, w.scale)
        xh["seqlens"] = x["seqlens"][: wsub.B].cpu()
        v, cores, desc, _ = oracle_sample(wsub, xh, args.cpu_seconds)
        cpu = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}
        # the step's output on the first rows against the oracle (the pages'
        # bench reports accuracy beside latency)
        import oracle
        rows = min(w.B, 8)
        step(bufs[0])
        torch.cuda.synchronize()
        ref = oracle.parallax_decode(xh["q"][:rows], xh["r"][:rows], xh["k"][:rows],
                                     xh["v"][:rows], xh["seqlens"][:rows], xh["scale"])
        got = out[:rows].double().cpu().numpy()
        err = float((abs(got - ref) / abs(ref).clip(min=1.0)).max())
        accuracy = {"max_scaled_err_vs_oracle": err, "rows": rows,
                    "out_dtype": args.out_dtype, "tolerance": 1e-4 if args.out_dtype == "f32" else 2e-2}

    # ---- the latency-bound Qwen step beside the default workload ----
    companion = None
    if args.workload != "qwen" and not args.no_companion:
        companion = qwen_companion(dev, stream, dist)

    hbm_peak, peak_src = measured_peaks()
    N = dist.world
    gbs = replicas.whole_job_rate(args.steps * step_kv, t_plx, N) / 1e9
    main_bytes = step_kv + qro_bytes(x)
    achieved = main_bytes / main_s / 1e9
    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": N, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_plx / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": w.B * N, "seq_len": w.Lmax,
                   "parallelism": f"replicas x{N}" if N > 1 else "single GPU",
                   "num_splits": args.num_splits, "plan": rig.plan, "l2": rig.l2_note,
                   "cuda_graphs": use_graphs,
                   "out_dtype": args.out_dtype,
                   "timing": "CUDA events around exactly K steps, enqueued behind a sleep "
                             "kernel so that no host launch gap is timed"},
        "us_per_step": t_plx / args.steps * 1e6,
        "kv_gbs_frac_of_hbm_peak": gbs / N / hbm_peak,
        "sustained": {"steps": k_sus, "seconds": t_sus, "us_per_step": t_sus / k_sus * 1e6,
                      "value": replicas.whole_job_rate(k_sus * step_kv, t_sus, N) / 1e9,
                      "unit": "GB/s",
                      "clocks": {k: sus_clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons",
                                                            "samples")},
                      "method": "whole steps over at least one second, one gated region"},
        "softmax_r0": {"us_per_step": t_soft * 1e6, "kv_gbs": N * step_kv / t_soft / 1e9,
                       "parallax_us_per_step_same_blocks": t_plx_blk * 1e6,
                       "parallax_over_softmax_latency": t_plx_blk / t_soft,
                       "method": f"{rounds} alternating gated blocks of {blk} steps each, medians"},
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
        "e2e": {"value": N * k_e2e * step_kv / t_e2e / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": t_e2e / k_e2e * 1e6, "transfer": transfer},
        # split-KV + merge per step, or the one cluster kernel, in the timed region
        "gpu_launches": (1 if cluster else 2) * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": profiled_traffic(w, "cluster" if cluster else "tc"),
                     "kernel": ("parallax_cluster_kernel (the whole step)" if cluster
                                else "parallax_tc_kernel (split-KV)"), "peak_source": peak_src,
                     "kernel_us": main_s * 1e6, "launches_timed": main_launches,
                     "algorithmic_bytes_per_launch": main_bytes},
        "cpu_baseline": cpu,
        "latency_distribution": q_stats,
        "accuracy": accuracy,
        "qwen_step": companion,
    }
    if dist.rank == 0:
        print(json.dumps(line))
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
