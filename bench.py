"""Benchmark of the fused chunked KL loss (forward + backward) on B200.

    python bench.py [--gpus N --steps K --warmup W] [--config 8b|small|tiny|large_vocab|sweep] [--N n]
    python bench.py --impl reference ...      # the CPU oracle on a bounded sample (baseline arm)
    python bench.py --sweep                   # peak GB and tokens/s vs N (d=4096, V=128256, tau=2)

One step = kdkl_forward + kdkl_backward over one batch of seeded synthetic
inputs already resident in HBM.  Rank 0 prints one JSON line.  With N > 1
(torchrun) the step is token-sharded data parallel: every rank holds its own
seeded batch of the workload's size (weak scaling), normalises by the
all-reduced valid-token count and all-reduces dW over NCCL; `value` is the
tokens of all ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "fused KL fwd+bwd tokens/sec and % of B200 bf16 tensor peak; peak GB vs N"
UNIT = "tokens/s"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]), "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ----------------------------------------------------------------------------- ncu traffic record
def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed (what the compiler sees)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_sources_digest(read=None) -> str:
    """sha256 over the code of the CUDA sources (comments and layout excluded); a traffic
    record only applies to the kernels it was taken on.  `read(name)` overrides how a
    source file's text is obtained (default: the working tree)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "output_head_kl_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            if read is None:
                with open(os.path.join(csrc, name), encoding="utf-8") as f:
                    text = f.read()
            else:
                text = read(name)
            h.update(name.encode() + b"\0" + _code_only(text).encode())
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes (read + write) per launch from the committed ncu record, or None if stale/absent."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("sources_sha256") != kernel_sources_digest():
        return None
    entry = rec.get("workloads", {}).get(workload, {}).get(kernel)
    return None if entry is None else float(entry["dram_bytes_per_launch"])


_NCU_KIND = {"0": "fwd_lse_gemm", "1": "bwd_grad_gemm", "2": "bwd_dhidden_gemm", "3": "bwd_dw_gemm",
             "4": "teacher_topk_gemm"}


def record_traffic(csv_path: str, workload: str) -> dict:
    """Writes profiles/traffic.json from an ncu --csv log of dram__bytes_{read,write}.sum (per-launch mean)."""
    import csv
    import re
    rows = list(csv.reader(open(csv_path)))
    head = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    hdr = rows[head]
    kname, mname, mval = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    per_launch = {}
    for r in rows[head + 1:]:
        if len(r) <= mval or not r[mname].startswith("dram__bytes_"):
            continue
        m = re.search(r"gemm_kernel<(\d+)", r[kname])
        if not m:
            continue
        key = (_NCU_KIND[m.group(1)], r[0])
        per_launch[key] = per_launch.get(key, 0.0) + float(r[mval].replace(",", ""))
    sums = {}
    for (kind, _), b in per_launch.items():
        sums.setdefault(kind, []).append(b)
    p = os.path.join(ROOT, "profiles", "traffic.json")
    rec = json.load(open(p)) if os.path.exists(p) else {}
    if rec.get("sources_sha256") != kernel_sources_digest():
        rec = {"sources_sha256": kernel_sources_digest(), "workloads": {}}
    # kernels captured in separate runs (the forward, the backward chunk) merge into one entry
    rec["workloads"].setdefault(workload, {}).update(
        {k: {"dram_bytes_per_launch": sum(v) / len(v), "launches_captured": len(v)} for k, v in sums.items()})
    with open(p, "w") as f:
        json.dump(rec, f, indent=1, sort_keys=True)
    return rec


# ----------------------------------------------------------------------------- clocks
_REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        cmd = ["nvidia-smi", "-i", self.gpu_id,
               "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=5)
        sm, smax, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 4:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                mask = int(parts[3], 16)
            except ValueError:
                continue
            for bit, name in _REASON_BITS.items():
                if mask & bit and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.3 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for(dev_index: int) -> str:
    import torch
    props = torch.cuda.get_device_properties(dev_index)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        s = str(uuid)
        return s if s.startswith("GPU-") else "GPU-" + s
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[dev_index]
    return str(dev_index)


# ----------------------------------------------------------------------------- same-GPU reference
def same_gpu_gemm_reference(dev, seconds: float = 3.0, size: int = 8192):
    """cuBLAS bf16 GEMM (torch.matmul, 2 n^3 flops) looped for `seconds` on this GPU,
    with its clock: context for how much of the gap to the fixed peak is this GPU's
    power-capped clock.  Not a kernel of this library."""
    import torch
    a = torch.randn(size, size, device=dev, dtype=torch.bfloat16)
    b = torch.randn(size, size, device=dev, dtype=torch.bfloat16)
    c = torch.empty(size, size, device=dev, dtype=torch.bfloat16)
    for _ in range(3):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    sampler = ClockSampler(gpu_id_for(dev.index or 0))
    sampler.start()
    n = 0
    e0.record()
    while time.perf_counter() - t0 < seconds:
        for _ in range(10):
            torch.matmul(a, b, out=c)
        n += 10
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / n
    del a, b, c
    return {"kind": "cuBLAS bf16 GEMM 8192^3 via torch.matmul, sustained loop", "tflops": 2.0 * size ** 3 / ms / 1e9,
            "sm_mhz": clocks.get("sm_mhz"), "reasons": clocks.get("reasons")}


# ----------------------------------------------------------------------------- oracle arm
# Rows per timed oracle sample, the same in the GPU line's cpu_baseline and in the
# reference arm: one block of the oracle's row loop (its default row chunk), so the
# two legs time identical work per sample.
CPU_SAMPLE_ROWS = 64


def oracle_weight(x: synth.Inputs):
    """W widened to float64 once, outside every timed region (input marshalling, not the method)."""
    from oracle import kl as O
    return O.bf16_bits_to_f64(x.W_bits)


def oracle_sample(x: synth.Inputs, W64, rows: int, seed: int):
    """Times the CPU oracle (as it stands) on a bounded seeded sample of the workload's rows:
    a full forward + backward of that sample (loss, lse, dHidden and its dW contribution)."""
    from oracle import kl as O
    sel = synth.sample_rows(x.hidden_bits.shape[0], rows, seed)
    sub = (x.hidden_bits[sel], x.W_bits, x.topk_idx[sel], x.topk_logit[sel], x.mask[sel], x.tau)
    t0 = time.perf_counter()
    O.kl_loss(*sub, W_f64=W64)
    dt = time.perf_counter() - t0
    return sel.size, dt


def sample_text(rows: int, w: synth.Workload) -> str:
    return (f"{rows} seeded rows of the {w.name} workload per sample, one full fwd+bwd (loss, lse, dHidden, "
            f"dW contribution) in numpy float64; W widened to float64 once before timing")


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def host_cpu_info() -> dict:
    """The BLAS library numpy calls and the CPU cores this process may run on."""
    blas = None
    try:
        dep = np.show_config(mode="dicts").get("Build Dependencies", {}).get("blas", {})
        blas = f"{dep.get('name', '?')} {dep.get('version', '')}".strip()
    except Exception:
        pass
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = os.cpu_count()
    return {"blas": blas, "blas_threads": blas_threads(), "affinity_cores": affinity}


def cpu_baseline(x: synth.Inputs, w: synth.Workload, W64, budget_s: float = 8.0, max_samples: int = 16):
    """The oracle timed on repeated seeded samples of CPU_SAMPLE_ROWS rows (about budget_s seconds)."""
    done, total, i = 0, 0.0, 0
    while i < max_samples and (i < 2 or total < budget_s):
        n, dt = oracle_sample(x, W64, CPU_SAMPLE_ROWS, seed=4242 + i)
        done += n
        total += dt
        i += 1
    return {"value": done / total, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": sample_text(min(CPU_SAMPLE_ROWS, x.hidden_bits.shape[0]), w) + f"; {i} samples, {total:.1f} s",
            **host_cpu_info()}


def run_reference(args, w: synth.Workload, N: int):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = synth.make_inputs(w, N=N)
    W64 = oracle_weight(x)
    for i in range(args.warmup):
        oracle_sample(x, W64, CPU_SAMPLE_ROWS, seed=1000 + i)
    times = []
    done = 0
    for i in range(args.steps):
        n, dt = oracle_sample(x, W64, CPU_SAMPLE_ROWS, seed=2000 + i)
        times.append(dt)
        done += n
    rows = done // max(1, args.steps)      # the sample never exceeds the workload's N rows
    total = sum(times)
    value = done / total
    cores = blas_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "N": N, "d": w.d, "V": w.V, "K": w.K, "tau": w.tau,
                       "sample_rows_per_step": rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample_text(rows, w), **host_cpu_info()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ranks
def replica_seed(w: synth.Workload, N: int, rank: int) -> int:
    """Each rank runs an independent replica on its own seeded batch."""
    return synth.seed_for(w, N) + 7919 * rank


def max_over_ranks(value: float, device, world: int) -> float:
    """The slowest rank's time (a collective only for timing, never on the data path)."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- GPU arm
def _bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def time_workload(K, dev, x: synth.Inputs, *, fused: bool, steps: int, warmup: int, chunk_tokens: int = 0):
    """Forward + backward (or the fused step) on device-resident inputs: warm-up steps,
    then `steps` steps timed with CUDA events on the launching stream, with the clocks
    sampled meanwhile and the peak of torch-allocated bytes (inputs, outputs, workspace)."""
    import torch
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    Nn, d, V, Kc = x.shape
    hidden, W = _bf16(x.hidden_bits).to(dev), _bf16(x.W_bits).to(dev)
    idx, logit = torch.from_numpy(x.topk_idx).to(dev), torch.from_numpy(x.topk_logit).to(dev)
    mask = torch.from_numpy(x.mask).to(dev)
    ws_bytes = (K.kdkl_forward_backward_workspace_bytes(Nn, d, V, Kc, chunk_tokens) if fused
                else K.kdkl_workspace_bytes(Nn, d, V, Kc, chunk_tokens))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(Nn, dtype=torch.float32, device=dev)
    dH = torch.empty(Nn, d, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if fused:
            K.kdkl_forward_backward(hidden, W, idx, logit, mask, x.tau, loss, lse, dH, dW, ws,
                                    chunk_tokens=chunk_tokens, stream=stream)
        else:
            K.kdkl_forward(hidden, W, idx, logit, mask, x.tau, loss, lse, ws, stream=stream)
            K.kdkl_backward(hidden, W, idx, logit, mask, x.tau, lse, None, dH, dW, ws, chunk_tokens=chunk_tokens,
                            stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    flags = K.kdkl_read_device_flags(ws)
    peak = torch.cuda.max_memory_allocated(dev) - base
    sampler = ClockSampler(gpu_id_for(dev.index or 0))
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / steps
    del hidden, W, idx, logit, mask, ws, loss, lse, dH, dW
    torch.cuda.empty_cache()
    flops = (6.0 if fused else 8.0) * Nn * d * V
    return {"N": Nn, "ms_per_step": ms, "tokens_per_s": Nn / (ms * 1e-3),
            "tflops": synth.flops_fwd_bwd(Nn, d, V) / (ms * 1e-3) / 1e12,
            "executed_tflops": flops / (ms * 1e-3) / 1e12, "peak_gb": peak / 1e9, "workspace_gb": ws_bytes / 1e9,
            "device_flags": flags, "steps": steps, "warmup": warmup,
            "sm_mhz": clocks.get("sm_mhz"), "clock_reasons": clocks.get("reasons")}


def extra_workloads(K, dev, peaks, steps: int = 2, warmup: int = 3) -> dict:
    """The metric's other parts on the same run: peak memory and throughput against N over
    the long-context sweep (one seeded draw at the largest N, leading rows for the smaller
    N), the large-vocabulary head, and the one-call fused step on the 8B-class head."""
    out = {}
    t0 = time.perf_counter()
    sw = synth.CONFIGS["sweep"]
    big = synth.make_inputs(sw, N=max(synth.SWEEP_N))
    pts = []
    for n in synth.SWEEP_N:
        sub = synth.Inputs(big.hidden_bits[:n], big.W_bits, big.topk_idx[:n], big.topk_logit[:n], big.mask[:n],
                           big.tau)
        r = time_workload(K, dev, sub, fused=False, steps=steps, warmup=warmup)
        r["frac_of_bf16_peak"] = r["tflops"] / peaks["bf16_tflops"]
        pts.append(r)
    del big
    # peak = a + b N over the points whose chunk buffer has its full 8192-token size
    fit_pts = [p for p in pts if p["N"] >= 16384]
    Ns = np.array([p["N"] for p in fit_pts], dtype=float)
    P = np.array([p["peak_gb"] * 1e9 for p in fit_pts])
    b, a = np.polyfit(Ns, P, 1)
    out["sweep"] = {"workload": f"sweep d={sw.d} V={sw.V} K={sw.K} tau={sw.tau}",
                    "inputs": f"one seeded draw at N={max(synth.SWEEP_N)}, leading rows for smaller N",
                    "points": pts,
                    "peak_fit": {"over_N": [int(n) for n in Ns], "intercept_gb": a / 1e9,
                                 "slope_kb_per_token": b / 1e3, "max_resid_mb": float(np.abs(P - a - b * Ns).max()) / 1e6,
                                 "nxv_bf16_kb_per_token": 2 * sw.V / 1e3}}
    lv = synth.CONFIGS["large_vocab"]
    r = time_workload(K, dev, synth.make_inputs(lv), fused=False, steps=steps, warmup=warmup)
    r["frac_of_bf16_peak"] = r["tflops"] / peaks["bf16_tflops"]
    r["frac_of_bf16_peak_sustained"] = r["tflops"] / peaks["bf16_tflops_sustained"]
    out["large_vocab"] = r
    w8 = synth.CONFIGS["8b"]
    r = time_workload(K, dev, synth.make_inputs(w8), fused=True, steps=max(steps, 3), warmup=warmup)
    r["note"] = "kdkl_forward_backward: each chunk's logits computed once (6 N d V executed); tflops counts 8 N d V"
    out["fused_step_8b"] = r
    out["extras_wall_s"] = time.perf_counter() - t0
    return out


def main_gpu(args, w: synth.Workload, N: int):
    import torch
    import torch.distributed as dist

    import output_head_kl_b200 as K

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    K.lib()
    t_gen = time.perf_counter()
    x = synth.make_inputs(w, N=N, seed=replica_seed(w, N, rank))
    t_gen = time.perf_counter() - t_gen
    Nn, d, V, Kc = x.shape

    h_hidden = _bf16(x.hidden_bits).pin_memory()
    h_idx = torch.from_numpy(x.topk_idx).pin_memory()
    h_logit = torch.from_numpy(x.topk_logit).pin_memory()
    h_mask = torch.from_numpy(x.mask).pin_memory()
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base_alloc = torch.cuda.memory_allocated(dev)
    W = _bf16(x.W_bits).to(dev)
    if world > 1:
        dist.broadcast(W, src=0)     # one output-head weight, replicated (data parallelism)

    hidden = h_hidden.to(dev)
    idx = h_idx.to(dev)
    logit = h_logit.to(dev)
    mask = h_mask.to(dev)
    if args.fused_step and world > 1:
        raise SystemExit("--fused-step is timed on one GPU")
    ws_bytes = (K.kdkl_forward_backward_workspace_bytes(Nn, d, V, Kc, args.chunk_tokens) if args.fused_step
                else K.kdkl_workspace_bytes(Nn, d, V, Kc, args.chunk_tokens))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(Nn, dtype=torch.float32, device=dev)
    dH = torch.empty(Nn, d, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # N > 1: token-sharded data parallelism (output_head_kl_b200.dp): each rank's batch
    # is its shard; the library counts the shard's valid tokens, the counts are summed
    # over NCCL, forward and backward normalise by that sum, the per-rank losses are
    # summed and dW is all-reduced (sum), the step's one real exchange.
    n_total = torch.zeros(1, dtype=torch.int32, device=dev)
    dp_opts = K.kdkl_options(n_valid_global=n_total) if world > 1 else None
    n_local = K.n_valid_view(ws) if world > 1 else None

    def step(bufs=None):
        hidden_, idx_, logit_, mask_ = bufs if bufs is not None else (hidden, idx, logit, mask)
        if args.fused_step:
            K.kdkl_forward_backward(hidden_, W, idx_, logit_, mask_, x.tau, loss, lse, dH, dW, ws,
                                    chunk_tokens=args.chunk_tokens, stream=stream)
            return
        if world > 1:
            K.kdkl_count_valid(idx_, logit_, mask_, x.tau, V, ws, dp_opts, stream=stream)
            n_total.copy_(n_local)
            dist.all_reduce(n_total)
            K.kdkl_forward_ex(hidden_, W, idx_, logit_, mask_, x.tau, loss, lse, ws, dp_opts, stream=stream)
            dist.all_reduce(loss)
            K.kdkl_backward_ex(hidden_, W, idx_, logit_, mask_, x.tau, lse, None, dH, dW, ws, dp_opts,
                               chunk_tokens=args.chunk_tokens, stream=stream)
            dist.all_reduce(dW)
        else:
            K.kdkl_forward(hidden_, W, idx_, logit_, mask_, x.tau, loss, lse, ws, stream=stream)
            K.kdkl_backward(hidden_, W, idx_, logit_, mask_, x.tau, lse, None, dH, dW, ws,
                            chunk_tokens=args.chunk_tokens, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flags = K.kdkl_read_device_flags(ws)
    peak_bytes = torch.cuda.max_memory_allocated(dev) - base_alloc
    K.kdkl_timing_read(reset=True)

    sampler = ClockSampler(gpu_id_for(local)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    K.kdkl_timing_enable(True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    K.kdkl_timing_enable(False)
    kt = K.kdkl_timing_read(reset=True)
    clocks = sampler.stop() if sampler else None
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, dev, world)

    # end-to-end through the public API with host buffers: every step's batch
    # (hidden, cache, mask) goes host -> device from pinned memory and its loss
    # comes back device -> host.  As a data loader would, the next batch's copy
    # runs on a second stream into a second set of buffers while this step
    # computes (the copy of batch i+1 waits until step i-1 has released them).
    h_loss = torch.empty(1, dtype=torch.float32).pin_memory()
    e2e_steps = args.steps
    bufs = [(hidden, idx, logit, mask),
            (torch.empty_like(hidden), torch.empty_like(idx), torch.empty_like(logit), torch.empty_like(mask))]
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    released = [torch.cuda.Event(), torch.cuda.Event()]

    def fetch(i):
        b = bufs[i % 2]
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(released[i % 2])
            for dst, src in zip(b, (h_hidden, h_idx, h_logit, h_mask)):
                dst.copy_(src, non_blocking=True)
            copied[i % 2].record(copy_stream)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    copy_stream.wait_event(t0)
    fetch(0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            fetch(i + 1)
        stream.wait_event(copied[i % 2])
        step(bufs[i % 2])
        released[i % 2].record(stream)
        h_loss.copy_(loss, non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / e2e_steps, dev, world)
    del bufs
    h2d = Nn * d * 2 + Nn * Kc * 4 * 2 + Nn
    d2h = 4

    out = None
    ref_gemm = None
    extras = None
    if rank == 0 and not args.no_gemm_reference:
        ref_gemm = same_gpu_gemm_reference(dev)
    if rank == 0:
        peaks = measured_peaks()
        flops = synth.flops_fwd_bwd(Nn, d, V)
        tflops = flops / (ms_max * 1e-3) / 1e12
        # dominant kernel by total time; its algorithmic flops are 2 N d V per step
        gemm_kinds = ("fwd_lse_gemm", "bwd_grad_gemm", "bwd_dhidden_gemm", "bwd_dw_gemm", "fused_fwd_gemm")
        dom = max(kt, key=lambda k: kt[k][1])
        launches, total_ms = kt[dom]
        if dom in gemm_kinds and launches:
            alg = 2.0 * Nn * d * V * args.steps / launches
            achieved = alg / (total_ms / launches * 1e-3) / 1e12
            roof = {"kernel": dom, "bound": "tensor", "achieved": achieved,
                    "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops_sustained"],
                    "peak_kind": f"bf16 dense, sustained ({peaks['source']})",
                    "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
                    "flops_per_launch": alg, "avg_launch_ms": total_ms / launches,
                    "traffic": recorded_traffic(w.name, dom)}
        else:
            roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": None, "traffic": None}
        kernels = {k: {"launches": v[0], "ms_per_step": v[1] / args.steps} for k, v in kt.items() if v[0]}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(x, w, oracle_weight(x))
        bwd_plan = K.kdkl_backward_plan(Nn, d, V, Kc, args.chunk_tokens)
        out = {
            "metric": METRIC, "value": Nn * world / (ms_max * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "N": Nn, "d": d, "V": V, "K": Kc, "tau": x.tau,
                       "chunk_tokens": bwd_plan[1], "bwd_tile_n": bwd_plan[0],
                       "l2": "inputs larger than L2 (W alone is %.2f GB); no flush" % (V * d * 2 / 1e9),
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "schedule": ("fused step: each chunk's logits computed once and kept for its gradient "
                                    "(6 N d V flops executed)") if args.fused_step else
                                   "kdkl_forward + kdkl_backward (the backward recomputes each chunk's logits)",
                       "e2e": "per step: the batch (hidden, topk_idx, topk_logit, mask) copied host->device from "
                              "pinned memory and the loss read back; W stays resident as a model weight, and "
                              "dHidden and dW stay on the device for the optimizer and the layers below"},
            "tflops": tflops,
            "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "frac_of_bf16_peak_sustained": tflops / peaks["bf16_tflops_sustained"],
            "executed_tflops": (0.75 if args.fused_step else 1.0) * tflops,
            "same_gpu_cublas": ref_gemm,
            "frac_of_same_gpu_cublas": ((0.75 if args.fused_step else 1.0) * tflops / ref_gemm["tflops"])
                                       if ref_gemm else None,
            "peak_gb": peak_bytes / 1e9,
            "workspace_gb": ws_bytes / 1e9,
            "roofline": roof,
            "kernels": kernels,
            "cpu_baseline": cpu,
            "e2e": {"value": Nn * world / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": int(sum(v[0] for v in kt.values())),
            "clocks": clocks,
            "device_flags": flags,
            "input_gen_s": t_gen,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    elif out is not None and not args.no_extras and not args.fused_step and w.name == "8b":
        del hidden, idx, logit, mask, ws, loss, lse, dH, dW, W, h_hidden, h_idx, h_logit, h_mask
        torch.cuda.empty_cache()
        extras = extra_workloads(K, dev, measured_peaks())
        out.update(extras)
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


def main_topk(args, w: synth.Workload, N: int):
    """Teacher top-K cache producer: z = hidden W^T (2 N d V flops) + per-row top-K (K = the workload's K)."""
    import torch

    import output_head_kl_b200 as K
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    K.lib()
    x = synth.make_inputs(w, N=N)
    Nn, d, V, Kc = x.shape

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    hidden, W = bf16(x.hidden_bits), bf16(x.W_bits)
    ws = torch.empty(K.kdkl_teacher_topk_workspace_bytes(Nn, d, V, Kc), dtype=torch.uint8, device=dev)
    idx = torch.empty(Nn, Kc, dtype=torch.int32, device=dev)
    val = torch.empty(Nn, Kc, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        K.kdkl_teacher_topk(hidden, W, Kc, idx, val, ws)
    torch.cuda.synchronize()
    K.kdkl_timing_read(reset=True)
    sampler = ClockSampler(gpu_id_for(0))
    sampler.start()
    time.sleep(0.3)
    K.kdkl_timing_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        K.kdkl_teacher_topk(hidden, W, Kc, idx, val, ws)
    e1.record()
    torch.cuda.synchronize()
    K.kdkl_timing_enable(False)
    kt = K.kdkl_timing_read(reset=True)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    peaks = measured_peaks()
    launches, total = kt["teacher_topk_gemm"]
    achieved = 2.0 * Nn * d * V / (total / launches * 1e-3) / 1e12
    print(json.dumps({
        "metric": "teacher top-K cache producer tokens/sec", "value": Nn / (ms * 1e-3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name + "_teacher_topk", "N": Nn, "d": d, "V": V, "K": Kc},
        "tflops": 2.0 * Nn * d * V / (ms * 1e-3) / 1e12,
        "roofline": {"kernel": "teacher_topk_gemm", "bound": "tensor", "achieved": achieved,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops_sustained"], "traffic": None},
        "kernels": {k: {"launches": v[0], "ms_per_step": v[1] / args.steps} for k, v in kt.items() if v[0]},
        "gpu_launches": int(sum(v[0] for v in kt.values())), "clocks": clocks}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kdkl", choices=["kdkl", "reference"])
    ap.add_argument("--config", default="8b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--N", type=int, default=None, help="token count override (sweep points)")
    ap.add_argument("--chunk-tokens", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sweep, large-vocabulary and fused-step objects of the default line")
    ap.add_argument("--no-gemm-reference", action="store_true",
                    help="skip the same-GPU cuBLAS GEMM timed after the run (context only)")
    ap.add_argument("--topk", action="store_true", help="time the teacher top-K cache producer instead")
    ap.add_argument("--fused-step", action="store_true",
                    help="time kdkl_forward_backward (no logit recompute) instead of kdkl_forward + kdkl_backward")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="write profiles/traffic.json from an ncu dram__bytes capture of --config's workload")
    ap.add_argument("--sweep", action="store_true",
                    help="long-context sweep (d=4096, V=128256, tau=2): one JSON line per N, single GPU")
    args = ap.parse_args()
    w = synth.CONFIGS[args.config]
    N = args.N if args.N is not None else w.N
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, w.name)))
        return 0
    if args.impl == "reference":
        return run_reference(args, w, N)
    if args.topk:
        return main_topk(args, w, N)
    if args.sweep:
        args.no_cpu_baseline = True
        args.no_gemm_reference = True
        args.no_extras = True
        for n in synth.SWEEP_N:
            rc = main_gpu(args, synth.CONFIGS["sweep"], n)
            if rc:
                return rc
            import torch
            torch.cuda.empty_cache()
        return 0
    return main_gpu(args, w, N)


if __name__ == "__main__":
    sys.exit(main())
