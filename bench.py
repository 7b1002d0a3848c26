#!/usr/bin/env python
"""Benchmark of the B200 LLaMA pre-norm decoder block.

Headline: prefill of the LLaMA-7B-shaped block (bf16, d=4096, 32 heads, head_dim
128, f=11008, B=1, T=2048) in tokens/s, with the fraction of dense BF16 tensor
peak it reaches; beside it, the KV-cache decode step of the same block (B=32,
cache 4096 -> 4224 over 128 steps) in HBM GB/s, with bf16 and with INT8 weight-only
projections.

One step = one prefill of the whole block (RMSNorm, fused QKV GEMM with RoPE and
the KV-cache scatter, causal attention, o_proj + residual, RMSNorm, gate/up GEMM
with SiLU*up, down_proj + residual) over the synthetic 2048-token input, called
through the C ABI. Inputs are resident in HBM; L2 is flushed (a 256 MB write,
then a 256 MB read, so that no dirty lines are left to write back) before every
timed step; each step is timed with CUDA events on the library's
stream. The ``e2e`` figure runs the same steps from pinned host buffers through the
public API, each step's H2D input copy and D2H output copy inside the timed region,
the copies on their own streams overlapping the neighbouring steps' compute.
Multi-GPU runs are independent replicas (one process per GPU, no data-path
collective): value = all ranks' tokens / the slowest rank's time.

The other prefill shapes are timed the same way and reported beside the headline:
``prefill_13b`` (d=5120, 40 heads, f=13824, B=4, T=1024), ``prefill_70b`` (d=8192,
64 query / 8 KV heads, f=28672, B=1, T=4096) and ``prefill_tiny_f32`` (the fp32
block, d=256, T=64), each with tokens/s, TFLOP/s, fraction of the bf16 peak, the
per-stage times and, on a 1-GPU run, the fp64 oracle timed on 64 sampled rows per
sequence with the GPU output's error at those rows. ``tp_prefill_shards`` (1-GPU runs)
times rank 0's share of a tensor-parallel 7B and 70B prefill layer at 2, 4 and 8 ranks,
with the layer's two all-reduces modelled at the measured peer bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
workload) on a bounded sample of the same prefill.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "7B-shape block prefill tokens/s & % BF16 peak; decode-step HBM GB/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
CPU_SAMPLE_T = 2048  # tokens of the 7B prefill the CPU oracle evaluates per sample (the full T)

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the dominant
# kernels, from one ncu capture on this workload (profiles/), with the SHA-256 prefix of
# the kernel's source file at capture time: once that file changes the figure no longer
# describes the kernel and the bench reports null until it is captured again.
NCU_TRAFFIC = {
    # gemm_tc_pair_kernel<256, 2>, 7B prefill (a --set full capture of the current source)
    "gate_up_swiglu_gemm": {"bytes": 197_526_784 + 37_168_128, "source": "gemm_tc.cu",
                            "sha256": "b704e33952a75bd4"},
    # attn_decode_split_kernel<128, 1>, 7B decode B=32, L=4096 (a --metrics capture)
    "attention_decode": {"bytes": 2_148_306_176 + 7_738_624, "source": "attn_decode.cu",
                         "sha256": "5ec1499e5ac75cd8"},
}


def ncu_traffic(kernel: str):
    """Captured DRAM bytes per launch of `kernel`, or None when its source changed since."""
    import hashlib

    t = NCU_TRAFFIC.get(kernel)
    if not t:
        return None
    src = ROOT / "llama_pre_norm_b200" / "csrc" / t["source"]
    try:
        sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    except OSError:
        return None
    return t["bytes"] if sha == t["sha256"] else None


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=128)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the 13B, 70B-GQA and fp32 tiny prefill lines")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write nvidia-smi clock samples of the timed region to this CSV file")
    return ap.parse_args()


def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ workload accounting
def prefill_flops(cfg) -> dict:
    """Algorithmic FLOPs of one prefill: 2MNK per GEMM, causal attention pairs only."""
    M = cfg.B * cfg.T
    d, f, H, Hkv, dh = cfg.d, cfg.f, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    qkv = 2 * M * (H + 2 * Hkv) * dh * d
    o = 2 * M * d * H * dh
    gu = 2 * M * 2 * f * d
    down = 2 * M * d * f
    pairs = cfg.B * cfg.T * (cfg.T + 1) // 2
    attn = 2 * 2 * pairs * dh * H  # QK^T and PV
    return {"qkv": qkv, "o": o, "gate_up": gu, "down": down, "attn": attn,
            "total": qkv + o + gu + down + attn}


def decode_bytes(cfg, L: int, int8_weights: bool = False) -> int:
    """Algorithmic HBM bytes of one decode step at cache length L (before the step):
    every weight once (bf16, or INT8 codes plus one fp32 scale per output row), K and
    V of L+1 keys per (sequence, KV head), the new K/V written, and the activations
    in and out."""
    es = 2
    d, f, H, Hkv, dh, B = cfg.d, cfg.f, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.B
    n_w = (H + 2 * Hkv) * dh * d + d * H * dh + 3 * d * f
    if int8_weights:
        rows = (H + 2 * Hkv) * dh + d + 2 * f + d
        weights = n_w + 4 * rows + 2 * d * es
    else:
        weights = (n_w + 2 * d) * es
    kv_read = 2 * B * Hkv * (L + 1) * dh * es
    kv_write = 2 * B * Hkv * dh * es
    act = 2 * B * d * es
    return weights + kv_read + kv_write + act


def decode_attn_bytes(cfg, L: int) -> int:
    return 2 * cfg.B * cfg.n_kv_heads * (L + 1) * cfg.head_dim * 2


# ------------------------------------------------------------------ L2 flush
class L2Flush:
    """Evicts L2 outside the timed interval: a write of one buffer larger than L2,
    then a read of another, so that the lines left in L2 when the timed step starts
    are clean lines of unrelated data (the write alone would leave dirty lines whose
    write-back the step's first kernel would pay for)."""

    def __init__(self, nbytes: int, device):
        import torch

        self.w = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.amax()


# ------------------------------------------------------------------ replicas
def reduce_max(v: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank_step: int, steps: int, world: int, slowest_ms: float) -> float:
    """Whole-job throughput of independent replicas: every rank processes the same
    units per step; the job takes as long as its slowest rank."""
    return units_per_rank_step * steps * world / (slowest_ms * 1e-3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons while the timed work runs:
    an NVML thread every 10 ms (read-only queries; the GPU is found by UUID) and,
    when a CSV path is given (--clocks-csv), beside it an nvidia-smi query of the
    same quantities every 200 ms written to that file."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int, csv_path: str | None = None):
        self.cuda_index = cuda_index
        self.csv_path = csv_path
        self.uuid = None
        self.proc = None
        self.samples = []  # (sm_mhz, power_w, reasons bitmask)
        self._stop = None
        self._thread = None
        self.max_mhz = None
        self._entered = False

    def _nvml_loop(self, handle, nv):
        import time as _t
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(handle) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((sm, pw, rs))
            except Exception:
                pass
            _t.sleep(0.01)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            self.uuid = uuid
            handle = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            self._nv = nv
            self._thread = threading.Thread(target=self._nvml_loop, args=(handle, nv), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        if self.csv_path:
            try:
                path = Path(self.csv_path)
                path.parent.mkdir(parents=True, exist_ok=True)
                self.fh = open(path, "a" if self._entered else "w")
                sel = ["-i", self.uuid] if self.uuid else []  # the UUID survives device remapping
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv", "-lms", "200", *sel],
                    stdout=self.fh, stderr=subprocess.DEVNULL)
            except (OSError, FileNotFoundError):
                self.proc = None
        self._entered = True
        time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self._thread:
            self._stop.set()
            self._thread.join(timeout=2)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no NVML samples"]}
        nv = self._nv
        names = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                 "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
                 "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        busy = [x for x in self.samples if not (x[2] & nv.nvmlClocksEventReasonGpuIdle)] or self.samples
        reasons = sorted({n for n, bit in names.items() for x in busy if x[2] & bit})
        sm = sorted(x[0] for x in busy)
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": sm[0], "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "busy_samples": len(busy),
                "power_w_max": max(x[1] for x in self.samples), "source": "NVML 10 ms + nvidia-smi 200 ms"}


# ------------------------------------------------------------------ CPU oracle baseline
def host_info() -> dict:
    """The host CPU the oracle runs on: logical cores, model name (lscpu), and the
    BLAS threads numpy uses (the threads the oracle actually runs on)."""
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.strip().startswith("Model name:"):
                model = line.split(":", 1)[1].strip()
                break
    except (OSError, subprocess.SubprocessError):
        pass
    if model is None:
        try:
            with open("/proc/cpuinfo") as fh:
                for line in fh:
                    if line.startswith("model name"):
                        model = line.split(":", 1)[1].strip()
                        break
        except OSError:
            pass
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        threads = os.cpu_count() or 1
    return {"blas_threads": int(threads), "host_cores": os.cpu_count(), "cpu_model": model}


def cpu_oracle_rows(cfg, W, X, rows) -> dict:
    """Time the fp64 oracle on a row-sampled prefill: K and V projected for every
    token (attention needs them), the query side, attention, o_proj and the MLP at
    the sampled rows of every sequence. Returns the oracle output and the seconds."""
    import numpy as np
    import torch
    from oracle import block as ob

    Wn = {k: np.asarray(v.to(dtype=torch.float64).numpy()) for k, v in W.items()}
    t0 = time.perf_counter()
    ref = ob.block_prefill(X, Wn, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base,
                           rows=rows)
    return {"ref": ref, "seconds": time.perf_counter() - t0}


def cpu_oracle_sample(cfg, W=None, X=None) -> dict:
    """Time the fp64 oracle on the first CPU_SAMPLE_T tokens of the prefill
    workload (a complete causal prefill of that length). Returns tokens/s."""
    import numpy as np
    from oracle import block as ob
    from synth import make_weights, make_x

    host = host_info()
    if W is None:
        W = make_weights(cfg)
    if X is None:
        X = make_x(cfg)
    Xs = X[:, :CPU_SAMPLE_T]
    Wn = {k: np.asarray(v.to(dtype=__import__("torch").float64).numpy()) for k, v in W.items()}
    t0 = time.perf_counter()
    ob.block_prefill(Xs, Wn, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.eps, cfg.rope_base)
    dt = time.perf_counter() - t0
    return {"value": cfg.B * CPU_SAMPLE_T / dt, "unit": UNIT, "cores": host["blas_threads"],
            "host_cores": host["host_cores"], "cpu_model": host["cpu_model"], "kind": "oracle",
            "sample": f"fp64 numpy oracle, full prefill of the first {CPU_SAMPLE_T} tokens of the "
                      f"7B-shaped block (B=1), {dt:.2f} s", "seconds": dt}


# ------------------------------------------------------------------ reference arm
def workload_config(cfg, world: int) -> dict:
    """The `config` object of both arms' JSON lines: the 7B-shaped prefill workload."""
    return {"workload": "llama7b block prefill, bf16, d=4096, 32 heads x 128, f=11008, B=1, T=2048",
            "global_batch": cfg.B * world, "seq_len": cfg.T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (256 MB write, then a 256 MB read)"}


NVLINK_GBS = 770.0  # measured peer copy per direction per GPU on this machine (900 nominal)


def bench_tp_shard(lb, cfg, world: int, args, peaks, dev, stream, flush) -> dict:
    """Per-rank compute of one tensor-parallel prefill layer at `world` ranks ("深入解析Llama
    MLP模块" page §6.3 split): rank 0's shard (n_heads / W query heads, n_kv_heads / W KV
    heads, f / W intermediate columns) runs llama_block_tp_attn_prefill and
    llama_block_tp_mlp on one GPU, L2 flushed before each timed step, CUDA events on the
    library's stream. The two all-reduces of the layer (the attention and MLP partial sums,
    M x d bf16 each) are not run here (one GPU per run); their time is modelled as a ring
    all-reduce at the measured peer-copy bandwidth and reported separately."""
    import torch

    H, Hkv, f = cfg.n_heads // world, cfg.n_kv_heads // world, cfg.f // world
    sc = cfg.with_(name=f"{cfg.name} shard 0/{world}", n_heads=H, n_kv_heads=Hkv, f=f)
    g = torch.Generator(device=dev).manual_seed(1234 + world)
    def rnd(*shape):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    d, dh = cfg.d, cfg.head_dim
    Ws = {"wq": rnd(H * dh, d), "wk": rnd(Hkv * dh, d), "wv": rnd(Hkv * dh, d), "wo": rnd(d, H * dh),
          "w_gate": rnd(f, d), "w_up": rnd(f, d), "w_down": rnd(d, f),
          "g_attn": torch.ones(d, dtype=torch.bfloat16, device=dev),
          "g_mlp": torch.ones(d, dtype=torch.bfloat16, device=dev)}
    blk = lb.LlamaBlock(d, H, Hkv, dh, f, cfg.eps, cfg.rope_base, torch.bfloat16, max_pos=cfg.T)
    blk.set_weights(Ws)
    del Ws
    x = (torch.randn(cfg.B, cfg.T, d, generator=g, device=dev)).to(torch.bfloat16)
    o_part, x1, m_part = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    kc = torch.zeros(cfg.B, Hkv, cfg.T, dh, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device=dev)

    def layer():
        lens.zero_()
        lb.llama_block_tp_attn_prefill(blk.handle, x, o_part, kc, vc, lens, stream=stream)
        # o_part stands in for the all-reduced attention sum (same shape; values only scale X')
        lb.llama_block_tp_mlp(blk.handle, x, o_part, x1, m_part, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            layer()
    blk.sync_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    l0 = blk.launch_count
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            layer()
            ends[i].record(stream)
    torch.cuda.synchronize()
    launches = blk.launch_count - l0
    blk.sync_status()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    fl = prefill_flops(sc)["total"]
    M = cfg.B * cfg.T
    ar_bytes = 2 * M * d * 2  # two all-reduces of an M x d bf16 partial per layer
    wire = ar_bytes * 2 * (world - 1) / world  # ring all-reduce: bytes each rank sends
    ex_ms = wire / (NVLINK_GBS * 1e9) * 1e3
    blk.close()
    return {"world": world, "shard": f"{H} heads / {Hkv} KV heads x {dh}, f={f}",
            "rank_compute_ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "allreduce_bytes_per_layer": ar_bytes,
            "modelled_allreduce_ms": ex_ms,
            "modelled_layer_ms_no_overlap": ms + ex_ms, "kernel_launches": launches}


def bench_prefill_config(lb, cfg, args, peaks, dev, stream, flush, barrier, max_over_ranks,
                         want_cpu: bool) -> dict:
    """Time the prefill of one more workload shape like the headline (own handle, L2
    flushed before every timed step, CUDA events on the library's stream, then a
    second pass with the library's per-stage events) and, on rank 0 of a 1-GPU run,
    the fp64 oracle on 64 sampled rows per sequence beside it (with the GPU output's
    error at those rows)."""
    import torch
    from synth import make_weights, make_x, sample_rows

    W = make_weights(cfg)
    X = make_x(cfg)
    dt = cfg.torch_dtype
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        dt, max_pos=cfg.T)
    blk.set_weights({k: v.to(dev) for k, v in W.items()})
    blk.reserve(cfg.B * cfg.T, cfg.B)
    x = X.to(dev)
    y = torch.empty_like(x)
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, cfg.T, cfg.head_dim, dtype=dt, device=dev)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device=dev)
    for _ in range(args.warmup):
        blk.prefill(x, y, kc, vc, lens)
    blk.sync_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    l0 = blk.launch_count
    barrier()
    for i in range(args.steps):
        flush()
        starts[i].record(stream)
        blk.prefill(x, y, kc, vc, lens)
        ends[i].record(stream)
    barrier()
    launches = blk.launch_count - l0
    blk.sync_status()
    ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends))) / args.steps
    stage_ms: dict = {}
    blk.enable_timing(True)
    barrier()
    for i in range(args.steps):
        flush()
        blk.prefill(x, y, kc, vc, lens)
        for name, t in blk.stage_times():
            stage_ms.setdefault(name, []).append(t)
    barrier()
    blk.enable_timing(False)
    blk.sync_status()
    flops = prefill_flops(cfg)
    tflops = flops["total"] / (ms * 1e-3) / 1e12
    stages = {k: round(statistics.mean(v), 4) for k, v in stage_ms.items()}
    world = int(os.environ.get("WORLD_SIZE", "1"))
    out = {"workload": f"{cfg.name}: {cfg.dtype}, d={cfg.d}, {cfg.n_heads} heads / {cfg.n_kv_heads} KV heads "
                       f"x {cfg.head_dim}, f={cfg.f}, B={cfg.B}, T={cfg.T}",
           "ms_per_step": ms, "tokens_per_s": replica_throughput(cfg.B * cfg.T, 1, world, ms),
           "tflops": tflops, "gflop_per_step": flops["total"] / 1e9, "stage_ms": stages,
           "steps": args.steps, "kernel_launches": launches}
    if cfg.dtype == "bf16":
        out["frac_of_bf16_peak"] = tflops / peaks["bf16_tflops"]
        if peaks.get("bf16_tflops_sustained"):  # the longer steps run under the power cap
            out["frac_of_bf16_sustained_peak"] = tflops / peaks["bf16_tflops_sustained"]
        if "attention" in stages:
            at = flops["attn"] / (stages["attention"] * 1e-3) / 1e12
            out["attention"] = {"ms": stages["attention"], "gflop": flops["attn"] / 1e9, "tflops": at,
                                "frac_of_bf16_peak": at / peaks["bf16_tflops"]}
    if want_cpu:
        import numpy as np

        rows = sample_rows(cfg.T, 64, seed=11)
        c = cpu_oracle_rows(cfg, W, X, rows)
        got = y[:, rows].float().cpu().numpy()
        want = c["ref"]["y"]
        err = float(np.max(np.max(np.abs(got - want), axis=-1) / np.max(np.abs(want), axis=-1)))
        host = host_info()
        out["cpu_oracle"] = {"seconds": c["seconds"], "rows_per_sequence": len(rows),
                             "sampled_rows_per_s": cfg.B * len(rows) / c["seconds"],
                             "cores": host["blas_threads"], "host_cores": host["host_cores"],
                             "cpu_model": host["cpu_model"], "kind": "oracle",
                             "sample": ("fp64 numpy oracle, row-sampled: K/V projected for all "
                                        f"{cfg.B * cfg.T} tokens, query side, attention, o_proj and "
                                        f"MLP at {len(rows)} rows per sequence (first, last, seeded)")}
        out["max_row_err_vs_oracle_at_sampled_rows"] = err
    blk.close()
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synth import LLAMA7B, make_weights, make_x

    cfg = LLAMA7B
    W, X = make_weights(cfg), make_x(cfg)
    for _ in range(args.warmup):
        cpu_oracle_sample(cfg, W, X)
    samples = [cpu_oracle_sample(cfg, W, X) for _ in range(args.steps)]
    secs = sum(s["seconds"] for s in samples)
    value = cfg.B * CPU_SAMPLE_T * args.steps / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": samples[0]["cores"], "kind": "oracle",
                         "host_cores": samples[0]["host_cores"], "cpu_model": samples[0]["cpu_model"],
                         "sample": samples[0]["sample"].rsplit(",", 1)[0]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    import llama_pre_norm_b200 as lb
    from synth import DECODE7B, LLAMA7B, make_weights, make_x

    peaks = measured_peaks()
    cfg = LLAMA7B
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    W = make_weights(cfg)
    X = make_x(cfg)
    Wd = {k: v.to(dev) for k, v in W.items()}
    blk = lb.LlamaBlock(cfg.d, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.f, cfg.eps, cfg.rope_base,
                        torch.bfloat16, max_pos=DECODE7B.cache_len + args.decode_steps + 64)
    blk.set_weights(Wd)
    blk.reserve(cfg.B * cfg.T, DECODE7B.B)
    x = X.to(dev)
    y = torch.empty_like(x)
    kc = torch.zeros(cfg.B, cfg.n_kv_heads, cfg.T, cfg.head_dim, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(cfg.B, dtype=torch.int32, device=dev)
    flush = L2Flush(L2_FLUSH_BYTES, dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dev)

    # ---------------- prefill: warm-up, then K timed steps
    for _ in range(args.warmup):
        blk.prefill(x, y, kc, vc, lens)
    blk.sync_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stage_ms: dict = {}
    csv = args.clocks_csv
    if csv and world > 1:  # one file per rank
        path = Path(csv)
        csv = str(path.with_name(f"{path.stem}_rank{rank}{path.suffix}"))
    clocks = ClockSampler(local, csv)
    with clocks:
        # headline: K steps, nothing between the library's kernels
        launches0 = blk.launch_count
        barrier()
        for i in range(args.steps):
            flush()  # evict L2 outside the timed interval
            starts[i].record(stream)
            blk.prefill(x, y, kc, vc, lens)
            ends[i].record(stream)
        barrier()
        prefill_launches = blk.launch_count - launches0
        step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        blk.sync_status()
        tot_ms = max_over_ranks(sum(step_ms))
        # per-kernel durations: the same K steps again with the library's stage events
        blk.enable_timing(True)
        barrier()
        for i in range(args.steps):
            flush()
            blk.prefill(x, y, kc, vc, lens)
            for name, ms in blk.stage_times():
                stage_ms.setdefault(name, []).append(ms)
        barrier()
        blk.enable_timing(False)
        blk.sync_status()

        # ---------------- decode: B=32, cache 4096 -> 4096 + decode_steps
        dec = None
        if not args.no_decode:
            dcfg = DECODE7B
            t_max = dcfg.cache_len + args.decode_steps
            g = torch.Generator(device=dev).manual_seed(2)
            kcd = torch.zeros(dcfg.B, dcfg.n_kv_heads, t_max, dcfg.head_dim, dtype=torch.bfloat16, device=dev)
            vcd = torch.zeros_like(kcd)
            kcd[:, :, :dcfg.cache_len].normal_(generator=g)
            vcd[:, :, :dcfg.cache_len].normal_(generator=g)
            xs = torch.randn(args.decode_steps, dcfg.B, 1, dcfg.d, generator=g, device=dev).to(torch.bfloat16)
            yd = torch.empty(dcfg.B, 1, dcfg.d, dtype=torch.bfloat16, device=dev)
            dlens = torch.full((dcfg.B,), dcfg.cache_len, dtype=torch.int32, device=dev)

            def reset():
                dlens.fill_(dcfg.cache_len)
                blk.set_lengths([dcfg.cache_len] * dcfg.B)

            reset()
            for s in range(min(args.warmup, args.decode_steps)):
                blk.decode(xs[s], yd, kcd, vcd, dlens)
            blk.sync_status()
            reps = 2
            dec_ms, attn_ms, dec_stage = [], [], {}
            dl0 = blk.launch_count
            barrier()
            for r in range(reps):
                reset()
                blk.enable_timing(r == reps - 1)  # stage timing on the last repetition
                ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ev0.record(stream)
                for s in range(args.decode_steps):
                    blk.decode(xs[s], yd, kcd, vcd, dlens)
                    if r == reps - 1:
                        for name, ms in blk.stage_times():
                            dec_stage.setdefault(name, []).append(ms)
                            if name == "attention":
                                attn_ms.append(ms)
                ev1.record(stream)
                ev1.synchronize()
                dec_ms.append(ev0.elapsed_time(ev1))
            barrier()
            blk.sync_status()
            dec_launches = blk.launch_count - dl0
            blk.enable_timing(False)
            # the untimed-stage repetition is the headline (no events between kernels)
            per_step_ms = max_over_ranks(dec_ms[0]) / args.decode_steps
            Ls = range(dcfg.cache_len, dcfg.cache_len + args.decode_steps)
            bytes_mean = statistics.mean(decode_bytes(dcfg, L) for L in Ls)
            attn_bytes_mean = statistics.mean(decode_attn_bytes(dcfg, L) for L in Ls)
            gbs = bytes_mean / (per_step_ms * 1e-3) / 1e9
            attn_gbs = attn_bytes_mean / (statistics.mean(attn_ms) * 1e-3) / 1e9
            # the same steps with INT8 weight-only projections (one repetition, no stage events)
            blk.quantize_decode_weights(True, stream)
            reset()
            for s in range(min(args.warmup, args.decode_steps)):
                blk.decode(xs[s], yd, kcd, vcd, dlens)
            blk.sync_status()
            reset()
            w8l0 = blk.launch_count
            barrier()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for s in range(args.decode_steps):
                blk.decode(xs[s], yd, kcd, vcd, dlens)
            ev1.record(stream)
            ev1.synchronize()
            barrier()
            blk.sync_status()
            w8_launches = blk.launch_count - w8l0
            blk.quantize_decode_weights(False, stream)
            w8_step_ms = max_over_ranks(ev0.elapsed_time(ev1)) / args.decode_steps
            w8_bytes = statistics.mean(decode_bytes(dcfg, L, int8_weights=True) for L in Ls)
            w8_gbs = w8_bytes / (w8_step_ms * 1e-3) / 1e9
            dec = {
                "workload": f"llama7b decode B={dcfg.B}, cache {dcfg.cache_len} -> {dcfg.cache_len + args.decode_steps}",
                "ms_per_step": per_step_ms, "hbm_gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                "bytes_per_step_mean": bytes_mean, "tokens_per_s": dcfg.B / (per_step_ms * 1e-3) * world,
                "steps": args.decode_steps, "repetitions": reps, "kernel_launches": dec_launches,
                "stage_ms": {k: round(statistics.mean(v), 4) for k, v in dec_stage.items()},
                "attention_kernel": {"ms": statistics.mean(attn_ms), "bytes_mean": attn_bytes_mean,
                                     "achieved_gbs": attn_gbs, "frac": attn_gbs / peaks["hbm_gbs"],
                                     "traffic": ncu_traffic("attention_decode")},
                "int8_weights": {"ms_per_step": w8_step_ms, "hbm_gbs": w8_gbs,
                                 "frac_of_hbm": w8_gbs / peaks["hbm_gbs"], "bytes_per_step_mean": w8_bytes,
                                 "tokens_per_s": dcfg.B / (w8_step_ms * 1e-3) * world,
                                 "speedup_vs_bf16": per_step_ms / w8_step_ms, "kernel_launches": w8_launches},
            }

    # ---------------- e2e: host buffers in and out through the public API, every step's
    # H2D copy of its input and D2H copy of its output inside the timed region. As a
    # serving loop would, the copies run on their own streams and overlap the
    # neighbouring steps: step i+1's input goes up and step i-1's output comes down while
    # step i computes (device inputs and outputs double-buffered).
    xh = X.pin_memory()
    yh = [torch.empty(X.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    flush()
    torch.cuda.synchronize()
    barrier()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(s_in)
    for i in range(args.steps):
        bb = i % 2
        if i >= 2:
            s_in.wait_event(comp_done[bb])  # step i-2 has consumed device input bb
        with torch.cuda.stream(s_in):
            xd[bb].copy_(xh, non_blocking=True)
        in_done[bb].record(s_in)
        stream.wait_event(in_done[bb])
        if i >= 2:
            stream.wait_event(out_done[bb])  # step i-2's output has left device buffer bb
        blk.prefill(xd[bb], yd[bb], kc, vc, lens, stream=stream)
        comp_done[bb].record(stream)
        s_out.wait_event(comp_done[bb])
        with torch.cuda.stream(s_out):
            yh[bb].copy_(yd[bb], non_blocking=True)
        out_done[bb].record(s_out)
    t_end.record(s_out)  # after the last D2H copy (s_out runs in order)
    t_end.synchronize()
    barrier()
    e2e_tot = max_over_ranks(t_start.elapsed_time(t_end))
    blk.sync_status()
    blk.close()
    del xd, yd, kc, vc

    # ---------------- the other prefill shapes (13B batched, 70B GQA, fp32 tiny), each timed
    # like the headline, with the row-sampled CPU oracle beside it
    extra = {}
    if not args.no_extra_configs:
        from synth import LLAMA13B, LLAMA70B, TINY_F32

        want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
        with clocks:
            for key, c in (("prefill_13b", LLAMA13B), ("prefill_70b", LLAMA70B), ("prefill_tiny_f32", TINY_F32)):
                extra[key] = bench_prefill_config(lb, c, args, peaks, dev, stream, flush, barrier,
                                                  max_over_ranks, want_cpu)
                torch.cuda.empty_cache()
            # tensor-parallel shards: one rank's compute of a 7B / 70B prefill layer at W = 2, 4, 8
            if world == 1:
                tp = {"note": "rank 0's compute of one tensor-parallel prefill layer, timed on one GPU; "
                              "the two all-reduces per layer are modelled (ring, 770 GB/s per direction), "
                              "not run: every run here has one GPU"}
                for key, c, one_ms in (("llama7b", cfg, tot_ms / args.steps),
                                       ("llama70b", LLAMA70B, extra["prefill_70b"]["ms_per_step"])):
                    rows = []
                    for Wn in (2, 4, 8):
                        r = bench_tp_shard(lb, c, Wn, args, peaks, dev, stream, flush)
                        r["one_gpu_ms"] = one_ms
                        r["modelled_speedup_vs_1_gpu"] = one_ms / r["modelled_layer_ms_no_overlap"]
                        rows.append(r)
                        torch.cuda.empty_cache()
                    tp[key] = {"workload": f"{c.name}: B={c.B}, T={c.T}", "shards": rows}
                tp["kernel_launches"] = sum(r["kernel_launches"] for k in ("llama7b", "llama70b")
                                            for r in tp[k]["shards"])
                extra["tp_prefill_shards"] = tp
    clk = clocks.summary()

    tokens = cfg.B * cfg.T
    flops = prefill_flops(cfg)
    ms_per_step = tot_ms / args.steps
    value = replica_throughput(tokens, args.steps, world, tot_ms)
    gu_ms = statistics.mean(stage_ms["gate_up_swiglu_gemm"])
    gu_tflops = flops["gate_up"] / (gu_ms * 1e-3) / 1e12
    stages = {k: round(statistics.mean(v), 4) for k, v in stage_ms.items()}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_sample(cfg, W, X)
        cpu = {k: c[k] for k in ("value", "unit", "cores", "host_cores", "cpu_model", "kind", "sample")}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) input)",
        "config": workload_config(cfg, world),
        "prefill": {"tflops": flops["total"] / (ms_per_step * 1e-3) / 1e12,
                    "frac_of_bf16_peak": flops["total"] / (ms_per_step * 1e-3) / 1e12 / peaks["bf16_tflops"],
                    "gflop_per_step": flops["total"] / 1e9, "stage_ms": stages},
        "decode": dec,
        **extra,
        "roofline": {"kernel": "gate_up_swiglu_gemm", "bound": "tensor", "achieved": gu_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": gu_tflops / peaks["bf16_tflops"],
                     "traffic": ncu_traffic("gate_up_swiglu_gemm"),
                     "peak_source": f"{peaks['source']} bf16 burst (kernel timed alone within a short step)",
                     "algorithmic_flop_per_launch": flops["gate_up"]},
        "cpu_baseline": cpu,
        "e2e": {"value": replica_throughput(tokens, args.steps, world, e2e_tot), "unit": UNIT,
                "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": X.numel() * 2,
                "ms_per_step": e2e_tot / args.steps,
                "overlap": "H2D of step i+1 and D2H of step i-1 run on their own streams during step i",
                "path": "pinned host buffers copied by torch (cudaMemcpyAsync on side streams) around the "
                        "device-pointer C-ABI call llama_block_prefill"},
        "gpu_launches": prefill_launches + (dec["kernel_launches"] + dec["int8_weights"]["kernel_launches"]
                                            if dec else 0) + sum(e["kernel_launches"] for e in extra.values()),
        "gpu_launches_note": ("library kernels launched in the timed prefill steps, the timed decode "
                              "repetitions and the timed steps of the other prefill shapes"),
        "clocks": clk,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
