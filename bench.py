"""Benchmark of the AB-Attention hot path on B200: one attention layer of the
Wan2.1-14B-shaped 480p workload (B=1, H=40, 21x30x52 = 32760 tokens, d=128,
query block 128, KV block 16, C=8, 11% of KV blocks kept).

A step is one pass of the whole path: ab_select (IBCS) -> ab_sample (SIP)
-> ab_attention (packed 1/pi-weighted sparse attention) over one layer's
Q, K, V.  Inputs are synthetic (seeded Fourier-feature Q/K, Gaussian V with
outlier tokens) at the workload's shapes; each of Q, K, V is 335 MB, larger
than the 126 MB L2, so no explicit L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--split replicas|heads]

Prints one JSON line (rank 0).  The metric is dense-equivalent attention
TFLOP/s (4 B H L^2 d flop per layer / time per layer; 4 B H L Lk d for the
cross-attention workload, whose keys and values come from a sequence of Lk
tokens).  `--impl reference`
times the CPU oracle (the reference arm of this repository) on a bounded
sample of the same workload on the host cores.

Multi-GPU (one process per GPU): `--split replicas` (default) runs one whole
layer per GPU (weak scaling); `--split heads` divides ONE layer's heads among
the GPUs (ab_forward_slice on each GPU's contiguous slice, strong scaling).
Either way no data crosses between GPUs: every (b, h) is independent on the
path; NCCL carries only the barrier and the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "dense-equivalent attention TFLOPS/s + tensor-pipe util; ms per attention layer"
UNIT = "TFLOP/s"
WORKLOAD_NAMES = {"wan480": "wan2.1-14b-480p-self-attention",
                  "hunyuan720": "hunyuanvideo-720p-self-attention",
                  "wan720": "wan-720p-self-attention",
                  "cross_wan480": "wan2.1-480p-clip-to-9-frame-reference-cross-attention"}


def workload(args):
    """The timed layer: Wan2.1-480p by default; the others (and the KV block /
    keep ratio / C overrides) are for the sweep runs."""
    from block_sparse_attention_queries_b200.synthetic import WORKLOADS
    w = WORKLOADS[getattr(args, "workload", "wan480")]
    kw = {}
    if getattr(args, "heads", None):
        kw["H"] = args.heads
    if getattr(args, "kv_block", None):
        kw["kv_block"] = args.kv_block
    if getattr(args, "keep", None):
        kw["keep_ratio"] = args.keep
    if getattr(args, "clusters", None):
        kw["C"] = args.clusters
    return w.with_(**kw) if kw else w


def dense_flop(w) -> float:
    """4 B H L Lk d: QK^T and PV of dense attention (Lk = L for self-attention)."""
    return 4.0 * w.B * w.H * float(w.L) * float(w.Lk) * w.d


def config_dict(w, extra=None):
    q_mb = w.B * w.H * w.L * w.d * 2 / 1e6
    kv_mb = w.B * w.H * w.Lk * w.d * 2 / 1e6
    c = {"workload": WORKLOAD_NAMES.get(w.name, w.name), "B": w.B, "H": w.H, "grid_txy": list(w.grid), "L": w.L,
         "d": w.d, "q_block": w.q_block, "kv_block": w.kv_block, "C": w.C, "kmeans_iters": w.kmeans_iters,
         "keep_ratio": w.keep_ratio, "sampler_seed": 42, "data_seed": 1234}
    if w.grid_kv is not None:
        c.update({"grid_kv_txy": list(w.grid_kv), "L_kv": w.Lk})
    big = min(q_mb, kv_mb) > 126
    c["l2"] = (f"inputs larger than L2 (Q {q_mb:.0f} MB, K and V {kv_mb:.0f} MB each); no flush" if big
               else f"Q {q_mb:.0f} MB, K and V {kv_mb:.0f} MB each; no flush")
    if extra:
        c.update(extra)
    return c


def peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk["hbm_gbs"]), "measured (burst)"
    except Exception:
        return 1590.0, 6650.0, "fallback"


# DRAM traffic of one sparse attention launch, from the ncu capture of the
# 8-head case of the Wan2.1-480p layer (dram__bytes_read.sum +
# dram__bytes_write.sum = 206.222 MB + 53.658 MB, kv_block 16, 11 % kept;
# summarised under profiles/), scaled to the layer's heads (the launch's
# traffic grows with the heads).  It describes the kernel sources it
# was measured on only: with any other sources (hash below) the bench reports
# null.
ATTN_TRAFFIC = {"sources_sha256_16": "91ae4471fe2799dc", "bytes_per_head": (206.221568e6 + 53.658368e6) / 8,
                "workload": "wan480", "kv_block": 16, "keep_ratio": 0.11}


def attention_traffic(w):
    import hashlib
    h = hashlib.sha256()
    for f in ("ab_attention.cuh", "ab_ptx.cuh"):
        with open(os.path.join(HERE, "block_sparse_attention_queries_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    t = ATTN_TRAFFIC
    if (h.hexdigest()[:16] != t["sources_sha256_16"] or w.name != t["workload"] or w.kv_block != t["kv_block"]
            or abs(w.keep_ratio - t["keep_ratio"]) > 1e-9):
        return None
    return round(t["bytes_per_head"] * w.B * w.H)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clocks, power and clock-event reasons sampled during the timed region.

    Reads NVML (read-only queries) from a background thread every 50 ms; if
    NVML is unusable it falls back to `nvidia-smi -lms`.  `stop()` returns the
    summary, or {"error": ...} saying why no sample was taken."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []
        self.error = None
        self._stop = None
        self._thread = None
        self._smi = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        uuid = str(getattr(props, "uuid", "") or "")
        if uuid:
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.lower().endswith(uuid.lower()):
                    return pynvml, h
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, mx, pw, rs))
                    except Exception as e:  # keep sampling; report the last failure
                        self.error = f"nvml: {e}"
                    self._stop.wait(0.05)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            self._nv = nv
        except Exception as e:
            self.error = f"nvml unavailable: {e}"
            self._start_smi()

    def _start_smi(self):
        import tempfile
        fd, self._smi_path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        try:
            self._smi = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self._smi_path, "w"), stderr=subprocess.DEVNULL)
        except Exception as e:
            self.error = f"{self.error}; nvidia-smi: {e}"

    def wait_first_sample(self, timeout_s: float = 5.0):
        t = time.time()
        while time.time() - t < timeout_s:
            if self.samples or (self._smi is not None and os.path.getsize(self._smi_path) > 0):
                return
            if self._thread is None and self._smi is None:
                return
            time.sleep(0.02)

    def stop(self):
        rows = []
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
            nv = self._nv
            for sm, mx, pw, rs in self.samples:
                rows.append((float(sm), float(mx), float(pw),
                             [name for name, attr in self.REASONS if rs & getattr(nv, attr, 0)]))
        elif self._smi is not None:
            self._smi.terminate()
            try:
                self._smi.wait(timeout=5)
            except Exception:
                self._smi.kill()
            names = [n for n, _ in self.REASONS[:4]]
            with open(self._smi_path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    try:
                        rows.append((float(parts[0]), float(parts[1]), float(parts[2]),
                                     [names[k] for k in range(4) if parts[3 + k].lower().startswith("active")]))
                    except (ValueError, IndexError):
                        continue
            os.unlink(self._smi_path)
        if not rows:
            return {"error": self.error or "no samples in the timed region"}
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_median": round(statistics.median(r[2] for r in rows), 1),
                "reasons": sorted({x for r in rows for x in r[3]}), "samples": len(rows),
                "source": "nvml" if self._thread is not None else "nvidia-smi"}


# ------------------------------------------------------- ranks (host logic)

def dist_env(gpus: int):
    """(rank, world, local rank) from the launcher's environment; one process
    per GPU, so --gpus must equal WORLD_SIZE when more than one rank runs."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and gpus != world:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE {world}")
    if not 0 <= rank < world:
        raise SystemExit(f"RANK {rank} outside WORLD_SIZE {world}")
    return rank, world, local


def rank_data_seed(rank: int) -> int:
    """Each rank runs its own layer: the synthetic inputs are seeded per rank."""
    return 1234 + rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank calls this at the same point)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def executed_flop(w, cnt, idx) -> float:
    """Algorithmic flop of the sparse attention on given lists:
    4 d sum_{b,h,i} n_i sum_{j in S_i} n_j (n_j < kv_block only for the last,
    partial KV block)."""
    cnt = np.asarray(cnt, np.int64)
    n_i = np.array([min(w.q_block, w.L - i * w.q_block) for i in range(w.Nq)], np.int64)
    flop = 4.0 * w.d * float((n_i[None, None, :] * cnt * w.kv_block).sum())
    n_last = w.Lk - (w.Nkv - 1) * w.kv_block
    if n_last < w.kv_block:
        # rows whose list holds the last KV block (lists are ascending: it is the last entry)
        pos = np.maximum(cnt - 1, 0)
        last = np.take_along_axis(np.asarray(idx), pos[..., None], axis=-1)[..., 0]
        has = (cnt > 0) & (last == w.Nkv - 1)
        flop -= 4.0 * w.d * float((n_i[None, None, :] * has * (w.kv_block - n_last)).sum())
    return flop


def tile_flop(w, cnt) -> float:
    """Tensor-core work of the sparse attention as executed: every query block
    runs ceil(count / (128 / kv_block)) tiles of 128 keys, each an S product
    and a P V product of 128 x 128 x d (the padding of a list's last tile and
    of a ragged last query block included): 4 * 128 * 128 * d flop per tile."""
    slots = 128 // w.kv_block
    tiles = (np.asarray(cnt, np.int64) + slots - 1) // slots
    return 4.0 * 128 * 128 * w.d * float(tiles.sum())


# Bytes one SM's TMA unit brings into shared memory per clock at most: a
# probe issuing back-to-back 32 KB tile loads into one SM (any grid size)
# measured 32 B per clock (about 48 cycles per box + 32 B per clock; 30 B at
# 16 KB boxes, 23 B at 4 KB boxes issued one at a time).
TMA_INGRESS_B_PER_CLK_SM = 32.0
NUM_SMS = 148


def ingress_bytes(w, cnt) -> float:
    """Bytes the sparse attention kernel brings into shared memory per
    launch: the two query blocks' Q tiles of every CTA and, per tile of
    128 keys, one K and one V tile (128 rows x d bf16 each, list padding
    included)."""
    slots = 128 // w.kv_block
    tiles = (np.asarray(cnt, np.int64) + slots - 1) // slots
    tile_bytes = 128 * w.d * 2
    return float(tiles.sum()) * 2 * tile_bytes + w.B * w.H * w.Nq * tile_bytes


def whole_job_value(w, world: int, ms_step: float) -> float:
    """Dense-equivalent TFLOP/s of the whole job: every rank processes one layer per step."""
    return dense_flop(w) * world / (ms_step * 1e-3) / 1e12


# ----------------------------------------------------------- our arm (GPU)

def run_ours(args):
    import torch
    import torch.distributed as dist
    import block_sparse_attention_queries_b200 as ab
    from block_sparse_attention_queries_b200.synthetic import make_workload_qkv

    rank, world, local = dist_env(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", rank=rank, world_size=world, device_id=dev,
                                timeout=datetime.timedelta(seconds=120))

    w = workload(args)
    p = ab.Params.of(w, seed=42)
    # weak scaling: every rank runs its own layer (independent batch element)
    Qc, Kc, Vc = make_workload_qkv(w, seed=rank_data_seed(rank))
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    bufs = ab.Buffers(p, dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        _select(ab, p, Q, K, bufs)
        if ev is not None:
            ev[1].record(stream)
        _sample(ab, p, bufs)
        if ev is not None:
            ev[2].record(stream)
        ab.ab_attention(p, Q, K, V, bufs.idx, bufs.pi_q32, bufs.count, out=bufs.O)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    barrier()
    code = ab.device_error(dev)
    if code:
        raise SystemExit(f"device error during warm-up: {ab.status_string(code)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()  # nvidia-smi needs a moment before its first sample
    clocks.wait_first_sample()
    barrier()
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    sel_ms = [e[0].elapsed_time(e[1]) for e in evs]
    smp_ms = [e[1].elapsed_time(e[2]) for e in evs]
    att_ms = [e[2].elapsed_time(e[3]) for e in evs]
    code = ab.device_error(dev)
    if code:
        raise SystemExit(f"device error in the timed region: {ab.status_string(code)}")

    cnt = bufs.count.cpu().numpy()
    exec_flop = executed_flop(w, cnt, bufs.idx.cpu().numpy())
    tiles_flop = tile_flop(w, cnt)
    kept_frac = float(cnt.sum()) / (w.B * w.H * w.Nq * w.Nkv)

    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / args.steps
    value = whole_job_value(w, world, ms_step)
    att_avg = statistics.mean(att_ms)
    bf16_peak, hbm_peak, peak_kind = peaks()
    achieved = exec_flop / (att_avg * 1e-3) / 1e12

    # e2e through the public C ABI with host buffers (copies inside the region), on every rank
    e2e = None if args.no_extras else run_e2e(ab, p, w, Qc, Kc, Vc, bufs, dev, max(2, min(args.steps, 5)),
                                              world, barrier)
    out = None
    if rank == 0:
        if args.no_extras:
            dense_ms, cpu, qual = float("nan"), None, None
        else:
            dense_ms = run_dense(ab, p, Q, K, V, dev, 3)
            qual = quality(ab, p, Q, K, V, bufs, dev)
            qual["ms_select_sample_fused"] = time_fused_select_sample(ab, p, Q, K, dev)
            qual.update(mass_found(w, Q, K, bufs.P, ab.budget(p)))
            qual["concentrated"] = quality_concentrated(ab, w, dev)
            cpu = cpu_baseline(w, args, Qc, Kc, Vc)
        out = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(w, {"parallelism": f"dp{world} (independent layers per GPU)"}),
            "ms_per_layer": round(ms_step, 4),
            "ms_select": round(statistics.mean(sel_ms), 4), "ms_sample": round(statistics.mean(smp_ms), 4),
            "ms_attention": round(att_avg, 4),
            "executed_tflops_attention": round(achieved, 2),
            "tile_tflops_attention": round(tiles_flop / (att_avg * 1e-3) / 1e12, 2),
            "tile_frac_of_peak": round(tiles_flop / (att_avg * 1e-3) / 1e12 / bf16_peak, 4),
            "kept_block_fraction": round(kept_frac, 5),
            "dense_kernel_ms": round(dense_ms, 3),
            "speedup_vs_own_dense_kernel": round(dense_ms / ms_step, 3),
            "gpu_launches": 5 * args.steps,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                         "frac": round(achieved / bf16_peak, 4), "traffic": attention_traffic(w),
                         "traffic_note": "ncu dram bytes of the 8-head capture x H/8 (profiles/)",
                         "kernel": "ab_attention_kernel<128,16>", "peak_kind": peak_kind,
                         "per_launch_flop": exec_flop},
            "ingress": ingress_roofline(w, cnt, att_avg, clk),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk,
            "quality": qual,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


def run_ours_split(args):
    """One layer per step, its heads divided among the ranks (ab_forward_slice
    on every rank's contiguous slice of the B*H heads); the step time is the
    slowest rank's and the value the layer's dense-equivalent rate."""
    import torch
    import torch.distributed as dist
    import block_sparse_attention_queries_b200 as ab
    from block_sparse_attention_queries_b200.synthetic import make_workload_qkv

    rank, world, local = dist_env(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", rank=rank, world_size=world, device_id=dev,
                                timeout=datetime.timedelta(seconds=120))
    w = workload(args)
    p = ab.Params.of(w, seed=42)
    bh0, nbh = ab.head_slices(w.B, w.H, world)[rank]
    Qc, Kc, Vc = make_workload_qkv(w)  # the whole layer, the same on every rank; each keeps its slice
    Qs, Ks, Vs = (t.reshape(1, w.B * w.H, *t.shape[2:])[:, bh0:bh0 + nbh].contiguous() for t in (Qc, Kc, Vc))
    Q, K, V = (t.to(dev) for t in (Qs, Ks, Vs))
    bufs = ab.Buffers(ab.slice_params(p, nbh), dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        ab.ab_forward_slice(p, bh0, nbh, Q, K, V, bufs)
    barrier()
    code = ab.device_error(dev)
    if code:
        raise SystemExit(f"device error during warm-up: {ab.status_string(code)}")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    clocks.wait_first_sample()
    barrier()
    t0.record(stream)
    for _ in range(args.steps):
        ab.ab_forward_slice(p, bh0, nbh, Q, K, V, bufs)
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    code = ab.device_error(dev)
    if code:
        raise SystemExit(f"device error in the timed region: {ab.status_string(code)}")
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)

    # end to end: each rank copies its slice in from pinned host memory, runs
    # it, and copies its output back; the layer's bytes, the slowest rank's time
    e2e = None
    if not args.no_extras:
        Qh, Kh, Vh = (t.pin_memory() for t in (Qs, Ks, Vs))
        Oh = torch.empty_like(Qs).pin_memory()
        steps = max(2, min(args.steps, 5))
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            Q.copy_(Qh, non_blocking=True)
            K.copy_(Kh, non_blocking=True)
            V.copy_(Vh, non_blocking=True)
            ab.ab_forward_slice(p, bh0, nbh, Q, K, V, bufs)
            Oh.copy_(bufs.O, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
        full = [t.numel() * t.element_size() for t in (Qc, Kc, Vc)]
        e2e = {"value": round(dense_flop(w) / (ems * 1e-3) / 1e12, 3), "unit": UNIT,
               "h2d_bytes_per_step": sum(full), "d2h_bytes_per_step": full[0], "ms_per_step": round(ems, 3),
               "api": "ab_forward_slice with the slice's copies from pinned host memory on every rank"}
    out = None
    if rank == 0:
        out = {"metric": METRIC, "value": round(dense_flop(w) / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
               "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic",
               "config": config_dict(w, {"parallelism": f"heads split over {world} GPUs "
                                                        f"({[n for _, n in ab.head_slices(w.B, w.H, world)]} heads)"}),
               "ms_per_layer": round(ms, 4), "gpu_launches": 5 * args.steps, "e2e": e2e, "clocks": clk}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


def _select(ab, p, Q, K, bufs):
    import ctypes
    lib = ab.lib()
    st = ab._stream(Q.device)
    ab._check(lib.ab_select(ctypes.byref(p.c()), ab._ptr(Q), ab._ptr(K), ab._ptr(bufs.P), None, None,
                            ab._ptr(bufs.ws), bufs.ws.numel(), st), "ab_select")


def _sample(ab, p, bufs):
    import ctypes
    lib = ab.lib()
    st = ab._stream(bufs.P.device)
    ab._check(lib.ab_sample(ctypes.byref(p.c()), ab._ptr(bufs.P), ab._ptr(bufs.idx), ab._ptr(bufs.pi_q32),
                            ab._ptr(bufs.count), st), "ab_sample")


def run_e2e(ab, p, w, Qc, Kc, Vc, bufs, dev, steps, world=1, barrier=None):
    """The same metric through the public host-buffer call, every rank on its
    own layer; the time is the slowest rank's, the bytes the whole job's."""
    import torch
    Qh, Kh, Vh = (t.pin_memory() for t in (Qc, Kc, Vc))
    Oh = torch.empty_like(Qc).pin_memory()
    Qd, Kd, Vd = (torch.empty_like(t, device=dev) for t in (Qc, Kc, Vc))
    stream = torch.cuda.current_stream(dev)
    ab.ab_forward_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs, dev)  # warm-up
    if barrier is not None:
        barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        ab.ab_forward_host(p, Qh, Kh, Vh, Oh, Qd, Kd, Vd, bufs, dev)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (Qh, Kh, Vh))
    d2h = Oh.numel() * Oh.element_size()
    return {"value": round(whole_job_value(w, world, ms), 3), "unit": UNIT,
            "h2d_bytes_per_step": world * h2d, "d2h_bytes_per_step": world * d2h, "ms_per_step": round(ms, 3),
            "api": "ab_forward_host (pinned host Q/K/V in, host O out)"}


def run_dense(ab, p, Q, K, V, dev, iters):
    import torch
    O = torch.empty_like(Q)
    ab.ab_attention_dense(p, Q, K, V, out=O)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(iters):
        ab.ab_attention_dense(p, Q, K, V, out=O)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / iters


def quality(ab, p, Q, K, V, bufs, dev):
    """Information only (no value on the pages pins it): relative L2 distance
    to dense attention of the SIP output (bufs.O) and of truncation at the same
    budget (top-Kb blocks of the same P, pi = 1), plus the truncation
    selection's time."""
    import torch
    Od = torch.empty_like(Q)
    ab.ab_attention_dense(p, Q, K, V, out=Od)
    # the selections are timed into preallocated lists (no allocation in the timed loops)
    idx, piq, cnt = ab.ab_sample_topk(p, bufs.P)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(3):
        ab.ab_sample_topk(p, bufs.P, out=(idx, piq, cnt))
    t1.record(stream)
    Ot = ab.ab_attention(p, Q, K, V, idx, piq, cnt)
    sidx, spiq, scnt = ab.ab_sample_systematic(p, bufs.P)
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    for _ in range(3):
        ab.ab_sample_systematic(p, bufs.P, out=(sidx, spiq, scnt))
    t3.record(stream)
    Os = ab.ab_attention(p, Q, K, V, sidx, spiq, scnt)
    torch.cuda.synchronize(dev)
    ref = torch.linalg.vector_norm(Od.double())

    def rel(o):
        return round(float(torch.linalg.vector_norm(o.double() - Od.double()) / ref), 5)

    return {"rel_l2_sip_vs_dense": rel(bufs.O), "rel_l2_systematic_vs_dense": rel(Os),
            "rel_l2_truncation_vs_dense": rel(Ot),
            "ms_sample_systematic": round(t2.elapsed_time(t3) / 3, 4),
            "ms_sample_truncation": round(t0.elapsed_time(t1) / 3, 4),
            "note": "same P and budget; information only, not a gate"}


def ingress_roofline(w, cnt, att_ms, clk):
    """Second roofline of the attention kernel: bytes its TMA loads bring into
    each SM's shared memory per SM clock (the median SM clock sampled during
    the timed region) against the probe's 32 B per clock."""
    mhz = clk.get("sm_mhz") if isinstance(clk, dict) else None
    b = ingress_bytes(w, cnt)
    if not mhz:
        return {"bytes_per_launch": b, "achieved": None, "note": "no SM clock sample"}
    per_clk = b / (att_ms * 1e-3 * mhz * 1e6 * NUM_SMS)
    return {"bound": "tma_ingress", "achieved": round(per_clk, 2), "peak": TMA_INGRESS_B_PER_CLK_SM,
            "unit": "B/clk per SM", "frac": round(per_clk / TMA_INGRESS_B_PER_CLK_SM, 4), "bytes_per_launch": b,
            "sm_mhz": mhz, "peak_kind": "probe (TMA tile loads into one SM, not driver-measured)"}


def time_fused_select_sample(ab, p, Q, K, dev, iters=3):
    """ab_select_sample (scoring that samples the rows it scores) on the same
    inputs, into preallocated outputs: information beside ms_select + ms_sample."""
    import torch
    ws = ab.alloc_workspace(p, dev)
    out = ab.ab_select_sample(p, Q, K, workspace=ws)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(iters):
        ab.ab_select_sample(p, Q, K, workspace=ws, out=out)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return round(t0.elapsed_time(t1) / iters, 4)


def mass_found(w, Q, K, P, Kb, heads=(0, 1, 2, 3), blocks=4):
    """Information only: on sampled query blocks, the share of the block's
    attention mass (dense softmax of its queries, averaged over its rows,
    summed per KV block) held by the Kb blocks with the largest P (what the
    IBCS estimate finds) and by the Kb blocks with the largest true mass (the
    ideal top-Kb).  A diagnostic computed with plain torch ops on the GPU,
    outside the timed path."""
    import math
    import torch
    found, ideal = [], []
    for h in heads:
        for i in sorted({int(round(k * (w.Nq - 1) / max(1, blocks - 1))) for k in range(blocks)}):
            q = Q[0, h, i * w.q_block:(i + 1) * w.q_block].float()
            logits = (q @ K[0, h].float().T) / math.sqrt(w.d)
            prob = torch.softmax(logits, dim=-1).mean(0)                       # [Lk]
            pad = w.Nkv * w.kv_block - prob.numel()
            mass = torch.nn.functional.pad(prob, (0, pad)).view(w.Nkv, w.kv_block).sum(1).double()
            sel = torch.topk(P[0, h, i].double(), Kb).indices
            found.append(float(mass[sel].sum()))
            ideal.append(float(torch.topk(mass, Kb).values.sum()))
    return {"mass_found_by_P_topKb": round(sum(found) / len(found), 4),
            "mass_ideal_topKb": round(sum(ideal) / len(ideal), 4), "query_blocks_sampled": len(found)}


def quality_concentrated(ab, w, dev, heads=8, s_peak=32.0):
    """Information only: the relative L2 distance to dense attention of SIP,
    systematic sampling and truncation at the same budget when attention is
    concentrated (inputs drawn with s_peak = 32 instead of 8, so that q.k /
    sqrt(d) of two tokens at the same position is about 32: a few blocks hold
    most of each row's weight), on the first `heads` heads of the workload."""
    import torch
    from block_sparse_attention_queries_b200.synthetic import make_cross_qkv, make_qkv
    wc = w.with_(H=min(heads, w.H))
    p = ab.Params.of(wc, seed=42)
    if wc.grid_kv is not None:
        Qc, Kc, Vc = make_cross_qkv(wc.B, wc.H, wc.grid, wc.grid_kv, wc.d, wc.F, s_peak=s_peak)
    else:
        Qc, Kc, Vc = make_qkv(wc.B, wc.H, wc.grid, wc.d, wc.F, s_peak=s_peak)
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    b = ab.ab_forward(p, Q, K, V)
    Od = ab.ab_attention_dense(p, Q, K, V)
    Ot = ab.ab_attention(p, Q, K, V, *ab.ab_sample_topk(p, b.P))
    Os = ab.ab_attention(p, Q, K, V, *ab.ab_sample_systematic(p, b.P))
    torch.cuda.synchronize(dev)
    ref = torch.linalg.vector_norm(Od.double())

    def rel(o):
        return round(float(torch.linalg.vector_norm(o.double() - Od.double()) / ref), 5)

    out = {"s_peak": s_peak, "heads": wc.H, "rel_l2_sip_vs_dense": rel(b.O),
           "rel_l2_systematic_vs_dense": rel(Os), "rel_l2_truncation_vs_dense": rel(Ot),
           "kept_block_fraction": round(float(b.count.sum()) / (wc.B * wc.H * wc.Nq * wc.Nkv), 5)}
    out.update(mass_found(wc, Q, K, b.P, ab.budget(p)))
    return out


# ---------------------------------------------------------- CPU oracle arm

def cpu_sample_units(w, n_heads=4, n_blocks=16):
    heads = sorted({int(round(k * (w.H - 1) / max(1, n_heads - 1))) for k in range(n_heads)})
    blocks = sorted({int(round(k * (w.Nq - 1) / max(1, n_blocks - 1))) for k in range(n_blocks)})
    return [(h, i) for h in heads for i in blocks]


def cpu_baseline(w, args, Qc=None, Kc=None, Vc=None):
    """The oracle, as it stands, on the host cores: IBCS + SIP + reweighted
    attention for a bounded sample of (head, query block) units of the
    workload, extrapolated to one layer."""
    import oracle
    from block_sparse_attention_queries_b200.synthetic import make_qkv
    units = cpu_sample_units(w)
    heads = sorted({h for h, _ in units})
    # inputs of the sampled heads only (same generator, same seed)
    if Qc is None:
        from block_sparse_attention_queries_b200.synthetic import make_workload_qkv
        Qc, Kc, Vc = make_workload_qkv(w)
    Qn = {h: Qc[0, h].float().numpy() for h in heads}
    Kn = {h: Kc[0, h].float().numpy() for h in heads}
    Vn = {h: Vc[0, h].float().numpy() for h in heads}
    Kb = oracle.budget(w.Nkv, w.keep_ratio)
    threads = os.cpu_count() or 1

    def one(u):
        h, i = u
        P = oracle.select_head(Qn[h], Kn[h], w.q_block, w.kv_block, w.C, w.kmeans_iters, rows=[i])
        idx, pq, n = oracle.sip_row(P[0].astype(np.float32), Kb, 42, 0, h, i)
        oracle.ht_attention_block(Qn[h], Kn[h], Vn[h], w.q_block, w.kv_block, i, idx, pq, n)
        return n

    t = time.perf_counter()
    oracle.run_units(one, units, threads)
    wall = time.perf_counter() - t
    total_units = w.B * w.H * w.Nq
    ms_layer = wall * 1e3 * total_units / len(units)
    return {"value": round(dense_flop(w) / (ms_layer * 1e-3) / 1e12, 6), "unit": UNIT,
            "cores": threads, "kind": "oracle",
            "sample": f"{len(units)} (head, query block) units of {total_units} (heads {heads}), "
                      f"select+sample+attention, {wall:.2f} s wall on {threads} threads; "
                      f"ms/layer extrapolated = wall x {total_units}/{len(units)}",
            "ms_per_layer_extrapolated": round(ms_layer, 1)}


def run_reference(args):
    rank, _, _ = dist_env(args.gpus)
    if rank != 0:
        return None  # the oracle runs once, on rank 0; the other ranks exit without work
    from block_sparse_attention_queries_b200.synthetic import make_workload_qkv
    w = workload(args)
    Qc, Kc, Vc = make_workload_qkv(w)
    for _ in range(args.warmup):  # untimed warm-up steps
        cpu_baseline(w, args, Qc, Kc, Vc)
    vals, walls = [], []
    last = None
    for _ in range(args.steps):
        t = time.perf_counter()
        last = cpu_baseline(w, args, Qc, Kc, Vc)
        walls.append(time.perf_counter() - t)
        vals.append(last["ms_per_layer_extrapolated"])
    ms = statistics.mean(vals)
    value = dense_flop(w) / (ms * 1e-3) / 1e12
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1),
            "ms_per_step_kind": "extrapolated from the sampled units (wall x units per layer / sampled units)",
            "ms_per_step_measured_wall": round(statistics.mean(walls) * 1e3, 1),
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_dict(w, {"parallelism": "host threads"}),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--heads", type=int, default=None,
                    help="run a smaller case of the same layer with this many heads (profiling only)")
    ap.add_argument("--workload", choices=["wan480", "hunyuan720", "wan720", "cross_wan480"], default="wan480",
                    help="layer shape (default: the Wan2.1-480p headline workload)")
    ap.add_argument("--kv-block", type=int, default=None, help="KV block size override (sweeps)")
    ap.add_argument("--keep", type=float, default=None, help="keep ratio override (sweeps)")
    ap.add_argument("--clusters", type=int, default=None, help="cluster count C override (sweeps)")
    ap.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                    help="multi-GPU: one layer per GPU (replicas) or one layer's heads divided among the GPUs")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the end-to-end, dense and CPU-baseline legs (profiling only)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        out = run_reference(args)
    elif args.split == "heads":
        out = run_ours_split(args)
    else:
        out = run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
