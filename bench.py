#!/usr/bin/env python
"""Benchmark: VideoMLA latent-KV chunk attention on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 480p]

One step = one pass of the hot path over one chunk of the 480P workload
(Wan2.1-1.3B shape: 30 x 52 patches per frame, a chunk of 3 frames = 4680
queries, a 21-frame window = 32760 keys, 12 heads x 128, d_c = 192, d_r = 32):
    vmla_cache_append     the chunk's 4680 tokens -> [c ; RoPE3D(k_r)] rows of the window
    vmla_chunk_attention  4680 queries x 12 heads over the 32760 cached keys
Inputs are seeded synthetic data (see the `workload` package) already resident in
HBM when the timed region starts.  L2 is flushed before every timed step: a 256 MiB
write evicts every cached line, then a 256 MiB read of a second buffer forces the
write-back of those dirty lines, so the timed step starts from a cold, clean L2.
`value` counts the absorbed-MLA tensor FLOPs of the attention,
2*B*Nq*H*Nkv*(224+192), plus the append's 2*B*Nq*224*1536, per second.  The dense
per-head baseline (3072 scalars/token) is timed on the same queries beside it.

Under torchrun (N > 1) every rank runs an independent replica on its own seed
(no data-path collective); the time is the max over ranks and `value` the work of
all ranks over that time.  --impl reference times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workload  # noqa: E402

METRIC = "MLA chunk-attention TFLOP/s & ms/chunk (Wan-1.3B 480P shape); % BF16 peak"
UNIT = "TFLOP/s"
SCALE = 160 ** -0.5
FLUSH_BYTES = 256 << 20
PROFILED_TRAFFIC = os.path.join(ROOT, "profiles", "chunk_attn_480p_traffic.json")
ATTN_SOURCES = [os.path.join(ROOT, "latent_kv_cache_b200", "csrc", f)
                for f in ("attention.cu", "sm100.cuh", "common.cuh")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="480p", choices=sorted(workload.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chunk", action="store_true",
                    help="skip the per-chunk schedule and the batch-8 / 1080P figures of the 480P run")
    ap.add_argument("--chunk-replays", type=int, default=7, help="timed chunk replays per schedule")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def workload_desc(w) -> dict:
    return {
        "workload": (f"{w.name}: B={w.batch}, {w.grid_h}x{w.grid_w} patches/frame, chunk {w.chunk_frames} "
                     f"frames = {w.n_q} queries, window {w.window_frames} frames = {w.n_kv} keys "
                     f"({w.cached_frames} cached + chunk), H={w.heads}x{w.d_head}, d_c={w.d_c}, d_r={w.d_r}"),
        "batch": w.batch, "n_q": w.n_q, "n_kv": w.n_kv, "heads": w.heads, "d_c": w.d_c, "d_r": w.d_r,
        "step": "cache_append(chunk) + chunk_attention(window)",
        "l2": "flushed before every timed step (256 MiB write, then 256 MiB read of another buffer)",
        "flops_convention": "absorbed MLA: 2*B*Nq*H*Nkv*(d_c+d_r+d_c) + append 2*B*Nq*224*1536",
    }


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0.0)), float(d["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for p in ATTN_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name: str):
    """DRAM bytes per launch of the attention kernel: a profiled constant (one ncu
    capture, kept with the source hash it was taken at), or None if the record is
    missing, covers another workload, or the kernel source changed since."""
    try:
        with open(PROFILED_TRAFFIC) as f:
            rec = json.load(f)
        if rec.get("source_sha256_16") != attn_source_hash() or rec.get("workload") != workload_name:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# Multi-rank accounting (replicas: no data-path collective, only the timing)
# ---------------------------------------------------------------------------
def max_over_ranks(v: float, dist=None, device=None) -> float:
    """Max of a per-rank time over all ranks (identity on one rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(v)
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, flops_per_step: float, total_ms: float) -> float:
    """Whole-job throughput (TFLOP/s): the work of all ranks over the slowest rank's time."""
    return world * steps * flops_per_step / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# Clock sampling during the timed region (NVML; falls back to nvidia-smi)
# ---------------------------------------------------------------------------
_REASONS = [(0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
            (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
            (0x2, "applications_clocks_setting"), (0x10, "sync_boost")]


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._period = period_s
        self._dev = device_index
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _reasons_now(self):
        n = self._nvml
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(n, fn):
                try:
                    return int(getattr(n, fn)(self._h))
                except Exception:
                    pass
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                self.reasons |= self._reasons_now()
            except Exception:
                pass
            time.sleep(self._period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self) -> dict:
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [name for bit, name in _REASONS if self.reasons & bit]}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle as it stands, on a bounded sample of the workload
# ---------------------------------------------------------------------------
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max(int(d.get("num_threads", 1)) for d in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_step(w, act, wts, cache_bits, rows, n_tok):
    """One bounded oracle step: append of n_tok chunk tokens + attention of `rows` queries."""
    import oracle
    x_tok = act["x"][:, w.n_cached:w.n_cached + n_tok]
    t0 = time.perf_counter()
    oracle.cache_append(x_tok, wts["w_dkv"], wts["w_kr"], w.chunk_t0, w.grid_h, w.grid_w)
    oracle.chunk_attention(act["q"], act["q_rope"], wts["w_uk"], wts["w_uv"], cache_bits, w.n_kv,
                           w.chunk_t0, w.grid_h, w.grid_w, SCALE, rows=rows)
    dt = time.perf_counter() - t0
    flops = (w.attention_flops() * len(rows) / w.n_q + w.append_flops(n_tok))
    return dt, flops


def oracle_prepare(w, act, wts):
    import oracle
    return oracle.cache_append(act["x"], wts["w_dkv"], wts["w_kr"], 0, w.grid_h, w.grid_w)


def size_oracle_sample(w, act, wts, cache_bits, target_s):
    """Rows/tokens of one oracle step taking about target_s seconds.  Two short
    calibration runs separate the per-call cost (the oracle forms every key's
    per-head K/V whatever the number of query rows) from the per-row cost."""
    def run(n):
        rows = np.linspace(0, w.n_q - 1, n).astype(np.int64)
        return oracle_sample_step(w, act, wts, cache_bits, rows, 2 * n)[0]
    lo, hi = min(64, w.n_q), min(256, w.n_q)
    d_lo, d_hi = run(lo), run(hi)
    per_row = max((d_hi - d_lo) / max(hi - lo, 1), 1e-6)
    fixed = max(d_lo - lo * per_row, 0.0)
    n_rows = int(min(w.n_q, max(8, (target_s - fixed) / per_row)))
    n_tok = int(min(w.n_q, max(32, 2 * n_rows)))
    return np.linspace(0, w.n_q - 1, n_rows).astype(np.int64), n_tok


def dense_oracle_sample(w, kv, act, n_rows):
    """The fp64 dense per-head oracle on n_rows query rows: seconds and TFLOP/s (2 x 2 x d per score)."""
    import oracle
    rows = np.linspace(0, w.n_q - 1, n_rows).astype(np.int64)
    t0 = time.perf_counter()
    oracle.dense_attention(act["q"], kv["k"], kv["v"], SCALE, rows=rows)
    dt = time.perf_counter() - t0
    return dt, w.dense_flops() * len(rows) / w.n_q / dt / 1e12


def cpu_baseline(w, act, wts, target_s):
    cache_bits = oracle_prepare(w, act, wts)
    rows, n_tok = size_oracle_sample(w, act, wts, cache_bits, target_s)
    dt, flops = oracle_sample_step(w, act, wts, cache_bits, rows, n_tok)
    line = {"value": flops / dt / 1e12, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": (f"fp64 oracle: append of {n_tok} chunk tokens + attention of {len(rows)} of "
                       f"{w.n_q} query rows x {w.heads} heads x {w.n_kv} keys; {dt:.1f} s; FLOPs "
                       f"counted with the same absorbed convention as the GPU value"),
            "seconds": dt}
    # The dense per-head baseline's oracle, timed the same way on a few seconds' worth of rows.
    kv = workload.batch_dense_kv(w)
    d64, _ = dense_oracle_sample(w, kv, act, 64)
    n_dense = int(min(w.n_q, max(64, 64 * max(1.0, (target_s / 3) / max(d64, 1e-3)))))
    dd, dense_tf = dense_oracle_sample(w, kv, act, n_dense)
    line["dense"] = {"value": dense_tf, "unit": "TFLOP/s", "seconds": dd,
                     "sample": f"fp64 dense oracle: {n_dense} of {w.n_q} query rows x {w.heads} heads x {w.n_kv} keys"}
    return line


# ---------------------------------------------------------------------------
# Reference arm: the oracle timed on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    wts = workload.layer_weights(w)
    act = workload.batch_activations(w)
    cache_bits = oracle_prepare(w, act, wts)
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows, n_tok = size_oracle_sample(w, act, wts, cache_bits, min(2.0, budget))
    for _ in range(args.warmup):
        oracle_sample_step(w, act, wts, cache_bits, rows, n_tok)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample_step(w, act, wts, cache_bits, rows, n_tok)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = (f"fp64 oracle per step: append of {n_tok} chunk tokens + attention of {len(rows)} of "
              f"{w.n_q} query rows x {w.heads} heads x {w.n_kv} keys")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_desc(w), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": _blas_threads(),
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def run_ours(args, w, rank, world, local_rank):
    import torch
    import latent_kv_cache_b200 as vm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # Each rank is an independent replica with its own seed (weak scaling).
    wr = w.with_(seed=w.seed + 100003 * rank)
    wts = workload.layer_weights(wr)
    act = workload.batch_activations(wr)

    def T(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    x_all = T(act["x"])
    wd, wk, wuk, wuv = T(wts["w_dkv"]), T(wts["w_kr"]), T(wts["w_uk"]), T(wts["w_uv"])
    q, qr = T(act["q"]), T(act["q_rope"])
    out = torch.empty_like(q)
    cache = torch.zeros(w.batch, w.n_kv, 224, dtype=torch.bfloat16, device=dev)
    per = w.tokens_per_frame
    for f0 in range(0, w.cached_frames, w.chunk_frames):  # the window's cached frames
        nf = min(w.chunk_frames, w.cached_frames - f0)
        vm.vmla_cache_append(x_all[:, f0 * per:(f0 + nf) * per].contiguous(), wd, wk, cache, f0 * per, f0,
                             w.grid_h, w.grid_w)
    x_chunk = x_all[:, w.n_cached:].contiguous()
    del x_all
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    class _Flush:
        def zero_(self):
            flush_w.zero_()          # evict: every L2 line now holds this (dirty) buffer
            flush_r.max()            # read another buffer: the dirty lines are written back now
    flush_buf = _Flush()

    def step():
        vm.vmla_cache_append(x_chunk, wd, wk, cache, w.n_cached, w.chunk_t0, w.grid_h, w.grid_w, stream)
        vm.vmla_chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                out, stream)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush_buf.zero_()
        step()
    vm.vmla_get_device_status(stream)

    # ---- timed region: K steps, L2 flushed before each, events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    barrier()
    sampler.start()
    for k in range(args.steps):
        flush_buf.zero_()
        ev[k][0].record(stream)
        vm.vmla_cache_append(x_chunk, wd, wk, cache, w.n_cached, w.chunk_t0, w.grid_h, w.grid_w, stream)
        ev[k][1].record(stream)
        vm.vmla_chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                out, stream)
        ev[k][2].record(stream)
    barrier()
    clocks = sampler.stop()
    vm.vmla_get_device_status(stream)
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    app_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    gpu_launches = 2 * args.steps

    flops_step = w.attention_flops() + w.append_flops()
    value = job_value(world, args.steps, flops_step, total_ms)
    ms_per_step = total_ms / args.steps
    attn_mean = sum(attn_ms) / len(attn_ms)
    app_mean = sum(app_ms) / len(app_ms)

    # ---- dense per-head baseline on the same queries (3072 scalars per token)
    kv = workload.batch_dense_kv(wr)
    kd, vd = T(kv["k"]), T(kv["v"])
    out_d = torch.empty_like(q)
    for _ in range(args.warmup):
        flush_buf.zero_()
        vm.vmla_dense_attention(q, kd, vd, SCALE, out_d, stream)
    dense_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush_buf.zero_()
        dense_ev[k][0].record(stream)
        vm.vmla_dense_attention(q, kd, vd, SCALE, out_d, stream)
        dense_ev[k][1].record(stream)
    barrier()
    vm.vmla_get_device_status(stream)
    dense_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in dense_ev), dist, dev) / args.steps
    del kd, vd, out_d

    # ---- non-absorbed form on the same cache and queries: materialise K_h / V_h, then attend
    kvm = torch.empty(w.batch, w.n_kv, 2 * w.heads, w.d_head, dtype=torch.bfloat16, device=dev)
    out_m = torch.empty_like(q)

    def mat_step(e=None):
        if e is not None:
            e[0].record(stream)
        vm.vmla_materialize_kv(wuk, wuv, cache, w.n_kv, kvm, stream)
        if e is not None:
            e[1].record(stream)
        vm.vmla_chunk_attention_materialized(q, qr, kvm, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                             out_m, stream)
        if e is not None:
            e[2].record(stream)

    for _ in range(args.warmup):
        flush_buf.zero_()
        mat_step()
    mat_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush_buf.zero_()
        mat_step(mat_ev[k])
    barrier()
    vm.vmla_get_device_status(stream)
    ms_mat = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in mat_ev), dist, dev) / args.steps
    ms_matt = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in mat_ev), dist, dev) / args.steps
    nonabsorbed = {
        "ms_materialize": ms_mat, "ms_attention": ms_matt, "ms_total": ms_mat + ms_matt,
        "attention_tflops": w.nonabsorbed_flops() / (ms_matt * 1e-3) / 1e12,
        "flops_per_call": w.nonabsorbed_flops(), "workspace_bytes": kvm.numel() * 2,
        "note": "materialise once per layer and chunk; every denoising step reuses it",
    }
    del kvm, out_m

    # ---- latent-width sweep: append + chunk attention at d_c = 64 / 128 / 192 / 256
    dc_sweep = {}
    for dc in (64, 128, 192, 256):
        wdc = wr.with_(d_c=dc)
        wts_dc = workload.layer_weights(wdc)
        wd_dc, wk_dc = T(wts_dc["w_dkv"]), T(wts_dc["w_kr"])
        wuk_dc, wuv_dc = T(wts_dc["w_uk"]), T(wts_dc["w_uv"])
        cache_dc = torch.zeros(w.batch, w.n_kv, dc + w.d_r, dtype=torch.bfloat16, device=dev)
        x_win = T(workload.batch_activations(wdc)["x"])
        for f0 in range(0, w.cached_frames, w.chunk_frames):
            nf = min(w.chunk_frames, w.cached_frames - f0)
            vm.vmla_cache_append_dc(x_win[:, f0 * per:(f0 + nf) * per].contiguous(), wd_dc, wk_dc, cache_dc,
                                    f0 * per, f0, w.grid_h, w.grid_w)
        del x_win

        def dc_step(e=None):
            if e is not None:
                e[0].record(stream)
            vm.vmla_cache_append_dc(x_chunk, wd_dc, wk_dc, cache_dc, w.n_cached, w.chunk_t0, w.grid_h, w.grid_w,
                                    stream)
            if e is not None:
                e[1].record(stream)
            vm.vmla_chunk_attention_dc(q, qr, wuk_dc, wuv_dc, cache_dc, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w,
                                       SCALE, out, stream)
            if e is not None:
                e[2].record(stream)

        for _ in range(args.warmup):
            flush_buf.zero_()
            dc_step()
        dc_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        barrier()
        for k in range(args.steps):
            flush_buf.zero_()
            dc_step(dc_ev[k])
        barrier()
        vm.vmla_get_device_status(stream)
        ms_app = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in dc_ev), dist, dev) / args.steps
        ms_att = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in dc_ev), dist, dev) / args.steps
        dc_sweep[str(dc)] = {
            "attention_ms": ms_att, "attention_tflops": wdc.attention_flops() / (ms_att * 1e-3) / 1e12,
            "append_us": ms_app * 1e3, "cache_bytes_per_token": (dc + w.d_r) * 2,
            "window_cache_mb": w.batch * w.n_kv * (dc + w.d_r) * 2 / 1e6,
        }
        del wd_dc, wk_dc, wuk_dc, wuv_dc, cache_dc

    # ---- the same attention with the last partial wave split over key ranges
    ws_bytes = vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, w.heads, w.n_kv)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    out_s = torch.empty_like(q)
    for _ in range(args.warmup):
        flush_buf.zero_()
        vm.vmla_chunk_attention_splitkv(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                        out_s, workspace=ws, stream=stream)
    sk_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush_buf.zero_()
        sk_ev[k][0].record(stream)
        vm.vmla_chunk_attention_splitkv(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                        out_s, workspace=ws, stream=stream)
        sk_ev[k][1].record(stream)
    barrier()
    vm.vmla_get_device_status(stream)
    splitkv_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in sk_ev), dist, dev) / args.steps
    splitkv = {"ms": splitkv_ms, "tflops": w.attention_flops() / (splitkv_ms * 1e-3) / 1e12,
               "workspace_bytes": ws_bytes,
               "note": "vmla_chunk_attention_splitkv: the last partial wave of units split over key ranges "
                       "(no split when the units fill whole waves)"}
    del ws, out_s

    # ---- the projections either side of the attention (same chunk, this layer's weights)
    iw = workload.io_weights(wr)
    wq, wqr, wo = T(iw["w_q"]), T(iw["w_qr"]), T(iw["w_o"])
    q_p, qr_p, y_p = torch.empty_like(q), torch.empty_like(qr), torch.empty_like(x_chunk)
    for _ in range(args.warmup):
        flush_buf.zero_()
        vm.vmla_query_projection(x_chunk, wq, wqr, q_p, qr_p, stream)
        vm.vmla_output_projection(out, wo, y_p, stream)
    proj_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush_buf.zero_()
        proj_ev[k][0].record(stream)
        vm.vmla_query_projection(x_chunk, wq, wqr, q_p, qr_p, stream)
        proj_ev[k][1].record(stream)
        vm.vmla_output_projection(out, wo, y_p, stream)
        proj_ev[k][2].record(stream)
    barrier()
    vm.vmla_get_device_status(stream)
    ms_qp = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in proj_ev), dist, dev) / args.steps
    ms_op = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in proj_ev), dist, dev) / args.steps
    nq_tok = w.batch * w.n_q
    fq = 2.0 * nq_tok * w.d_model * w.heads * (w.d_head + w.d_r)
    fo = 2.0 * nq_tok * w.heads * w.d_head * w.d_model
    projections = {
        "query": {"us": ms_qp * 1e3, "tflops": fq / (ms_qp * 1e-3) / 1e12},
        "output": {"us": ms_op * 1e3, "tflops": fo / (ms_op * 1e-3) / 1e12},
        "note": "x W_Q^T with x W_QR^T in one pass; o W_O^T; bf16 in, fp32 accumulate",
    }
    del wq, wqr, wo, q_p, qr_p, y_p

    # ---- end to end through the public API: pinned host inputs -> device -> host result.
    # Every step copies its own inputs in (x of the chunk, q, q_rope) and its output
    # out.  The step's device tensors are double-buffered so that, as in a serving
    # loop, step k+1's host-to-device copies and step k-1's device-to-host copy run
    # on two copy streams while step k computes.  Instead of a flush kernel inside
    # the timed region, the steps rotate over n_rot window caches (as a server
    # interleaving n_rot streams would), so a step's cache was last touched n_rot - 1
    # steps earlier, with more than 3x the L2 capacity of traffic in between.
    h_x = x_chunk.cpu().pin_memory()
    h_q = q.cpu().pin_memory()
    h_qr = qr.cpu().pin_memory()
    h_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = h_x.numel() * 2 + h_q.numel() * 2 + h_qr.numel() * 2
    d2h = h_out[0].numel() * 2
    l2_bytes = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20)
    per_step_bytes = cache.numel() * 2 + h2d + d2h
    n_rot = max(2, min(256, -(-3 * l2_bytes // per_step_bytes) + 1))
    l2_between = (n_rot - 1) * per_step_bytes / l2_bytes  # traffic between two uses of a cache, in L2 sizes
    caches = [cache] + [cache.clone() for _ in range(n_rot - 1)]
    dbuf = [{"x": x_chunk, "q": q, "qr": qr, "out": out},
            {"x": torch.empty_like(x_chunk), "q": torch.empty_like(q), "qr": torch.empty_like(qr),
             "out": torch.empty_like(out)}]
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_issue(k):
        i = k & 1
        d = dbuf[i]
        with torch.cuda.stream(s_h2d):
            if k >= 2:
                s_h2d.wait_event(ev_done[i])  # step k-2 has finished reading these inputs
            d["x"].copy_(h_x, non_blocking=True)
            d["q"].copy_(h_q, non_blocking=True)
            d["qr"].copy_(h_qr, non_blocking=True)
            ev_in[i].record(s_h2d)
        stream.wait_event(ev_in[i])
        if k >= 2:
            stream.wait_event(ev_out[i])  # step k-2's output has reached the host
        ck = caches[k % n_rot]
        vm.vmla_cache_append(d["x"], wd, wk, ck, w.n_cached, w.chunk_t0, w.grid_h, w.grid_w, stream)
        vm.vmla_chunk_attention(d["q"], d["qr"], wuk, wuv, ck, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE,
                                d["out"], stream)
        ev_done[i].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_done[i])
            h_out[i].copy_(d["out"], non_blocking=True)
            ev_out[i].record(s_d2h)

    for k in range(args.warmup):
        e2e_issue(k)
    e2e_start, e2e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e2e_start.record(s_h2d)
    for k in range(args.steps):
        e2e_issue(args.warmup + k)
    e2e_end.record(s_d2h)
    barrier()
    vm.vmla_get_device_status(stream)
    e2e_total = max_over_ranks(e2e_start.elapsed_time(e2e_end), dist, dev)
    e2e_value = job_value(world, args.steps, flops_step, e2e_total)

    # ---- the full per-chunk schedule of this shape (30 layers x 4 denoising steps +
    # 30 appends, CUDA graphs) and a >= 2 s back-to-back attention loop
    chunk = None
    others = None
    if w.name == "480p" and not args.no_chunk:
        others = {name: single_layer_figures(vm, workload.CONFIGS[name], dev, dist, 5, 3, local_rank,
                                             seed=7000 + rank)
                  for name in ("480p_b8", "1080p")}
        del dbuf, h_x, h_q, h_qr, h_out, caches
        torch.cuda.empty_cache()
        chunk = chunk_schedule_figures(vm, workload.CONFIGS["480p_chunk"].with_(seed=wr.seed), dev, rank, dist,
                                       args.chunk_replays, args.warmup, local_rank, full_layer=False)

    peak, peak_sust, hbm, peak_src = measured_peaks()
    achieved = w.attention_flops() / (attn_mean * 1e-3) / 1e12
    traffic = profiled_traffic(w.name)
    sm_max = clocks.get("sm_max_mhz") or 1965
    fp32_peak = 148 * 128 * 2 * sm_max * 1e6 / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_desc(w),
        "ms_chunk_attention": attn_mean, "ms_cache_append": app_mean,
        "attention_tflops": achieved,
        "pct_bf16_peak": 100.0 * achieved / peak,
        "pct_bf16_peak_sustained": 100.0 * achieved / peak_sust if peak_sust else None,
        "pct_bf16_nominal_2250": 100.0 * achieved / 2250.0,
        "attention_layer_tokens_per_s": w.batch * w.n_q / (attn_mean * 1e-3),
        "nonabsorbed": nonabsorbed,
        "splitkv": splitkv,
        "projections": projections,
        "dc_sweep": dc_sweep,
        "dense": {"ms": dense_ms, "tflops": w.dense_flops() / (dense_ms * 1e-3) / 1e12,
                  "mla_over_dense_ms": attn_mean / dense_ms,
                  "cache_bytes_per_token": {"mla": 224 * 2, "dense": 3072 * 2}},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": "profiled constant (profiles/chunk_attn_480p_traffic.json), "
                                       "null unless the kernel source hash matches",
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "kernel": "k_chunk_attn"},
        "attention_dram_read_gbs": (traffic / (attn_mean * 1e-3) / 1e9) if traffic else None,
        "append": {"us": app_mean * 1e3, "bound": "alu",
                   "fp32_tflops": w.append_flops() / (app_mean * 1e-3) / 1e12,
                   "fp32_peak_tflops": fp32_peak, "frac": w.append_flops() / (app_mean * 1e-3) / 1e12 / fp32_peak,
                   "fp32_peak_source": "148 SMs x 128 FMA lanes x 2 flop x the max SM clock",
                   "gbs": (x_chunk.numel() * 2 + 224 * w.d_model * 2 + w.batch * w.n_q * 224 * 2)
                   / (app_mean * 1e-3) / 1e9, "hbm_peak_gbs": hbm},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_total / args.steps,
                "pipeline": "double-buffered: next step's H2D and previous step's D2H overlap this step's compute",
                "l2": f"no flush kernel in the timed region: the steps rotate over {n_rot} window caches "
                      f"({n_rot * cache.numel() * 2 / 1e6:.0f} MB), so each step's cache was last touched "
                      f"{n_rot - 1} steps earlier, with {l2_between:.1f}x the L2 capacity of traffic in between"},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
    }
    if chunk is not None:
        line["chunk_480p"] = chunk
    if others is not None:
        line["other_workloads"] = others
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, act, wts, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# The full per-chunk schedule: L layers x (1 append + S denoising-step attentions),
# captured once as a CUDA graph and replayed (timing-only inputs drawn on device)
# ---------------------------------------------------------------------------
def build_chunk_schedule(vm, w, dev, seed=0, dense=False, nonabsorbed=False, nonabsorbed_reuse=False,
                         full_layer=False, attention_only=False, chunks=1):
    """Per-layer caches (filled by appends over the cached frames), the chunk's
    tokens, per-(layer, step) queries and outputs.  Returns, for each of `chunks`
    consecutive chunks, a list of zero-argument launch closures in schedule order,
    and the tensors they use.  Chunk g starts at frame cached_frames + g * chunk_frames
    and its tokens go to ring slots (n_cached + g * n_q) mod n_kv: from the second
    chunk on, each append evicts the window's oldest frames.
    full_layer: each (step, layer) also computes its queries from the hidden
    states (q, q_r = x W_Q^T, x W_QR^T) and projects the heads' output (o W_O^T).
    dense: the per-head baseline, whose per-layer append writes the chunk's
    K = x W_K^T and V = x W_V^T (3072 scalars per token) into its ring.
    nonabsorbed: each layer materialises its K_h / V_h once per chunk into a
    buffer of its own, which the chunk's denoising steps reuse (one buffer per
    layer live during the chunk).  nonabsorbed_reuse: every (step, layer)
    materialises into one shared buffer right before its attention (one buffer
    live in all).  attention_only: the latent attentions alone, no appends (the
    caches keep their window), for a back-to-back attention loop."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    D, H, per = w.d_model, w.heads, w.tokens_per_frame

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    x_win = rnd(w.batch, w.n_kv, D)
    x_chunk = x_win[:, w.n_cached:].contiguous()
    layers = []
    for _ in range(w.layers):
        L = {"wd": rnd(w.d_c, D, std=D ** -0.5), "wk": rnd(w.d_r, D, std=D ** -0.5),
             "wuk": rnd(H * w.d_head, w.d_c, std=w.d_c ** -0.5), "wuv": rnd(H * w.d_head, w.d_c, std=w.d_c ** -0.5),
             "cache": torch.empty(w.batch, w.n_kv, w.d_c + w.d_r, dtype=torch.bfloat16, device=dev),
             "q": [rnd(w.batch, w.n_q, H, w.d_head) for _ in range(w.steps)],
             "qr": [rnd(w.batch, w.n_q, H, w.d_r) for _ in range(w.steps)],
             "out": [torch.empty(w.batch, w.n_q, H, w.d_head, dtype=torch.bfloat16, device=dev) for _ in range(w.steps)]}
        for f0 in range(0, w.cached_frames, w.chunk_frames):
            nf = min(w.chunk_frames, w.cached_frames - f0)
            vm.vmla_cache_append(x_win[:, f0 * per:(f0 + nf) * per].contiguous(), L["wd"], L["wk"], L["cache"],
                                 f0 * per, f0, w.grid_h, w.grid_w)
        if dense:
            if w.batch != 1 or D != H * w.d_head:
                raise ValueError("the dense schedule writes K/V slices in place: batch 1, d_model = heads * 128")
            L["k"] = rnd(w.batch, w.n_kv, H, w.d_head)
            L["v"] = rnd(w.batch, w.n_kv, H, w.d_head)
            L["w_kd"] = rnd(H * w.d_head, D, std=D ** -0.5)
            L["w_vd"] = rnd(H * w.d_head, D, std=D ** -0.5)
        if full_layer:
            L["wq"] = rnd(H * w.d_head, D, std=D ** -0.5)
            L["wqr"] = rnd(H * w.d_r, D, std=D ** -0.5)
            L["wo"] = rnd(D, H * w.d_head, std=(H * w.d_head) ** -0.5)
            L["y"] = torch.empty(w.batch, w.n_q, D, dtype=torch.bfloat16, device=dev)
        if nonabsorbed:  # this layer's materialised K/V, live for the chunk's denoising steps
            L["kv"] = torch.empty(w.batch, w.n_kv, 2 * H, w.d_head, dtype=torch.bfloat16, device=dev)
        layers.append(L)
    if nonabsorbed_reuse:  # one materialised K/V buffer for every (step, layer)
        shared_kv = torch.empty(w.batch, w.n_kv, 2 * H, w.d_head, dtype=torch.bfloat16, device=dev)
        for L in layers:
            L["kv"] = shared_kv
    del x_win
    x_heads = x_chunk.view(w.batch, w.n_q, H, w.d_head) if dense else None

    def chunk_ops(ci):
        slot = (w.n_cached + ci * w.n_q) % w.n_kv
        t0 = w.chunk_t0 + ci * w.chunk_frames
        ops = []
        for s in range(w.steps):
            for L in layers:
                if dense:
                    if s == 0:  # the chunk's K and V enter the dense ring once per layer
                        for wn, cn in (("w_kd", "k"), ("w_vd", "v")):
                            dst = L[cn][:, slot:slot + w.n_q].view(w.batch, w.n_q, D)
                            ops.append(lambda L=L, wn=wn, dst=dst: vm.vmla_output_projection(x_heads, L[wn], dst))
                    ops.append(lambda L=L, s=s: vm.vmla_dense_attention(L["q"][s], L["k"], L["v"], SCALE, L["out"][s]))
                    continue
                if s == 0 and not attention_only:  # the chunk's latents enter the window's ring once per layer
                    ops.append(lambda L=L: vm.vmla_cache_append(x_chunk, L["wd"], L["wk"], L["cache"], slot, t0,
                                                                w.grid_h, w.grid_w))
                    if nonabsorbed:
                        ops.append(lambda L=L: vm.vmla_materialize_kv(L["wuk"], L["wuv"], L["cache"], w.n_kv, L["kv"]))
                if nonabsorbed_reuse:
                    ops.append(lambda L=L: vm.vmla_materialize_kv(L["wuk"], L["wuv"], L["cache"], w.n_kv, L["kv"]))
                if nonabsorbed or nonabsorbed_reuse:
                    ops.append(lambda L=L, s=s: vm.vmla_chunk_attention_materialized(
                        L["q"][s], L["qr"][s], L["kv"], L["cache"], w.n_kv, t0, w.grid_h, w.grid_w, SCALE,
                        L["out"][s]))
                    continue
                if full_layer:
                    ops.append(lambda L=L, s=s: vm.vmla_query_projection(x_chunk, L["wq"], L["wqr"], L["q"][s],
                                                                         L["qr"][s]))
                ops.append(lambda L=L, s=s: vm.vmla_chunk_attention(L["q"][s], L["qr"][s], L["wuk"], L["wuv"],
                                                                    L["cache"], w.n_kv, t0, w.grid_h, w.grid_w,
                                                                    SCALE, L["out"][s]))
                if full_layer:
                    ops.append(lambda L=L, s=s: vm.vmla_output_projection(L["out"][s], L["wo"], L["y"]))
        return ops

    return [chunk_ops(ci) for ci in range(chunks)], layers


def single_layer_figures(vm, w, dev, dist, reps, warmup, local_rank=0, seed=0):
    """Event-timed append, latent attention, non-absorbed form and dense baseline of
    one layer of workload `w` (timing-only inputs drawn on the device from a seeded
    generator; the parity tests cover these shapes with the oracle's inputs).  L2 is
    flushed before every timed call; clocks are sampled during the timed calls."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    D, H = w.d_model, w.heads

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    wd, wk = rnd(w.d_c, D, std=D ** -0.5), rnd(w.d_r, D, std=D ** -0.5)
    wuk, wuv = rnd(H * w.d_head, w.d_c, std=w.d_c ** -0.5), rnd(H * w.d_head, w.d_c, std=w.d_c ** -0.5)
    cache = torch.empty(w.batch, w.n_kv, w.d_c + w.d_r, dtype=torch.bfloat16, device=dev)
    per = w.tokens_per_frame
    for f0 in range(0, w.cached_frames, w.chunk_frames):
        nf = min(w.chunk_frames, w.cached_frames - f0)
        vm.vmla_cache_append(rnd(w.batch, nf * per, D), wd, wk, cache, f0 * per, f0, w.grid_h, w.grid_w)
    x_chunk = rnd(w.batch, w.n_q, D)
    q, qr = rnd(w.batch, w.n_q, H, w.d_head), rnd(w.batch, w.n_q, H, w.d_r)
    out = torch.empty_like(q)
    kd, vd = rnd(w.batch, w.n_kv, H, w.d_head), rnd(w.batch, w.n_kv, H, w.d_head)
    kvm = torch.empty(w.batch, w.n_kv, 2 * H, w.d_head, dtype=torch.bfloat16, device=dev)
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    ws_bytes = vm.vmla_chunk_attention_splitkv_workspace_bytes(w.batch, w.n_q, H, w.n_kv)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    calls = {
        "append": lambda: vm.vmla_cache_append(x_chunk, wd, wk, cache, w.n_cached, w.chunk_t0, w.grid_h, w.grid_w),
        "attention": lambda: vm.vmla_chunk_attention(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0, w.grid_h,
                                                     w.grid_w, SCALE, out),
        "materialize": lambda: vm.vmla_materialize_kv(wuk, wuv, cache, w.n_kv, kvm),
        "attention_materialized": lambda: vm.vmla_chunk_attention_materialized(
            q, qr, kvm, cache, w.n_kv, w.chunk_t0, w.grid_h, w.grid_w, SCALE, out),
        "dense": lambda: vm.vmla_dense_attention(q, kd, vd, SCALE, out),
        "attention_splitkv": lambda: vm.vmla_chunk_attention_splitkv(q, qr, wuk, wuv, cache, w.n_kv, w.chunk_t0,
                                                                     w.grid_h, w.grid_w, SCALE, out, workspace=ws),
    }
    ms = {}
    sampler = ClockSampler(local_rank)
    for name, fn in calls.items():
        for _ in range(warmup):
            flush_w.zero_()
            flush_r.max()
            fn()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        if name == "attention":
            sampler.start()
        for e in ev:
            flush_w.zero_()
            flush_r.max()
            e[0].record()
            fn()
            e[1].record()
        torch.cuda.synchronize()
        if name == "attention":
            clocks = sampler.stop()
        if dist is not None:
            dist.barrier()
        ms[name] = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / reps, dist, dev)
    vm.vmla_get_device_status()
    res = {
        "workload": (f"{w.name}: B={w.batch}, {w.grid_h}x{w.grid_w} patches/frame, Nq={w.n_q}, n_kv={w.n_kv}, "
                     f"H={H}x{w.d_head}, d_c={w.d_c}, d_r={w.d_r}"),
        "reps": reps,
        "attention": {"ms": ms["attention"], "tflops": w.attention_flops() / (ms["attention"] * 1e-3) / 1e12},
        "attention_splitkv": {"ms": ms["attention_splitkv"],
                              "tflops": w.attention_flops() / (ms["attention_splitkv"] * 1e-3) / 1e12,
                              "workspace_bytes": ws_bytes,
                              "note": "the last partial wave of (sample, query tile, head) units split over key "
                                      "ranges (no split when the units fill whole waves)"},
        "append": {"us": ms["append"] * 1e3},
        "nonabsorbed": {"ms_materialize": ms["materialize"], "ms_attention": ms["attention_materialized"],
                        "ms_total": ms["materialize"] + ms["attention_materialized"],
                        "attention_tflops": w.nonabsorbed_flops() / (ms["attention_materialized"] * 1e-3) / 1e12},
        "dense": {"ms": ms["dense"], "tflops": w.dense_flops() / (ms["dense"] * 1e-3) / 1e12},
        "clocks_attention": clocks,
        "inputs": "drawn on the device (torch normal, seeded); timing only",
    }
    del cache, q, qr, out, kd, vd, kvm, flush_w, flush_r, ws
    torch.cuda.empty_cache()
    return res


def capture_graph(ops):
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for op in ops:  # eager pass: first-call setup happens outside the capture
            op()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for op in ops:
            op()
    torch.cuda.synchronize()
    return graph


def chunk_schedule_figures(vm, w, dev, rank, dist, replays, warmup, local_rank=0, full_layer=True,
                           sustained_s=2.0):
    """ms per chunk of the full per-chunk schedule (one replay of a captured graph =
    one chunk) for the absorbed, both non-absorbed and the dense schedules, plus a
    back-to-back loop of the latent attentions alone for at least `sustained_s`
    seconds with the SM clock sampled during it."""
    import torch

    # One graph per ring position: chunk c replays graph c mod G, so consecutive
    # chunks slide the window (each append evicts the oldest frames).
    G = w.n_kv // w.n_q if w.n_kv % w.n_q == 0 else 1

    def sync_all():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()

    def timed(graphs, n):
        for i in range(max(warmup, len(graphs))):
            graphs[i % len(graphs)].replay()
        sync_all()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for i in range(n):
            graphs[i % len(graphs)].replay()
        ev[1].record()
        sync_all()
        return max_over_ranks(ev[0].elapsed_time(ev[1]) / n, dist, dev)

    def measure(n=None, sampler=None, **kind):
        op_lists, _ = build_chunk_schedule(vm, w, dev, seed=(2000 if kind.get("dense") else 1000) + rank,
                                           chunks=G, **kind)
        graphs = [capture_graph(ops) for ops in op_lists]
        vm.vmla_get_device_status()
        if sampler is not None:
            sampler.start()
        ms = timed(graphs, n or replays)
        clocks = sampler.stop() if sampler is not None else None
        vm.vmla_get_device_status()
        del graphs, op_lists
        torch.cuda.empty_cache()
        return ms, clocks

    ms_chunk, clocks = measure(sampler=ClockSampler(local_rank))
    ms_nonabs, _ = measure(nonabsorbed=True)
    ms_reuse, _ = measure(nonabsorbed_reuse=True)
    ms_dense, _ = measure(dense=True)
    ms_full = measure(full_layer=True)[0] if full_layer else None
    kv_one = w.batch * w.n_kv * 2 * w.heads * w.d_head * 2
    res = {
        "workload": (f"{w.name}: {w.layers} layers x ({w.steps} chunk attentions) + {w.layers} cache appends "
                     f"per chunk, 480P shapes (Nq={w.n_q}, n_kv={w.n_kv}), one CUDA graph replay per chunk"),
        "window": (f"sliding: {G} graphs (one per ring position) replayed in rotation, each chunk's append "
                   f"evicts the oldest {w.chunk_frames} frames"),
        "l2": "inputs larger than L2 (per-layer caches, queries and outputs)",
        "replays": replays,
        "ms_per_chunk": ms_chunk, "clocks": clocks,
        "tflops": (w.layers * w.steps * w.attention_flops() + w.layers * w.append_flops()) / (ms_chunk * 1e-3) / 1e12,
        "nonabsorbed": {"ms_per_chunk": ms_nonabs, "transient_kv_bytes": w.layers * kv_one,
                        "how": "each layer materialises K_h/V_h once per chunk into its own buffer; "
                               "the chunk's denoising steps reuse it"},
        "nonabsorbed_reuse": {"ms_per_chunk": ms_reuse, "transient_kv_bytes": kv_one,
                              "how": "every (step, layer) materialises into one shared buffer before its attention"},
        "dense": {"ms_per_chunk": ms_dense, "layers": w.layers, "steps": w.steps,
                  "append": "K = x W_K^T and V = x W_V^T of the chunk written into the dense ring per layer",
                  "kv_cache_bytes": {"mla": w.layers * w.batch * w.n_kv * 448,
                                     "dense": w.layers * w.batch * w.n_kv * 6144}},
    }
    if full_layer:
        res["full_layer"] = {"ms_per_chunk": ms_full,
                             "step": "per (step, layer): q/q_r projection + chunk attention + output projection; "
                                     "one append per layer",
                             "projection_flops_per_chunk": w.layers * w.steps * w.io_projection_flops()}
    if sustained_s > 0:
        # Back-to-back latent attentions (30 layers x 4 steps per replay, no appends)
        # for >= sustained_s seconds: the power-capped steady state of a rollout.
        est_ms = ms_chunk * w.layers * w.steps / (w.layers * w.steps + w.layers)
        n = max(replays, int(sustained_s * 1e3 / max(est_ms, 1e-3)) + 1)
        ms_att, sclocks = measure(n=n, sampler=ClockSampler(local_rank, period_s=0.005), attention_only=True)
        tf = w.layers * w.steps * w.attention_flops() / (ms_att * 1e-3) / 1e12
        _, peak_sust, _, src = measured_peaks()
        mhz = (sclocks or {}).get("sm_mhz")
        res["sustained"] = {
            "seconds": n * ms_att / 1e3, "replays": n, "launches": n * w.layers * w.steps,
            "ms_per_attention": ms_att / (w.layers * w.steps), "attention_tflops": tf,
            "peak_sustained": peak_sust, "frac_of_sustained": tf / peak_sust if peak_sust else None,
            "peak_source": f"{src} bf16_tflops_sustained",
            "tflops_per_sm_ghz": tf / (mhz / 1e3) if mhz else None,
            "clocks": sclocks,
            "how": "graph replays of the 120 chunk attentions of one chunk (30 layers x 4 steps), back to back",
        }
    return res


def run_chunk_schedule(args, w, rank, world, local_rank):
    """ms per chunk of the full schedule, as its own JSON line."""
    import torch
    import latent_kv_cache_b200 as vm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fig = chunk_schedule_figures(vm, w, dev, rank, dist, args.steps, args.warmup, local_rank)
    ms_chunk = fig["ms_per_chunk"]
    flops = w.layers * w.steps * w.attention_flops() + w.layers * w.append_flops()
    value = job_value(world, 1, flops, ms_chunk)
    n_launch = w.layers * w.steps + w.layers  # the absorbed graph, whose time is `value`
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_chunk, "ms_per_chunk": ms_chunk, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_desc(w), step=f"one chunk: {w.layers} layers x ({w.steps} chunk attentions) "
                                               f"+ {w.layers} cache appends, one CUDA graph replay",
                       window=fig["window"], l2=fig["l2"]),
        "nonabsorbed": fig["nonabsorbed"], "nonabsorbed_reuse": fig["nonabsorbed_reuse"],
        "full_layer": fig["full_layer"], "dense": fig["dense"], "sustained": fig.get("sustained"),
        "gpu_launches": args.steps * n_launch, "clocks": fig["clocks"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workload.CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if w.layers > 1 or w.steps > 1:
        return run_chunk_schedule(args, w, rank, world, local_rank)
    return run_ours(args, w, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
