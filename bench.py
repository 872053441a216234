"""Benchmark of one absorbed-MLA decode step on the DeepSeek-V2-scale workload.

A step is the whole hot path over one batch, from the new tokens' hidden states x to the layer
output y: the input projections (query latent c' = x W'_c, the per-head query halves, the latent and
rotary key x [W_c, W_kr]) with the append of the new latent (RMSNorm + RoPE), the absorption of the
queries into the latent (W_UK), attention over the latent cache (fused split-KV decode), and the
value and output projections (W_UV, W_O). Workload: batch 64, 128 heads, d_c 512, d_r 64, qk_nope
128, v_head 128, d_model 5120, q_rank 1536, 4096 cached positions per sequence, bf16 storage, fp32
accumulation. Inputs are seeded and synthetic; the per-step traffic (302 MB of cache + 298 MB of
weights) is larger than the 126 MB L2, so no separate flush is needed between steps.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun every rank runs an independent replica (the path
shards over sequences with no exchange step), and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA absorbed decode tokens/s and latent-cache HBM GB/s, % of B200 roofline"
WORKLOAD = dict(batch=64, n_heads=128, kv_lora_rank=512, rope_dim=64, qk_nope=128, v_head=128,
                d_model=5120, seqlen=4096, q_lora_rank=1536)
SEED = 1003
CONFIG = {
    "workload": "DeepSeek-V2-scale absorbed MLA decode step from hidden states: input projections "
                "(query latent q_rank 1536, KV down-projection) + append + absorb + split-KV decode + "
                "W_UV/W_O projection; B64 H128 d_c512 d_r64 qk_nope128 v_head128 d_model5120 "
                "T4096 per sequence, bf16 storage, fp32 accumulate",
    "batch": 64, "n_heads": 128, "kv_lora_rank": 512, "rope_dim": 64, "qk_nope": 128,
    "v_head": 128, "d_model": 5120, "q_lora_rank": 1536, "seq_len": 4096, "n_q": 1,
    "l2": "no flush: every step streams 302 MB of latent cache + 298 MB of weights (> 126 MB L2)",
    "parallelism": "replicas (one independent decode per GPU, no collective)",
}
DECODE_SOURCES = ("head_latent_attention_08_b200/csrc/tc_decode.cu",
                  "head_latent_attention_08_b200/csrc/sm100.cuh",
                  "head_latent_attention_08_b200/csrc/common.cuh")


def replica_seed(rank: int) -> int:
    """Every rank decodes its own replica of the workload, drawn from its own seed."""
    return SEED + rank


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank sets the job's time (all ranks take part; world size 1 returns value)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cache_bytes() -> int:
    w = WORKLOAD
    return w["batch"] * w["seqlen"] * (w["kv_lora_rank"] + w["rope_dim"]) * 2


def decode_flops() -> int:
    w = WORKLOAD
    return w["batch"] * w["n_heads"] * w["seqlen"] * (2 * (w["kv_lora_rank"] + w["rope_dim"]) +
                                                      2 * w["kv_lora_rank"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def sustained_tflops() -> float:
    """The measured seconds-long bf16 GEMM rate under the power cap (the fallback's figure if the
    measurement file is absent)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p)).get("bf16_tflops_sustained", 1400.0))
    return 1400.0


def _code_only(text: str) -> str:
    """The source without comments, blank lines or trailing spaces: edits to comments do not change
    the kernel the counters were taken on."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_hash() -> str:
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            h.update(_code_only(open(p, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on the current
    decode sources (else None)."""
    p = os.path.join(ROOT, "profiles", "decode_c3_traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p))
    if j.get("source_hash") != source_hash():
        return None
    return j.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU, read through NVML every
    ~2 ms by a background thread while the timed region runs (read-only queries)."""

    REASONS = {  # NVML clocks-event reason bits
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.window = None
        self._stop = threading.Event()
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
                except Exception:
                    h = None
            self.h = h if h is not None else pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((time.time(), sm, reasons, power))
            except Exception:
                pass
            time.sleep(0.002)

    def wait_first(self, timeout_s: float = 2.0):
        t0 = time.time()
        while self.ok and not self.samples and time.time() - t0 < timeout_s:
            time.sleep(0.005)

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def mark_extra(self, t0: float, t1: float):
        """A second sampled window (the same steps repeated, untimed) whose samples count with the
        timed region's: the timed region alone lasts a few milliseconds, a few NVML samples."""
        self.extra = (t0, t1)

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self.t.join(timeout=2)
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return None
        rows = self.samples
        timed = extra = []
        if self.window:
            t0, t1 = self.window
            timed = [r for r in rows if t0 <= r[0] <= t1]
        if getattr(self, "extra", None):
            e0, e1 = self.extra
            extra = [r for r in rows if e0 <= r[0] <= e1]
        if self.window:
            rows = (timed + extra) or [min(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))]
        reasons = set()
        for _, _, bits, _ in rows:
            for name, bit in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(rows), "samples_in_timed_region": len(timed),
                "samples_in_clock_window": len(extra),
                "power_w_median": statistics.median(r[3] for r in rows),
                "source": "nvml, 2 ms polling, over the timed region and an untimed window of the same steps"}


# --------------------------------------------------------------------------------------------
# CPU oracle legs (the oracle as it stands, timed on the host cores)
# --------------------------------------------------------------------------------------------

def oracle_problem(n_seqs: int, seed: int = SEED):
    """``n_seqs`` sequences of the benchmark workload, with every array already in float64: the
    oracle's own conversions are then no-ops, and the one-off widening of the 168 MB output weight
    stays out of the timed region in both CPU legs."""
    from head_latent_attention_08_b200 import inputs as I
    w = WORKLOAD
    p = I.decode_problem(batch=n_seqs, n_heads=w["n_heads"], kv_lora_rank=w["kv_lora_rank"],
                         rope_dim=w["rope_dim"], qk_nope=w["qk_nope"], v_head=w["v_head"],
                         d_model=w["d_model"], seqlens=[w["seqlen"]] * n_seqs, dtype="bf16",
                         seed=seed)
    for name in ("w_uk", "w_uv", "w_o", "cache"):
        setattr(p, name, np.ascontiguousarray(getattr(p, name), dtype=np.float64))
    pw = I.projection_weights(n_tokens=n_seqs, d_model=w["d_model"], q_rank=w["q_lora_rank"],
                              n_heads=w["n_heads"], qk_nope=w["qk_nope"], rope_dim=w["rope_dim"],
                              kv_lora_rank=w["kv_lora_rank"], dtype="bf16", seed=seed + 100)
    H, n, dr, dc, q_rank = w["n_heads"], w["qk_nope"], w["rope_dim"], w["kv_lora_rank"], w["q_lora_rank"]

    def f64(a):
        return np.ascontiguousarray(a, dtype=np.float64)

    # the page's row-vector layout of the Linear-convention weights (reshape / transpose only)
    p.proj = dict(x=f64(pw.x), w_cq=f64(pw.w_cq.T), w_qc=f64(pw.w_qc.reshape(H, n, q_rank).transpose(0, 2, 1)),
                  w_qr=f64(pw.w_qr.reshape(H, dr, q_rank).transpose(0, 2, 1)), w_c=f64(pw.w_dkv[:dc].T),
                  w_kr=f64(pw.w_dkv[dc:].T))
    return p


class OneCore:
    """Run the oracle single-threaded on one host core: BLAS and torch limited to one thread and
    the process pinned to the first core it may use (restored on exit)."""

    def __enter__(self):
        import torch
        from threadpoolctl import threadpool_limits
        self.torch_threads = torch.get_num_threads()
        torch.set_num_threads(1)
        self.limits = threadpool_limits(limits=1)
        self.affinity = None
        if hasattr(os, "sched_getaffinity"):
            self.affinity = os.sched_getaffinity(0)
            os.sched_setaffinity(0, {min(self.affinity)})
        self.host_cores = len(self.affinity) if self.affinity else (os.cpu_count() or 1)
        return self

    def __exit__(self, *exc):
        import torch
        if self.affinity is not None:
            os.sched_setaffinity(0, self.affinity)
        self.limits.restore_original_limits()
        torch.set_num_threads(self.torch_threads)


def oracle_sample(p) -> float:
    """The full step of the sequences of ``p`` through the oracle; returns seconds."""
    from oracle import mla_oracle as O
    t0 = time.perf_counter()
    w = p.proj
    q_nope, q_pe, c, k_r = O.project_inputs(w["x"], w["w_cq"], w["w_qc"], w["w_qr"], w["w_c"], w["w_kr"],
                                            p.positions)
    cache = O.append_latent(p.cache, p.row_idx, c, k_r, p.positions, norm=True, rope=True, dtype="bf16")
    q_abs = O.absorb_query(q_nope, q_pe, p.w_uk)
    out_lat, _ = O.decode_absorbed(q_abs, cache, p.cu_seqlens, 1, p.kv_lora_rank, p.kq_scale, True)
    O.out_project(out_lat, p.w_uv, p.w_o)
    return time.perf_counter() - t0


CPU_SAMPLE = ("full step (input projections, append, absorb, decode, W_UV/W_O) of one sequence of "
              "the workload per oracle call, float64 numpy oracle, inputs widened to float64 before "
              "timing, one thread pinned to one core")


def cpu_baseline(target_s: float = 12.0):
    """The oracle timed on one host core, one sequence per call (the same call the reference arm
    times per step), repeated for about ``target_s`` seconds."""
    p = oracle_problem(1)
    with OneCore() as oc:
        oracle_sample(p)                          # first call pages everything in
        secs, calls = 0.0, 0
        while secs < target_s and calls < WORKLOAD["batch"]:
            secs += oracle_sample(p)
            calls += 1
    return {"value": calls / secs, "unit": "tokens/s", "cores": 1, "host_cores": oc.host_cores,
            "kind": "oracle", "sample": f"{CPU_SAMPLE}; {calls} calls, {secs:.1f} s; 1 core of {oc.host_cores}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = 1
    p = oracle_problem(per_step)
    with OneCore() as oc:
        for _ in range(args.warmup):
            oracle_sample(p)
        secs = 0.0
        for k in range(args.steps):
            secs += oracle_sample(p)
    value = args.steps * per_step / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": CONFIG,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "host_cores": oc.host_cores,
                             "kind": "oracle",
                             "sample": f"{CPU_SAMPLE}; one call per step; 1 core of {oc.host_cores}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist
    from head_latent_attention_08_b200 import build, inputs as I, mla as M

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    M.lib()

    w = WORKLOAD
    B, H, dc, dr, T = w["batch"], w["n_heads"], w["kv_lora_rank"], w["rope_dim"], w["seqlen"]
    n, dv, D, QR = w["qk_nope"], w["v_head"], w["d_model"], w["q_lora_rank"]
    p = I.decode_problem(batch=B, n_heads=H, kv_lora_rank=dc, rope_dim=dr, qk_nope=n, v_head=dv, d_model=D,
                         seqlens=[T] * B, dtype="bf16", seed=replica_seed(rank))
    pw = I.projection_weights(n_tokens=B, d_model=D, q_rank=QR, n_heads=H, qk_nope=n, rope_dim=dr,
                              kv_lora_rank=dc, dtype="bf16", seed=replica_seed(rank) + 100)
    bf = torch.bfloat16
    dev = torch.device("cuda", local)

    def d_(x, dt=bf):
        return torch.from_numpy(np.ascontiguousarray(x)).to(device=dev, dtype=dt)

    cache = d_(p.cache)
    cu = torch.from_numpy(p.cu_seqlens.astype(np.int32)).to(dev)
    d = M.dims(H, dc, dr, n, dv, D)
    wts = dict(w_cq=d_(pw.w_cq), w_qc=d_(pw.w_qc), w_qr=d_(pw.w_qr), w_dkv=d_(pw.w_dkv), w_uk=d_(p.w_uk),
               w_uv=d_(p.w_uv), w_o=d_(p.w_o))
    layer = M.DecodeLayerStep(d, QR, B, T, cache, cu, **wts)
    x = d_(pw.x)
    row_idx = torch.from_numpy(p.row_idx).to(dev)
    positions = torch.from_numpy(p.positions).to(dev)
    flags = M.MLA_APPEND_NORM | M.MLA_APPEND_ROPE
    # the step call by call (the same calls mla_decode_step makes), so that the decode can be timed alone
    q_nope = torch.empty(B, H, n, dtype=bf, device=dev)
    q_pe = torch.empty(B, H, dr, dtype=bf, device=dev)
    q_abs = torch.empty(B, H, dc + dr, dtype=bf, device=dev)
    out_lat = torch.empty(B, H, dc, dtype=bf, device=dev)     # the decode writes the W_UV operand in bf16
    y = torch.empty(B, D, dtype=bf, device=dev)
    ws_proj = M.workspace(M.mla_project_workspace_size(d, bf, QR, B), dev)
    ws_dec = M.workspace(M.mla_decode_workspace_size(d, bf, B, 1, T, cache.shape[0], M.MLA_DECODE_CAUSAL), dev)
    ws_out = M.workspace(M.mla_out_project_workspace_size(d, bf, B), dev)
    h_x = torch.from_numpy(pw.x).to(bf).pin_memory()
    del p, pw
    stream = torch.cuda.current_stream()

    def step(ev=None):
        M.mla_project_inputs(d, QR, x, wts["w_cq"], wts["w_qc"], wts["w_qr"], wts["w_dkv"], positions, q_nope,
                             q_pe, cache, row_idx, flags, ws_proj)
        M.mla_absorb_weights(d, M.MLA_ABSORB_QUERY, q_nope, q_pe, wts["w_uk"], B, q_abs)
        if ev:
            ev[0].record(stream)
        M.mla_decode_absorbed(d, q_abs, cache, cu, B, 1, T, M.MLA_DECODE_CAUSAL | M.MLA_DECODE_OUT_BF16, out_lat,
                              None, ws_dec)
        if ev:
            ev[1].record(stream)
        M.mla_out_project_bf16(d, out_lat, wts["w_uv"], wts["w_o"], None, B, y, ws_out)

    # ---- device-resident timing -------------------------------------------------------------
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if M.mla_check_status() != 0:
        raise SystemExit("device status word reports a timeout")
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nq = B
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.wait_first()
        # keep the GPU busy until the sampler has seen it under load, then time
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        launches0 = M.mla_launch_count()
        start.record(stream)
        for k in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
        clk.mark(t_wall0, time.time())
        launches = M.mla_launch_count() - launches0
        # the decode call's own duration: the same steps again, with CUDA events around each decode
        # call. An event between two kernels ends their programmatic overlap (about 15 us of the step),
        # so the region above, which gives the step time, carries none.
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for k in range(args.steps):
            step(ev_dec[k])
        torch.cuda.synchronize()
        # clock window: the same steps again for about 0.3 s, untimed, so that the clock record holds
        # enough samples (the timed region itself lasts a few milliseconds)
        t_x0 = time.time()
        while time.time() - t_x0 < 0.3:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        clk.mark_extra(t_x0, time.time())
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), dist if world > 1 else None, dev)
    dec_mean_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev_dec), dist if world > 1 else None,
                                 dev)
    status = M.mla_check_status()

    # ---- end to end through the C ABI's step call with host buffers -------------------------
    # every step copies x, cu_seqlens, row_idx and positions host -> device and y device -> host
    # (mla_decode_step with MLA_IO_HOST, page-locked host memory), all inside the timed region
    h_y = torch.empty(B, D, dtype=bf).pin_memory()
    h_rows, h_pos, h_cu = row_idx.cpu().pin_memory(), positions.cpu().pin_memory(), cu.cpu().pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_x, h_rows, h_pos, h_cu))
    d2h = h_y.numel() * h_y.element_size()

    def e2e_step():
        layer(h_x, h_rows, h_pos, y=h_y, io=M.MLA_IO_HOST, cu_seqlens=h_cu)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
    # the two routes run the same kernels on the same inputs: their outputs agree bit for bit
    step()
    torch.cuda.synchronize()
    same_output = bool(torch.equal(h_y, y.cpu()))

    cpu = cpu_baseline() if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if world > 1:
        dist.barrier()
    if rank == 0:
        hbm, tflops, src = peaks()
        dec_avg_s = dec_mean_ms / 1e3
        achieved = cache_bytes() / dec_avg_s / 1e9
        tokens = world * nq * args.steps
        line = {
            "metric": METRIC, "value": tokens / (elapsed_ms / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": CONFIG,
            "roofline": {
                "kernel": "mla_decode_absorbed (split-KV decode + combine)",
                "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": recorded_traffic(),
                "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback",
                "algorithmic_bytes_per_launch": cache_bytes(),
                "decode_ms": dec_mean_ms,
                "decode_timing": "CUDA events around each of the K decode calls, in a second timed pass of the "
                                 "same K steps (events end the kernels' programmatic overlap, so the step-time "
                                 "pass has none); max over ranks",
                "tensor_tflops": decode_flops() / dec_avg_s / 1e12,
                "tensor_frac_of_measured_bf16": decode_flops() / dec_avg_s / 1e12 / tflops,
                "tensor_frac_of_sustained_bf16": decode_flops() / dec_avg_s / 1e12 / sustained_tflops(),
                "roofline_time_ms": 1e3 * max(cache_bytes() / (hbm * 1e9), decode_flops() / (tflops * 1e12)),
            },
            "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                    "route": "C ABI mla_decode_step with MLA_IO_HOST (page-locked host x, y, index arrays)",
                    "same_output_as_device_route": same_output},
            "gpu_launches": int(launches),
            "clocks": clk.summary(),
            "device_status": status,
        }
        line["roofline"]["frac_of_roofline_time"] = line["roofline"]["roofline_time_ms"] / line["roofline"]["decode_ms"]
        if line["clocks"]:
            # step time scaled by the sampled SM clock: comparable across boxes whose clocks differ
            line["clocks"]["ms_per_step_x_sm_mhz"] = line["ms_per_step"] * line["clocks"]["sm_mhz"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_rows(args):
    """Each step of the path on its own (the hot-path rows), timed with CUDA events around the C-ABI
    call, the L2 flushed between repetitions, against its roofline time max(bytes / HBM, FLOPs /
    tensor peak). One JSON line per row. Inputs are seeded and drawn on the device with the
    workloads' shapes and distributions; parity lives in the tests."""
    import torch
    from head_latent_attention_08_b200 import build, mla as M
    from head_latent_attention_08_b200 import inputs as I
    build.build()
    M.lib()
    dev = torch.device("cuda")
    bf, f32 = torch.bfloat16, torch.float32
    hbm, tflops, src = peaks()
    sustained = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops_sustained"]) \
        if src == "measured" else 1400.0
    gen = torch.Generator(device=dev).manual_seed(SEED)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clk = ClockSampler(torch.cuda.current_device()).__enter__()

    def rnd(*shape, scale=1.0, dtype=bf):
        return (torch.randn(*shape, device=dev, generator=gen) * scale).to(dtype)

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); fn(); b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def report(row, config, ms, nbytes, flops, note=""):
        t_mem, t_flop = nbytes / (hbm * 1e9), flops / (tflops * 1e12)
        bound = "hbm" if t_mem >= t_flop else "tensor"
        roof_ms = 1e3 * max(t_mem, t_flop)
        line = {"row": row, "config": config, "ms": ms, "bound": bound, "roofline_ms": roof_ms,
                "frac": roof_ms / ms, "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
                "tensor_tflops": flops / (ms * 1e-3) / 1e12 if flops else 0.0,
                "peaks": {"hbm_gbs": hbm, "bf16_tflops": tflops, "bf16_tflops_sustained": sustained,
                          "source": src},
                "frac_of_sustained_tensor": (flops / (sustained * 1e12)) * 1e3 / ms if flops else None}
        if note:
            line["note"] = note
        print(json.dumps(line), flush=True)

    # ---- C3: B64 H128 d_c512 d_r64 T4096, one query token per sequence --------------------------
    B, H, dc, dr, n, dv, D, T = 64, 128, 512, 64, 128, 128, 5120, 4096
    d = M.dims(H, dc, dr, n, dv, D)
    cache = rnd(B * T, dc + dr)
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=dev)
    w_uk, w_uv, w_o = rnd(H, n, dc, scale=n ** -0.5), rnd(H, dv, dc, scale=dc ** -0.5), rnd(D, H * dv, scale=(H * dv) ** -0.5)
    step = M.DecodeStep(d, bf, B, 1, T, cache, cu, w_uk, w_uv, w_o)
    q_nope, q_pe = rnd(B, H, n), rnd(B, H, dr)
    c_new, kpe_new = rnd(B, dc, dtype=f32), rnd(B, dr, dtype=f32)
    row_idx = torch.arange(B, device=dev, dtype=torch.int64) * T + T - 1
    positions = torch.full((B,), T - 1, dtype=torch.int32, device=dev)
    c3 = "C3 B64 H128 d_c512 d_r64 T4096 bf16"
    ms = timed(lambda: M.mla_append_latent(d, cache, row_idx, c_new, kpe_new, positions, step.append_flags))
    report("a1 latent append (RMSNorm + RoPE)", c3, ms, B * (dc + dr) * (4 + 2), 0,
           "64 rows: launch- and latency-bound, the roofline time is a few ns")
    ms = timed(lambda: M.mla_absorb_weights(d, M.MLA_ABSORB_QUERY, q_nope, q_pe, w_uk, B, step.q_abs))
    report("a2 query absorption", c3, ms, 2 * (H * n * dc + B * H * (n + dr) + B * H * (dc + dr)),
           2 * B * H * n * dc)
    ms = timed(lambda: M.mla_decode_absorbed(d, step.q_abs, cache, cu, B, 1, T, step.flags, step.out_lat,
                                             step.lse, step.ws_dec))
    report("a3+a4 split-KV decode + combine", c3, ms, B * T * (dc + dr) * 2, B * H * T * (2 * (dc + dr) + 2 * dc))
    ms = timed(lambda: M.mla_out_project(d, step.out_lat, w_uv, w_o, None, B, step.y, step.ws_out))
    report("a5 value + output projection", c3, ms, 4 * B * H * dc + 2 * (H * dv * dc + D * H * dv + B * D),
           2 * B * H * dv * dc + 2 * B * D * H * dv)
    ms = timed(lambda: step(q_nope, q_pe, c_new, kpe_new, row_idx, positions))
    report("a1..a5 whole decode step", c3, ms,
           B * T * (dc + dr) * 2 + 2 * (H * n * dc + H * dv * dc + D * H * dv),
           B * H * T * (2 * (dc + dr) + 2 * dc) + 2 * B * H * (n * dc + dv * dc) + 2 * B * D * H * dv)
    # ---- f2: the input projections fused with the append, and the whole step from x -----------------
    QR = 1536
    w_cq, w_qc = rnd(QR, D, scale=D ** -0.5), rnd(H * n, QR, scale=QR ** -0.5)
    w_qr, w_dkv = rnd(H * dr, QR, scale=QR ** -0.5), rnd(dc + dr, D, scale=D ** -0.5)
    x = rnd(B, D)
    qn2, qp2 = torch.empty(B, H, n, dtype=bf, device=dev), torch.empty(B, H, dr, dtype=bf, device=dev)
    ws_p = M.workspace(M.mla_project_workspace_size(d, bf, QR, B), dev)
    proj_w = QR * D + H * n * QR + H * dr * QR + (dc + dr) * D
    ms = timed(lambda: M.mla_project_inputs(d, QR, x, w_cq, w_qc, w_qr, w_dkv, positions, qn2, qp2, cache, row_idx,
                                            step.append_flags, ws_p))
    report("f2 input projections + append", c3 + " q_rank1536 d_model5120", ms,
           2 * (proj_w + B * D + B * H * (n + dr) + B * (dc + dr)), 2 * B * proj_w,
           "weight-read bound: 97 MB of projection weights for 64 tokens")
    layer = M.DecodeLayerStep(d, QR, B, T, cache, cu, w_cq, w_qc, w_qr, w_dkv, w_uk, w_uv, w_o)
    ms = timed(lambda: layer(x, row_idx, positions))
    report("f2 + a1..a5 whole step from x (mla_decode_step)", c3 + " q_rank1536 d_model5120", ms,
           B * T * (dc + dr) * 2 + 2 * (proj_w + H * n * dc + H * dv * dc + D * H * dv),
           B * H * T * (2 * (dc + dr) + 2 * dc) + 2 * B * (proj_w + H * (n * dc + dv * dc) + D * H * dv))
    # ---- f1: the same decode over an e4m3 cache (half the bytes; tensor cores with a bf16 query) --------
    codes = cache.view(torch.uint16)[:, : (dc + dr) // 2].contiguous().view(torch.uint8)   # any finite codes
    codes = (codes & 0x77)                                                                 # |value| <= 240
    ws8 = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, B, 1, T, B * T, M.MLA_DECODE_CAUSAL), dev)
    ms = timed(lambda: M.mla_decode_absorbed_fp8(d, step.q_abs, codes, 1.0, cu, B, 1, T, M.MLA_DECODE_CAUSAL,
                                                 step.out_lat, step.lse, ws8))
    report("f1 decode over an e4m3 cache (tensor cores)", c3, ms, B * T * (dc + dr),
           B * H * T * (2 * (dc + dr) + 2 * dc),
           "bf16 query split into two e4m3 parts for QK^T, P.C in f16 over the converted codes; bytes = the e4m3 "
           "cache; FLOPs counted once (the two query parts double the QK^T MMAs at twice the bf16 rate)")
    del codes, ws8
    # ---- f3: the context-parallel merge of R partial (out_lat, lse) pairs, parts local to this GPU -------
    for R in (2, 4):
        parts = [rnd(B, H, dc, dtype=f32) for _ in range(R)]
        lses = [rnd(B, H, dtype=f32) for _ in range(R)]
        ms = timed(lambda: M.mla_lse_merge(d, parts, lses, 0, B, step.out_lat, step.lse))
        report("f3 context-parallel merge (log-sum-exp)", c3 + f" R={R} parts", ms, 4 * (R + 1) * B * H * (dc + 1), 0,
               "every part read once, the result written once; across GPUs the parts are peers' buffers read "
               "over NVLink")
        del parts, lses
    del cache, step, w_o, layer, w_qc, w_qr
    torch.cuda.empty_cache()
    # ---- C4: B16, T ~ U[1024, 32768], n_q 1 and 4 (causal) -----------------------------------------
    Bs = 16
    lens = I.ragged_seqlens(Bs, 1024, 32768, seed=I.CONFIG_SEEDS[4])
    cu4 = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).to(dev)
    rows_total, tmax = int(lens.sum()), int(lens.max())
    cache4 = rnd(rows_total, dc + dr)
    for nq in (1, 4):
        q4 = rnd(Bs * nq, H, dc + dr)
        out4 = torch.empty(Bs * nq, H, dc, device=dev)
        lse4 = torch.empty(Bs * nq, H, device=dev)
        ws4 = M.workspace(M.mla_decode_workspace_size(d, bf, Bs, nq, tmax, rows_total, M.MLA_DECODE_CAUSAL), dev)
        ms = timed(lambda: M.mla_decode_absorbed(d, q4, cache4, cu4, Bs, nq, tmax, M.MLA_DECODE_CAUSAL, out4,
                                                 lse4, ws4))
        seen = sum(int(t) - nq + 1 + j for t in lens for j in range(nq))
        report("a3+a4 split-KV decode + combine", f"C4 B16 T~U[1024,32768] (sum {rows_total}) n_q {nq} causal",
               ms, rows_total * (dc + dr) * 2, H * seen * (2 * (dc + dr) + 2 * dc))
    del cache4
    torch.cuda.empty_cache()
    # ---- C5: gated prefill B4 S2048 D2048 H16 L512 (causal): the decode with n_q = S and the linears --
    B5, S5, D5, H5, L5 = 4, 2048, 2048, 16, 512
    d5 = M.dims(H5, L5, 0, D5 // H5, D5 // H5, D5, 1.0 / math.sqrt(D5 // H5))
    c5 = "C5 gated prefill B4 S2048 D2048 H16 L512 causal bf16"
    x = rnd(B5 * S5, D5)
    wq = rnd(D5, D5, scale=D5 ** -0.5)
    yq = torch.empty(B5 * S5, D5, dtype=bf, device=dev)
    ms = timed(lambda: M.mla_linear(x, wq, B5 * S5, D5, D5, 0, yq))
    report("a6 dense linear (Q = X Wq^T)", c5, ms, 2 * (B5 * S5 * D5 * 2 + D5 * D5), 2 * B5 * S5 * D5 * D5)
    q5 = rnd(B5 * S5, H5, L5)
    cache5 = rnd(B5 * S5, L5)
    cu5 = torch.arange(0, (B5 + 1) * S5, S5, dtype=torch.int32, device=dev)
    out5 = torch.empty(B5 * S5, H5, L5, device=dev)
    ws5 = M.workspace(M.mla_decode_workspace_size(d5, bf, B5, S5, S5, B5 * S5, M.MLA_DECODE_CAUSAL), dev)
    ms = timed(lambda: M.mla_decode_absorbed(d5, q5, cache5, cu5, B5, S5, S5, M.MLA_DECODE_CAUSAL, out5, None,
                                             ws5))
    seen5 = B5 * H5 * S5 * (S5 + 1) // 2
    report("a3+a4 split-KV decode + combine", c5 + " (n_q = S, rows = (token, head))", ms,
           B5 * S5 * L5 * 2 + B5 * S5 * H5 * L5 * (2 + 4), seen5 * (2 * L5 + 2 * L5))
    del q5, out5, ws5
    # ---- f4: the same prompt through the un-absorbed route -----------------------------------------
    Dh5 = D5 // H5
    k5, v5, g5, o5 = (rnd(B5 * S5, D5) for _ in range(4))
    ms = timed(lambda: M.mla_prefill_attention(yq, k5, v5, g5, B5, S5, H5, Dh5, 0.0, M.MLA_DECODE_CAUSAL, o5))
    report("f4 un-absorbed prefill attention (causal, gated)", c5 + " (heads of 128)", ms,
           4 * B5 * S5 * D5 * 2, seen5 * 4 * Dh5)
    wc5, wk5, wv5, wg5, wo5 = (rnd(L5, D5, scale=D5 ** -0.5), rnd(D5, L5, scale=L5 ** -0.5),
                               rnd(D5, L5, scale=L5 ** -0.5), rnd(D5, D5, scale=D5 ** -0.5),
                               rnd(D5, D5, scale=D5 ** -0.5))
    x5 = x.reshape(B5, S5, D5)
    lin_flops = 2 * B5 * S5 * (3 * D5 * D5 + D5 * L5 + 2 * L5 * D5)
    for route in ("unabsorbed", "absorbed"):
        attn = seen5 * 4 * (Dh5 if route == "unabsorbed" else L5)
        ms = timed(lambda: M.gated_mla(x5, wq, wc5, wk5, wv5, wg5, wo5, H5, True, route=route), reps=5)
        report(f"whole gated MLA prefill, {route} route", c5, ms, 2 * (B5 * S5 * (2 * D5 + L5) + 3 * D5 * D5),
               lin_flops + attn)
    clk.__exit__(None, None, None)
    print(json.dumps({"clocks": clk.summary(), "device_status": M.mla_check_status()}), flush=True)
    return 0


def run_profile_decode(args):
    """The decode call alone on the workload's shape (--batch sequences of 4096 positions, H 128), over a
    bf16 or an e4m3 cache: a fixed small case for profiler captures (ncu -k regex:tc_decode_kernel),
    not a benchmark line. Prints the median CUDA-event time of --steps calls after --warmup calls."""
    import torch
    from head_latent_attention_08_b200 import mla as M
    dev = torch.device("cuda")
    B, T, H, dc, dr = WORKLOAD["batch"], WORKLOAD["seqlen"], WORKLOAD["n_heads"], WORKLOAD["kv_lora_rank"], \
        WORKLOAD["rope_dim"]
    d = M.dims(H, dc, dr, WORKLOAD["qk_nope"], WORKLOAD["v_head"], WORKLOAD["d_model"])
    gen = torch.Generator(device=dev).manual_seed(SEED)
    vals = torch.randn(B * T, dc + dr, device=dev, generator=gen)
    q = torch.randn(B, H, dc + dr, device=dev, generator=gen).to(torch.bfloat16)
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=dev)
    out = torch.empty(B, H, dc, device=dev)
    lse = torch.empty(B, H, device=dev)
    flags = M.MLA_DECODE_CAUSAL
    if args.profile_decode == "e4m3":
        cache = vals.to(torch.float8_e4m3fn).view(torch.uint8)
        ws = M.workspace(M.mla_decode_workspace_size(d, torch.uint8, B, 1, T, B * T, flags), dev)

        def call():
            M.mla_decode_absorbed_fp8(d, q, cache, 1.0, cu, B, 1, T, flags, out, lse, ws)
    else:
        cache = vals.to(torch.bfloat16)
        ws = M.workspace(M.mla_decode_workspace_size(d, torch.bfloat16, B, 1, T, B * T, flags), dev)

        def call():
            M.mla_decode_absorbed(d, q, cache, cu, B, 1, T, flags, out, lse, ws)
    del vals
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); call(); b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    print(json.dumps({"profile_decode": args.profile_decode, "batch": B, "seqlen": T, "ms_median": statistics.median(ts),
                      "device_status": M.mla_check_status(), "note": "profiling case, not a benchmark line"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", action="store_true",
                    help="time each step of the path on its own against its roofline (one JSON line "
                         "per row) instead of the benchmark line")
    ap.add_argument("--profile-decode", choices=["bf16", "e4m3"], default=None,
                    help="run only the decode call over a bf16 or e4m3 cache (a profiler capture case)")
    ap.add_argument("--batch", type=int, default=WORKLOAD["batch"],
                    help="sequences per step (default 64: the benchmark workload; smaller batches "
                         "are for profiling captures and are not benchmark numbers)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.batch != WORKLOAD["batch"]:
        WORKLOAD["batch"] = args.batch
        CONFIG["batch"] = args.batch
        CONFIG["workload"] += f" [batch reduced to {args.batch}: profiling case, not the benchmark]"
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_decode:
        return run_profile_decode(args)
    if args.rows:
        return run_rows(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
