"""Benchmark of the Polar Attention hot path on B200.

One step = one pass of the whole path on one GPU's batch of synthetic input:
  * causal prefill, B=2, Hq=16, Hkv=4, T=16384, d=64, bf16, length temperature
    active (the extrapolation workload), through polar_attn_fwd_ws (the prefill
    with its key-moment workspace); then
  * paged GQA decode, 32 sequences with 128K-256K tokens of context in 64-token
    pages behind a shuffled page table, Hq=16, Hkv=4, bf16, through
    polar_attn_decode_paged.
value: prefill TFLOP/s (algorithmic flops of the visible causal triangle,
4*d per visible query-key pair) over all ranks / max-over-ranks prefill time;
decode.value: HBM GB/s (algorithmic KV bytes, 1024 per cached token per
sequence: K and V, 4 heads, 64 dims, bf16) likewise.  Times come from CUDA
events on the launching stream.  Multi-GPU (torchrun) runs independent
replicas, one batch per rank with its own seed ("scaling": "weak"); the only
collectives are the barrier and the max of the timings.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from polar_attention_b200 import workloads as W  # noqa: E402

METRIC = "Polar-attn fwd TFLOP/s & % BF16 peak at T=16K; decode HBM GB/s at 256K ctx"
PREFILL = W.EXTRAP
DECODE = W.DECODE
KV_BYTES_PER_TOKEN = DECODE.Hkv * DECODE.D * 2 * 2  # K and V, 4 heads, 64 dims, bf16: 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- plumbing --

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--only", choices=["both", "prefill", "decode", "gdelta"], default="both",
                    help="time one half of the step, or only the memory-channel legs "
                         "(profiling runs)")
    ap.add_argument("--prefill", choices=sorted(W.PREFILL_WORKLOADS), default=W.EXTRAP.name,
                    help="prefill workload (profiling runs use a smaller one)")
    ap.add_argument("--decode-seqs", type=int, default=W.DECODE.num_seqs,
                    help="decode sequences (profiling runs use fewer)")
    ap.add_argument("--bwd-steps", type=int, default=10,
                    help="timed launches of the prefill backward on the train-length workload "
                         "(0 skips it)")
    ap.add_argument("--gdelta-steps", type=int, default=20,
                    help="timed launches of the memory channel (prefill and decode step); 0 skips")
    ap.add_argument("--window", type=int, default=4096,
                    help="sliding window of the separately timed windowed prefill (0 skips it)")
    ap.add_argument("--per-head-steps", type=int, default=5,
                    help="timed launches of the test-only per-head decode (each page read once "
                         "per query head), for the grouped kernel's traffic saving; 0 skips it")
    ap.add_argument("--chunk", type=int, default=4,
                    help="query tokens per sequence of the separately timed multi-token decode "
                         "(0 skips it)")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch: weak scaling over independent problems."""
    return base + 1000 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_throughput(work_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return work_per_rank * world / max_seconds


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "polar_attention_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, sha: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the kernel as it is now (same source hash); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_sha") != sha:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_indices):
        # nvidia-smi numbers the GPUs of the host; name the process's own by UUID
        # where torch knows it, so that CUDA_VISIBLE_DEVICES does not matter.
        self.idx = []
        for i in gpu_indices:
            try:
                u = str(torch.cuda.get_device_properties(i).uuid)
                self.idx.append(u if u.startswith("GPU-") else "GPU-" + u)
            except Exception:  # noqa: BLE001
                self.idx.append(str(i))
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", ",".join(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None and self.proc.returncode is None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""
        return False

    def summary(self):
        if self.proc is None or not getattr(self, "out", ""):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = [r for r in csv.reader(io.StringIO(self.out)) if len(r) >= 10]
        sm, mx, reasons, load = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                s, m, util = float(r[1]), float(r[2]), float(r[4])
            except ValueError:
                continue
            mx.append(m)
            if util >= 50:
                load.append(s)
                for n, v in zip(names, r[6:10]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            sm.append(s)
        use = load if load else sm
        return {"sm_mhz": statistics.median(use) if use else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(load)}


class NvmlSampler:
    """The SM clock and the active clock-event reasons read through NVML about
    every millisecond, on a thread, while the timed step loop runs: at small
    step counts the whole loop is shorter than nvidia-smi's sampling interval.
    Read-only queries; the device is found by its UUID, so a remapped
    CUDA_VISIBLE_DEVICES still names the right GPU."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, dev):
        self.samples, self.max_mhz, self.err = [], None, None
        self._stop = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(dev).uuid)
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- NVML is optional; the record says why it is absent
            self.h, self.err = None, f"nvml unavailable: {type(e).__name__}"

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append((n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM),
                                     n.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception as e:  # noqa: BLE001
                self.err = f"nvml read failed: {type(e).__name__}"
                return
            self._stop.wait(0.001)

    def start(self):
        if self.h is None:
            return
        import threading
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        mhz = [m for m, _ in self.samples]
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


def clock_record(fast: NvmlSampler, smi: ClockSampler) -> dict:
    """The clock record of the line: NVML samples taken during the timed step
    loop where there are any, else nvidia-smi's; nvidia-smi's samples over all
    timed legs are kept beside them."""
    s = smi.summary()
    f = fast.summary()
    if f is None:
        return dict(s, source="nvidia-smi over the timed legs", nvml=fast.err)
    return dict(f, source="nvml during the timed step loop, about 1 ms apart", nvidia_smi=s)


# -------------------------------------------------------------- CPU oracle --

def _oracle_prefill_rows(x_host, rows, w):
    import oracle
    return oracle.polar_fwd(x_host["q"], x_host["k"], x_host["v"], x_host["u"],
                            oracle.Params(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta), rows=rows)


def prefill_rows_flops(rows, w) -> float:
    i = np.asarray(rows) % w.T
    return float(4.0 * w.D * np.sum(i + 1))


def gdelta_mma_flops(B: int, T: int, H: int) -> float:
    """bf16 tensor-core flops the memory-channel prefill executes per launch:
    per 64-token chunk and (sequence, head), 256 m16n8k16 products in the chunk
    kernel (K K^T and Q K^T) and 1056 in the scan (two slices of 32 value rows,
    each 320 for U = Ut + (-W) S^T with three hi/lo terms and Q S^T with two,
    80 for P U with two, 128 for the state update with two); 4096 flops each."""
    chunks = (T + 63) // 64
    return float(B) * H * chunks * (256 + 1056) * 4096.0


def gdelta_io_bytes(w) -> float:
    """Compulsory HBM bytes of one memory-channel prefill: q, k, v read and out
    written (bf16), alpha and beta read (fp32), the state read and written."""
    tok = w.B * w.T * w.H
    return float(tok * w.D * 2 * 4 + tok * 4 * 2 + w.B * w.H * w.D * w.D * 4 * 2)


def cpu_prefill_inputs(seed=0):
    x = W.prefill_inputs(PREFILL, "cpu", seed=seed)
    return {"q": W.to_host_bits(x["q"]), "k": W.to_host_bits(x["k"]), "v": W.to_host_bits(x["v"]),
            "u": x["u"].numpy()}


def oracle_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def calibrated_rows(x_host, budget_s: float, rng, probe_rows=32):
    """Seeded sample of prefill rows sized to about budget_s of oracle time."""
    total = PREFILL.B * PREFILL.Hq * PREFILL.T
    probe = rng.integers(0, total, size=probe_rows)
    t0 = time.perf_counter()
    _oracle_prefill_rows(x_host, probe, PREFILL)
    dt = max(time.perf_counter() - t0, 1e-3)
    n = int(max(probe_rows, min(200000, probe_rows * budget_s / dt)))
    return rng.integers(0, total, size=n)


def cpu_baseline(budget_s: float, seed=0) -> dict:
    x_host = cpu_prefill_inputs(seed)
    rng = np.random.default_rng(seed + 7)
    rows = calibrated_rows(x_host, budget_s, rng)
    t0 = time.perf_counter()
    _oracle_prefill_rows(x_host, rows, PREFILL)
    dt = time.perf_counter() - t0
    res = {"value": prefill_rows_flops(rows, PREFILL) / dt / 1e12, "unit": "TFLOP/s",
           "cores": oracle_threads(), "kind": "oracle",
           "sample": f"{rows.size} seeded random rows of the T=16384 prefill workload "
                     f"(fp64 two-pass oracle, {dt:.1f} s)"}
    res["decode"] = cpu_decode_baseline(seed)
    return res


def cpu_decode_baseline(seed=0, num_seqs=4) -> dict:
    """The decode oracle on `num_seqs` seeded sequences drawn from the decode
    workload's length range (every head of each), in algorithmic KV GB/s."""
    import oracle
    w = W.small_decode(num_seqs=num_seqs, min_len=DECODE.min_len, max_len=DECODE.max_len,
                       Hq=DECODE.Hq, Hkv=DECODE.Hkv, seed=seed + 5)
    x = W.decode_inputs(w, "cpu")
    q, kv = W.to_host_bits(x["q"]), W.to_host_bits(x["kv_pages"])
    pt, sl, u = x["page_table"].numpy(), x["seqlens"].numpy(), x["u"].numpy()
    prm = oracle.Params(s=w.s, alpha=w.alpha, L=w.L, beta=w.beta)
    t0 = time.perf_counter()
    oracle.polar_decode(q, kv, pt, sl, u, prm)
    dt = time.perf_counter() - t0
    kv_bytes = float(sl.astype(np.int64).sum()) * KV_BYTES_PER_TOKEN
    return {"value": kv_bytes / dt / 1e9, "unit": "GB/s", "cores": oracle_threads(),
            "kind": "oracle",
            "sample": f"{num_seqs} seeded sequences of {int(sl.min())}-{int(sl.max())} tokens, "
                      f"all {w.Hq} heads (fp64 oracle, {dt:.1f} s)"}


# ------------------------------------------------------------------ GPU arm --

def run_ours(args):
    import dataclasses

    import polar_attention_b200 as pa

    global PREFILL, DECODE
    PREFILL = W.PREFILL_WORKLOADS[args.prefill]
    DECODE = dataclasses.replace(W.DECODE, num_seqs=args.decode_seqs)
    do_pre = args.only in ("both", "prefill")
    do_dec = args.only in ("both", "decode")

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    seed = rank_seed(0, rank)
    if do_pre:
        xp = W.prefill_inputs(PREFILL, dev, seed=seed)
        out_p = torch.empty_like(xp["q"])
        neff_p = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.T), device=dev)
        ws_p = torch.empty(pa.fwd_workspace_size(PREFILL.B, PREFILL.T, PREFILL.Hq, PREFILL.Hkv),
                           device=dev, dtype=torch.uint8)
    kv_bytes, tokens = 0.0, 0
    if do_dec:
        xd = W.decode_inputs(DECODE, dev, seed=seed)
        out_d = torch.empty_like(xd["q"])
        neff_d = torch.empty((DECODE.num_seqs, DECODE.Hq), device=dev)
        ws = torch.empty(pa.decode_workspace_size(DECODE.num_seqs, xd["max_pages"], DECODE.Hq,
                                                  DECODE.Hkv), device=dev, dtype=torch.uint8)
        tokens = int(xd["seqlens"].to(torch.int64).sum().item())
        kv_bytes = float(tokens) * KV_BYTES_PER_TOKEN
    p = dict(s=PREFILL.s, alpha=PREFILL.alpha, L=PREFILL.L, beta=PREFILL.beta)

    def prefill():
        if not do_pre:
            return
        pa.fwd(xp["q"], xp["k"], xp["v"], xp["u"], out_p, neff_p, ws_p, stream=stream, **p)

    def decode():
        if not do_dec:
            return
        pa.decode_paged(xd["q"], xd["kv_pages"], xd["page_table"], xd["seqlens"], xd["u"], out_d,
                        neff_d, ws, stream=stream, **p)

    K, Wm = args.steps, args.warmup
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for _ in range(Wm):
        prefill()
        decode()
    torch.cuda.synchronize(dev)
    st = pa.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # The sampler runs through every timed leg below (the step loop alone is
    # shorter than its sampling interval at small K).
    clk = ClockSampler([dev.index]).__enter__()
    import atexit
    atexit.register(clk.__exit__, None, None, None)  # stop the sampler on any exit path
    time.sleep(0.3)  # let the sampler start before the timed region
    fast_clk = NvmlSampler(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    fast_clk.start()
    n0 = pa.launch_count()
    outer[0].record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        prefill()
        ev[i][1].record(stream)
        decode()
        ev[i][2].record(stream)
    outer[1].record(stream)
    torch.cuda.synchronize(dev)
    fast_clk.stop()
    launches = pa.launch_count() - n0
    barrier(world, dev)
    st = pa.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")

    t_pre = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / 1e3
    t_dec = sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / 1e3

    # ---- sliding-window prefill on the same inputs, timed on its own ----
    window_res = None
    if do_pre and 0 < args.window < PREFILL.T:
        wp = dataclasses.replace(PREFILL, window=args.window)

        def prefill_window():
            pa.fwd(xp["q"], xp["k"], xp["v"], xp["u"], out_p, neff_p, ws_p, stream=stream,
                   window=args.window, **p)

        for _ in range(Wm):
            prefill_window()
        torch.cuda.synchronize(dev)
        ew = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(K):
            ew[i][0].record(stream)
            prefill_window()
            ew[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        if pa.get_status() != 0:
            raise RuntimeError("device status after the windowed prefill")
        t_win = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ew) / 1e3, world, dev)
        window_res = (wp, t_win)

    # ---- the 8-argument polar_attn_fwd (no workspace) on the same inputs ----
    plain_res = None
    if do_pre:
        def prefill_plain():
            pa.fwd(xp["q"], xp["k"], xp["v"], xp["u"], out_p, neff_p, stream=stream,
                   moments=False, **p)

        for _ in range(Wm):
            prefill_plain()
        torch.cuda.synchronize(dev)
        ep = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(K):
            ep[i][0].record(stream)
            prefill_plain()
            ep[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        if pa.get_status() != 0:
            raise RuntimeError("device status after the 8-argument prefill")
        plain_res = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ep) / 1e3, world, dev)

    # ---- prefill backward on the train-length workload, timed on its own ----
    bwd_res = None
    if do_pre and args.bwd_steps > 0:
        wb = W.TRAIN
        xb = W.prefill_inputs(wb, dev, seed=seed + 1)
        gb = torch.randn(xb["q"].shape, device=dev, generator=torch.Generator(device=dev).manual_seed(seed)).to(xb["q"].dtype)
        gq = torch.empty(xb["q"].shape, device=dev)
        gk = torch.empty(xb["k"].shape, device=dev)
        gv = torch.empty(xb["v"].shape, device=dev)
        gu = torch.empty(xb["u"].shape, device=dev)
        wsb = torch.empty(pa.bwd_workspace_size(wb.B, wb.T, wb.Hq, wb.Hkv), device=dev,
                          dtype=torch.uint8)

        def backward():
            pa.bwd(xb["q"], xb["k"], xb["v"], xb["u"], gb, gq, gk, gv, gu, wsb, stream=stream,
                   s=wb.s, alpha=wb.alpha, L=wb.L, beta=wb.beta)

        for _ in range(min(Wm, 3)):
            backward()
        torch.cuda.synchronize(dev)
        Kb = args.bwd_steps
        eb = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kb)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(Kb):
            eb[i][0].record(stream)
            backward()
            eb[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        if pa.get_status() != 0:
            raise RuntimeError("device status after the backward")
        t_b = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in eb) / 1e3, world, dev)

        # The training pair: the forward that saves each row's state, then the
        # backward from that state (no forward sweep in the backward).
        ob = torch.empty_like(xb["q"])
        nb = torch.empty((wb.B, wb.Hq, wb.T), device=dev, dtype=torch.float32)
        sb = torch.empty((wb.B, wb.Hq, wb.T, 8), device=dev, dtype=torch.float32)

        def forward_train():
            pa.fwd_train(xb["q"], xb["k"], xb["v"], xb["u"], ob, nb, sb, stream=stream,
                         s=wb.s, alpha=wb.alpha, L=wb.L, beta=wb.beta)

        def backward_state():
            pa.bwd_from_state(xb["q"], xb["k"], xb["v"], xb["u"], ob, sb, gb, gq, gk, gv, gu, wsb,
                              stream=stream, s=wb.s, alpha=wb.alpha, L=wb.L, beta=wb.beta)

        def timed(fn):
            for _ in range(min(Wm, 3)):
                fn()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kb)]
            barrier(world, dev)
            torch.cuda.synchronize(dev)
            for i in range(Kb):
                ev[i][0].record(stream)
                fn()
                ev[i][1].record(stream)
            torch.cuda.synchronize(dev)
            barrier(world, dev)
            if pa.get_status() != 0:
                raise RuntimeError("device status after the training pair")
            return max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3, world, dev)

        t_ft = timed(forward_train)
        t_bs = timed(backward_state)
        bwd_res = (wb, Kb, t_b, t_ft, t_bs)
        del xb, gb, gq, gk, gv, gu, wsb, ob, nb, sb

    # ---- memory channel: chunked prefill and in-place decode step, timed on their own ----
    gd_res = None
    if args.gdelta_steps > 0:
        wg, wst = W.GD_TRAIN, W.GD_STEP
        xg = W.gdelta_inputs(wg, dev, seed=seed + 2)
        og = torch.empty_like(xg["q"])
        sg = torch.empty((wg.B, wg.H, wg.D, wg.D), device=dev)
        wsg = torch.empty(pa.gdelta_workspace_size(wg.B, wg.T, wg.H), device=dev,
                          dtype=torch.uint8)
        xs = W.gdelta_step_inputs(wst, dev, seed=seed + 3)
        os_ = torch.empty_like(xs["q"])

        def gd_prefill():
            sg.zero_()  # not timed: outside the events below
            pa.gdelta_prefill(xg["q"], xg["k"], xg["v"], xg["alpha"], xg["beta"], sg, og, wsg,
                              stream=stream)

        def gd_step():
            pa.gdelta_step(xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"], xs["state_pool"],
                           xs["slots"], os_, stream=stream)

        Kg = args.gdelta_steps
        times = []
        for fn in (gd_prefill, gd_step):
            for _ in range(max(Wm, 3)):
                fn()
            torch.cuda.synchronize(dev)
            eg = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kg)]
            barrier(world, dev)
            torch.cuda.synchronize(dev)
            for i in range(Kg):
                if fn is gd_prefill:
                    sg.zero_()
                eg[i][0].record(stream)
                if fn is gd_prefill:
                    pa.gdelta_prefill(xg["q"], xg["k"], xg["v"], xg["alpha"], xg["beta"], sg, og,
                                      wsg, stream=stream)
                else:
                    fn()
                eg[i][1].record(stream)
            torch.cuda.synchronize(dev)
            barrier(world, dev)
            if pa.get_status() != 0:
                raise RuntimeError("device status after the memory channel")
            times.append(max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in eg) / 1e3, world, dev))
        gd_res = (wg, wst, Kg, times[0], times[1])
        del xg, og, sg, wsg, xs, os_

    # ---- multi-token decode (chunk query tokens per sequence), timed on its own ----
    chunk_res = None
    if do_dec and args.chunk > 1:
        C = args.chunk
        qc = W.decode_chunk_queries(DECODE, xd, C, seed=seed)
        out_c = torch.empty_like(qc)
        neff_c = torch.empty((DECODE.num_seqs, C, DECODE.Hq), device=dev)
        ws_c = torch.empty(pa.decode_chunk_workspace_size(DECODE.num_seqs, xd["max_pages"], C,
                                                          DECODE.Hq, DECODE.Hkv),
                           device=dev, dtype=torch.uint8)

        def chunk_decode():
            pa.decode_paged_chunk(qc, xd["kv_pages"], xd["page_table"], xd["seqlens"], xd["u"],
                                  out_c, neff_c, ws_c, stream=stream, **p)

        for _ in range(Wm):
            chunk_decode()
        torch.cuda.synchronize(dev)
        ec = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(K):
            ec[i][0].record(stream)
            chunk_decode()
            ec[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        if pa.get_status() != 0:
            raise RuntimeError("device status after the multi-token decode")
        t_chunk = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ec) / 1e3, world, dev)
        chunk_res = (C, t_chunk)
    clk.__exit__(None, None, None)
    # ---- test-only per-head decode on the same cache, timed on its own ----
    per_head_res = None
    if do_dec and args.per_head_steps > 0:
        from polar_attention_b200 import native as N

        def per_head_decode():
            N.selftest_decode_per_head(xd["q"], xd["kv_pages"], xd["page_table"], xd["seqlens"],
                                       xd["u"], out_d, neff_d, ws, stream=stream, **p)

        for _ in range(min(Wm, 3)):
            per_head_decode()
        torch.cuda.synchronize(dev)
        Kh = args.per_head_steps
        eh = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kh)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for i in range(Kh):
            eh[i][0].record(stream)
            per_head_decode()
            eh[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        if pa.get_status() != 0:
            raise RuntimeError("device status after the per-head decode")
        per_head_res = (Kh, max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in eh) / 1e3, world,
                                           dev))
    t_all = outer[0].elapsed_time(outer[1]) / 1e3
    t_pre_max = max_over_ranks(t_pre, world, dev)
    t_dec_max = max_over_ranks(t_dec, world, dev)
    t_all_max = max_over_ranks(t_all, world, dev)

    # ---- end to end through the host-buffer C ABI (pinned host memory) ----
    e2e = None
    if args.e2e_steps > 0 and do_pre and do_dec:
        pin = lambda t: t.detach().cpu().pin_memory()  # noqa: E731
        hq, hk, hv, hu = pin(xp["q"]), pin(xp["k"]), pin(xp["v"]), pin(xp["u"])
        ho = torch.empty_like(hq).pin_memory()
        hn = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.T)).pin_memory()
        stg = torch.empty(pa.fwd_staging_size(PREFILL.B, PREFILL.T, PREFILL.Hq, PREFILL.Hkv),
                          device=dev, dtype=torch.uint8)
        dq, dpt, dsl, du = pin(xd["q"]), pin(xd["page_table"]), pin(xd["seqlens"]), pin(xd["u"])
        do = torch.empty_like(dq).pin_memory()
        dn = torch.empty((DECODE.num_seqs, DECODE.Hq)).pin_memory()
        dstg = torch.empty(pa.decode_staging_size(DECODE.num_seqs, xd["max_pages"], DECODE.Hq,
                                                  DECODE.Hkv), device=dev, dtype=torch.uint8)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hu, dq, dpt, dsl, du))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hn, do, dn))
        e_pre = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        tp = td = 0.0
        for i in range(args.e2e_steps + 1):
            barrier(world, dev)
            e_pre[0].record(stream)
            pa.fwd_host(hq, hk, hv, hu, ho, hn, stg, stream=stream, **p)
            e_pre[1].record(stream)
            torch.cuda.synchronize(dev)
            a = e_pre[0].elapsed_time(e_pre[1]) / 1e3
            e_pre[0].record(stream)
            pa.decode_paged_host(dq, xd["kv_pages"], dpt, dsl, du, do, dn, dstg, stream=stream, **p)
            e_pre[1].record(stream)
            torch.cuda.synchronize(dev)
            b = e_pre[0].elapsed_time(e_pre[1]) / 1e3
            if i > 0:  # the first is a warm-up
                tp += a
                td += b
        tp = max_over_ranks(tp, world, dev)
        td = max_over_ranks(td, world, dev)
        ns = args.e2e_steps
        e2e = {"value": aggregate_throughput(PREFILL.flops * ns, world, tp) / 1e12,
               "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "decode_value": aggregate_throughput(kv_bytes * ns, world, td) / 1e9,
               "decode_unit": "GB/s", "steps": ns,
               "note": "host-buffer C ABI calls (pinned), copies inside the timed region"}

    result = None
    if rank == 0:
        peaks, peak_src = measured_peaks()
        pre_launch_s = t_pre / K
        dec_launch_s = t_dec / K
        tf = PREFILL.flops / pre_launch_s / 1e12 if do_pre else 0.0
        gbs = kv_bytes / dec_launch_s / 1e9 if do_dec else 0.0
        sha_p = source_sha("fwd_tc.cu", "fwd_moments.cu", "polar_common.cuh", "tc_common.cuh",
                           "bwd_coef.cuh")
        sha_d = source_sha("decode.cu", "polar_common.cuh")
        value = aggregate_throughput(PREFILL.flops * K, world, t_pre_max) / 1e12 if do_pre else 0.0
        dec_value = aggregate_throughput(kv_bytes * K, world, t_dec_max) / 1e9 if do_dec else 0.0
        result = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": t_all_max / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": f"{PREFILL.describe()} + {DECODE.describe()}",
                "prefill": {"B": PREFILL.B, "T": PREFILL.T, "Hq": PREFILL.Hq, "Hkv": PREFILL.Hkv,
                            "head_dim": PREFILL.D, "alpha": PREFILL.alpha, "L_train": PREFILL.L,
                            "logit_scale": PREFILL.s, "flops_per_launch": PREFILL.flops},
                "decode": {"num_seqs": DECODE.num_seqs, "ctx": [DECODE.min_len, DECODE.max_len],
                           "Hq": DECODE.Hq, "Hkv": DECODE.Hkv, "page": W.PAGE,
                           "kv_bytes_per_launch": kv_bytes, "tokens": tokens},
                "l2": "inputs larger than L2: each step streams the 6.5 GB KV pool, which "
                      "evicts the prefill operands between prefill launches",
                "parallelism": f"replicas x{world} (one batch per rank)"},
            "prefill": {"value": value, "unit": "TFLOP/s", "ms_per_launch": pre_launch_s * 1e3,
                        "pct_bf16_peak": 100 * tf / peaks["bf16_tflops"],
                        "tokens_per_s": aggregate_throughput(PREFILL.B * PREFILL.T * K, world,
                                                             t_pre_max) if do_pre else 0.0},
            "decode": {"value": dec_value, "unit": "GB/s", "ms_per_launch": dec_launch_s * 1e3,
                       "pct_hbm_peak": 100 * gbs / peaks["hbm_gbs"],
                       "tokens_per_s": aggregate_throughput(DECODE.num_seqs * K, world,
                                                            t_dec_max) if do_dec else 0.0},
            "roofline": {"bound": "tensor", "kernel": "fwd_moments_kernel+fwd_tc_kernel",
                         "achieved": tf,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"],
                         "frac_of_sustained": tf / peaks.get("bf16_tflops_sustained",
                                                              peaks["bf16_tflops"]),
                         "traffic": profiled_traffic("prefill", sha_p),
                         "peak_source": f"{peak_src} (burst cuBLAS bf16)"},
            "roofline_decode": {"bound": "hbm", "kernel": "decode_split_kernel+decode_merge_kernel",
                                "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": gbs / peaks["hbm_gbs"],
                                "traffic": profiled_traffic("decode", sha_d),
                                "peak_source": f"{peak_src} (copy bandwidth)"},
            "gpu_launches": int(launches),
            "clocks": clock_record(fast_clk, clk),
            "e2e": e2e,
        }
        if bwd_res is not None:
            wb, Kb, t_b, t_ft, t_bs = bwd_res
            b_launch = t_b / Kb
            b_fl = 2.5 * wb.flops
            result["backward"] = {
                "workload": wb.describe(), "value": b_fl / b_launch / 1e12, "unit": "TFLOP/s",
                "ms_per_launch": b_launch * 1e3, "flops_per_launch": b_fl, "launches": Kb,
                "note": "prefill backward that recomputes each row's forward state (polar_attn_bwd: "
                        "dq, dk, dv, du; tcgen05 tensor cores for bf16 inputs), flops counted as "
                        "2.5x the forward's visible-pair flops; timed separately; not part of value"}
            ft_launch, bs_launch = t_ft / Kb, t_bs / Kb
            result["training_pair"] = {
                "workload": wb.describe(), "launches": Kb,
                "forward_train": {"ms_per_launch": ft_launch * 1e3,
                                  "value": wb.flops / ft_launch / 1e12, "unit": "TFLOP/s",
                                  "flops_per_launch": wb.flops},
                "backward_from_state": {"ms_per_launch": bs_launch * 1e3,
                                        "value": b_fl / bs_launch / 1e12, "unit": "TFLOP/s",
                                        "flops_per_launch": b_fl},
                "step": {"ms_per_launch": (ft_launch + bs_launch) * 1e3,
                         "value": 3.5 * wb.flops / (ft_launch + bs_launch) / 1e12,
                         "unit": "TFLOP/s"},
                "note": "polar_attn_fwd_train (forward that also saves each row's streaming state) "
                        "then polar_attn_bwd_from_state (backward from out and that state, no "
                        "forward sweep); flops: 1x and 2.5x the forward's visible-pair flops; "
                        "timed separately; not part of value"}
        if gd_res is not None:
            wg, wst, Kg, t_gp, t_gs = gd_res
            sha_g = source_sha("gdelta.cu", "polar_common.cuh", "tc_common.cuh")
            gp_launch, gs_launch = t_gp / Kg, t_gs / Kg
            tok = wg.B * wg.T
            # The recurrence's own arithmetic (S k, the rank-one write, S q:
            # 6 D^2 flops per token and head) against the fp32 CUDA-core peak;
            # the chunked kernels execute more (the triangular solve, hi/lo
            # splits) to expose parallelism, partly on the tensor cores.
            gp_tf = wg.flops / gp_launch / 1e12
            mma_fl = gdelta_mma_flops(wg.B, wg.T, wg.H)
            mma_tf = mma_fl / gp_launch / 1e12
            traffic_g = profiled_traffic("gdelta", sha_g)
            io_bytes = gdelta_io_bytes(wg)
            step_bytes = wst.state_bytes + wst.num_seqs * wst.H * wst.D * (4 * 2) + \
                wst.num_seqs * wst.H * 8 + wst.num_seqs * 4
            gs_gbs = step_bytes / gs_launch / 1e9
            result["gdelta"] = {
                "workload": wg.describe(), "ms_per_launch": gp_launch * 1e3,
                "tokens_per_s": aggregate_throughput(tok * Kg, world, t_gp),
                "recurrence_tflops": gp_tf,
                "note": "memory channel prefill (polar_gdelta_prefill: chunk kernel + scan kernel; "
                        "bf16 inputs, products on mma.sync with hi/lo-split fp32 operands), timed "
                        "separately; not part of value.  recurrence_tflops counts only the "
                        "recurrence's own 6 D^2 flops per token and head"}
            result["roofline_gdelta"] = {
                "bound": "tensor", "kernel": "gd_chunk_mma_kernel+gd_scan_mma_kernel",
                "achieved": mma_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": mma_tf / peaks["bf16_tflops"], "flops_per_launch": mma_fl,
                "traffic": traffic_g, "io_bytes_per_launch": io_bytes,
                "hbm_frac": (None if traffic_g is None else
                             traffic_g / gp_launch / 1e9 / peaks["hbm_gbs"]),
                "hbm_frac_of_io": io_bytes / gp_launch / 1e9 / peaks["hbm_gbs"],
                "peak_source": f"{peak_src} (burst cuBLAS bf16); flops = the bf16 m16n8k16 "
                               "products the kernels execute, every hi/lo term counted"}
            result["gdelta_step"] = {
                "workload": wst.describe(), "ms_per_launch": gs_launch * 1e3,
                "tokens_per_s": aggregate_throughput(wst.num_seqs * Kg, world, t_gs),
                "note": "in-place decode step (polar_gdelta_step), timed separately"}
            result["roofline_gdelta_step"] = {
                "bound": "hbm", "kernel": "gd_step_kernel", "achieved": gs_gbs,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gs_gbs / peaks["hbm_gbs"],
                "bytes_per_launch": step_bytes, "traffic": profiled_traffic("gdelta_step", sha_g),
                "peak_source": f"{peak_src} (copy bandwidth)"}
        if plain_res is not None:
            pl_launch = plain_res / K
            pl_tf = PREFILL.flops / pl_launch / 1e12
            result["prefill_no_workspace"] = {
                "value": pl_tf, "unit": "TFLOP/s", "ms_per_launch": pl_launch * 1e3,
                "pct_bf16_peak": 100 * pl_tf / peaks["bf16_tflops"],
                "traffic": profiled_traffic("prefill_no_workspace", sha_p),
                "note": "polar_attn_fwd(q, k, v, u, params, out, neff_out, stream): the same "
                        "prefill without the key-moment workspace (null-floor sums formed score "
                        "by score); timed separately after the step loop; not part of value"}
        if window_res is not None:
            wp, t_win = window_res
            w_launch = t_win / K
            w_tf = wp.flops / w_launch / 1e12
            result["prefill_window"] = {
                "window": wp.window, "value": w_tf, "unit": "TFLOP/s",
                "ms_per_launch": w_launch * 1e3, "flops_per_launch": wp.flops,
                "pct_bf16_peak": 100 * w_tf / peaks["bf16_tflops"],
                "note": "sliding-window prefill on the same T=16384 inputs, flops of the visible "
                        "(query, key) pairs; timed separately after the step loop, L2 warm from "
                        "the previous launch; not part of value"}
        if per_head_res is not None:
            Kh, t_h = per_head_res
            h_launch = t_h / Kh
            result["decode_per_head"] = {
                "ms_per_launch": h_launch * 1e3,
                "time_vs_grouped": h_launch / dec_launch_s,
                "kv_bytes_requested_per_launch": kv_bytes * DECODE.Hq / DECODE.Hkv,
                "note": "test-only polar_attn_selftest_decode_per_head: the same decode with one "
                        "query head per CTA, so each KV page is requested once per query head "
                        "(Hq/Hkv = 4 times per group); timed separately.  Concurrent CTAs of a "
                        "group share the re-reads in L2, so its DRAM bytes grow far less than 4x "
                        "(measured with ncu)"}
        if chunk_res is not None:
            C, t_chunk = chunk_res
            c_launch = t_chunk / K
            c_gbs = kv_bytes / c_launch / 1e9
            result["decode_chunk"] = {
                "chunk": C, "value": c_gbs, "unit": "GB/s", "ms_per_launch": c_launch * 1e3,
                "query_tokens_per_s": aggregate_throughput(DECODE.num_seqs * C * K, world, t_chunk),
                "pct_hbm_peak": 100 * c_gbs / peaks["hbm_gbs"],
                "note": "multi-token paged decode (polar_attn_decode_paged_chunk) on the same "
                        "32-sequence cache, timed separately after the step loop; not part of value"}
            result["roofline_decode_chunk"] = {
                "bound": "hbm", "kernel": "decode_split_kernel<4,16 rows>+decode_merge_kernel",
                "achieved": c_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": c_gbs / peaks["hbm_gbs"], "traffic": profiled_traffic("decode_chunk", sha_d),
                "peak_source": f"{peak_src} (copy bandwidth)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------- reference arm --

def run_reference(args):
    """The fp64 CPU oracle as it stands, on the host cores, on the same metric
    and unit: each step is a seeded sample of prefill rows, sized (as the
    cpu_baseline sample is) to keep every host core busy and the whole run
    within a few minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    x_host = cpu_prefill_inputs(0)
    rng = np.random.default_rng(11)
    total = PREFILL.B * PREFILL.Hq * PREFILL.T
    budget = min(6.0, 150.0 / max(1, args.steps + args.warmup))  # seconds per step
    rows_per_step = calibrated_rows(x_host, budget, rng, probe_rows=4 * oracle_threads()).size
    for _ in range(args.warmup):
        _oracle_prefill_rows(x_host, rng.integers(0, total, size=rows_per_step), PREFILL)
    flops = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        rows = rng.integers(0, total, size=rows_per_step)
        _oracle_prefill_rows(x_host, rows, PREFILL)
        flops += prefill_rows_flops(rows, PREFILL)
    dt = time.perf_counter() - t0
    v = flops / dt / 1e12
    sample = (f"{rows_per_step} seeded random rows of the T=16384 prefill per step "
              f"(fp64 two-pass oracle, {oracle_threads()} threads)")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": PREFILL.describe(), "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_ours(args)
        rank, world, _ = dist_env()
        if res is not None and args.only != "both":
            res["partial_step"] = (f"only the {args.only} legs were timed (profiling run)"
                                   if args.only == "gdelta" else
                                   f"only the {args.only} half was timed (profiling run)")
        if res is not None and world == 1 and not args.no_cpu_baseline and args.only == "both":
            res["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        elif res is not None:
            res["cpu_baseline"] = None
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
