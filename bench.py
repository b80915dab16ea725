#!/usr/bin/env python
"""STCA forward throughput on one or more B200s, through the C ABI.

One step = stca_encode (the M history encodings, Eq. (2)) + stca_forward (the
M stacked single-query cross-attention layers with query fusion, Eqs. (3)-(8))
over one synthetic jagged batch shaped like the request-level-batched serving
workload: 64 requests, L = 10000 history tokens each, 16 targets per request,
d = 128, h = 8, M = 3, r = 4, bf16 storage with fp32 accumulation.

Prints ONE JSON line (rank 0): history-tokens/s over all ranks, the targets/s
companion, the roofline of the dominant kernel (timed live with CUDA events
around its launches), the whole-step roofline, an end-to-end figure through
the host-buffer entry point, the fp64 CPU oracle timed on a bounded sample, and
the SM clocks sampled during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config c1..c5]
Under torchrun (N > 1) every rank runs its own batch (weak scaling).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gen import CONFIGS, TRAIN_BATCH, make_config_workload, make_training_histories  # noqa: E402

METRIC = "STCA fwd history-tokens/s & targets/s at L=10k; % of HBM/tensor roofline"
UNIT = "history-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- counts
def counts(wl):
    """Algorithmic FLOPs and bytes of one step (encode + forward)."""
    N, T, d, h, M, rd = wl.N, wl.T, wl.d, wl.h, wl.M, wl.r * wl.d
    s = 2 if wl.dtype == "bf16" else 4
    TL = int(np.sum(wl.lengths.astype(np.int64) * wl.target_counts.astype(np.int64)))
    enc_flops = M * N * 6 * d * rd                     # GEMM1 (2 x 2 d rd) + GEMM2 (2 rd d)
    attn_flops = M * 4 * h * d * TL                    # u X~^T and alpha X~ over d, per head
    tgt_flops = T * 6 * rd * d + T * sum(
        8 * d * d + ((2 * (i + 2) * d * d + 6 * rd * d) if i + 1 < M else 0) for i in range(M))
    return {
        "N": N, "T": T, "TL": TL, "elem": s,
        "enc_flops": enc_flops, "attn_flops": attn_flops, "tgt_flops": tgt_flops,
        "tensor_flops": enc_flops + attn_flops + tgt_flops,
        "enc_bytes_per_layer": 2 * N * d * s,          # read X, write X~(i)
        "attn_bytes_per_layer": N * d * s,             # read X~(i) once for all T_r h rows
        "bytes_min": M * N * d * s,
        "bytes_materialised": (2 * M + 1) * N * d * s,
        "io_bytes": T * d * s + T * M * d * 4,
        # prediction head of Eq. (9): v W_Z, v' [zW_u | zW_g], h zW_d per target
        "head_flops": T * 2 * ((M + 1) * d * d + 3 * d * rd),
        # naive form (Eq. (12)) of the attention: K, V projection (4 L d^2) and the
        # packed query tiles' 64 head-group features (G = 64 / d_h heads per tile)
        "attn_flops_naive": M * sum(
            4 * int(L) * d * d + 4 * 128 * (h // (64 // (d // h))) *
            ((int(t) + 128 // (64 // (d // h)) - 1) // (128 // (64 // (d // h)))) * int(L) * 64
            for L, t in zip(wl.lengths, wl.target_counts) if t > 0) if (d // h) in (16, 32, 64) else None,
    }


# ----------------------------------------------------------------- clocks
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read only)."""

    def __init__(self, torch_device_index=0, period_s=0.01):
        self.samples, self.max_mhz, self.ok = [], None, False
        self.period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(torch_device_index)
            h = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            log(f"clock sampling unavailable: {e}")
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((sm, int(rs), util))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        bits = 0
        for s in loaded:
            bits |= s[1]
        reasons = sorted(n for b, n in _REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": float(statistics.median(s[0] for s in loaded)),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(loaded)}


# ----------------------------------------------------------------- oracle leg
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(wl, budget_s=15.0, seed=0):
    """Time the fp64 oracle on whole requests of `wl` until ~budget_s of CPU work."""
    from oracle import stca_oracle as O
    rng = np.random.default_rng(seed)
    order = [int(r) for r in rng.permutation(wl.R)]
    done, t0 = [], time.perf_counter()
    for r in order:
        O.forward_workload(wl, requests=[r])
        done.append(r)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    toks = int(sum(int(wl.lengths[r]) for r in done))
    tg = int(sum(int(wl.target_counts[r]) for r in done))
    return {"value": toks / dt, "unit": UNIT, "targets_per_s": tg / dt, "cores": blas_threads(),
            "kind": "oracle", "sample": f"{len(done)} of {wl.R} requests ({toks} history tokens, "
                                        f"{tg} targets) of the same workload, {dt:.1f} s"}


def oracle_one_thread(wl, budget_s=5.0, seed=1):
    """The same oracle sample with its BLAS pinned to one thread, or None when
    the thread count cannot be limited."""
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    with threadpool_limits(limits=1, user_api="blas"):
        s = oracle_sample(wl, budget_s=budget_s, seed=seed)
    return {"value": s["value"], "unit": s["unit"], "targets_per_s": s["targets_per_s"], "cores": 1,
            "sample": s["sample"]}


def run_reference(args, rank):
    """The oracle as the reference arm: each step runs it on a bounded sample."""
    if rank != 0:
        return
    wl = make_config_workload(args.config)
    from oracle import stca_oracle as O
    rng = np.random.default_rng(123)
    # one step = the oracle on `per_step` whole requests, sized to keep the run short
    t0 = time.perf_counter()
    O.forward_workload(wl, requests=[0])
    t1 = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)
    per_step = int(max(1, min(wl.R, budget // max(t1, 1e-6))))
    times, toks, tgs = [], 0, 0
    for it in range(args.warmup + args.steps):
        reqs = [int(x) for x in rng.choice(wl.R, size=per_step, replace=False)]
        s0 = time.perf_counter()
        O.forward_workload(wl, requests=reqs)
        dt = time.perf_counter() - s0
        if it >= args.warmup:
            times.append(dt)
            toks += int(sum(int(wl.lengths[r]) for r in reqs))
            tgs += int(sum(int(wl.target_counts[r]) for r in reqs))
    tot = sum(times)
    value = toks / tot
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "targets_per_s": tgs / tot,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: the oracle on {per_step} random whole requests "
                                   f"of the workload, on {cores} host threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, n):
    cfg = {"workload": wl.name, "R": wl.R, "history_tokens": wl.N, "targets": wl.T,
           "L": (int(wl.lengths[0]) if np.all(wl.lengths == wl.lengths[0])
                 else f"{int(wl.lengths.min())}..{int(wl.lengths.max())}"),
           "d": wl.d, "h": wl.h, "M": wl.M, "r": wl.r, "storage": wl.dtype,
           "parallelism": f"dp{n}"}
    s = 2 if wl.dtype == "bf16" else 4
    in_bytes = wl.N * wl.d * s
    if in_bytes * (wl.M + 1) > L2_BYTES:
        cfg["l2"] = (f"no flush: inputs larger than L2 (X {in_bytes / 1e6:.0f} MB and "
                     f"X~ {wl.M * in_bytes / 1e6:.0f} MB per step vs 126 MB L2)")
    else:
        cfg["l2"] = "L2 flushed between steps (256 MB write, outside each step's events)"
    return cfg


# ----------------------------------------------------------------- our arm
def to_dev(wl, a, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(wl.storage(a)))
    if wl.dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device)


def storage_weights(wl):
    out = {}
    for k, v in wl.weights.items():
        if v is None:
            out[k] = None
        elif isinstance(v, list):
            out[k] = [None if a is None else wl.storage(a) for a in v]
        else:
            out[k] = wl.storage(v)
    return out


KERNEL_SOURCES = {"encode": ("encode_tc.cu",), "attention": ("attn_tc_dev.cuh", "attn_tc.cu"),
                  "target_step": ("step_tc.cu", "target_step.cu")}


def source_hash(kind):
    """sha256 (first 16 hex digits) of a kernel class's sources: its files
    (KERNEL_SOURCES) followed by the shared tcgen05/TMA helper header."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind] + ("tc_common.cuh",):
        with open(os.path.join(ROOT, "target_attention_jagged_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kind, config_key):
    """DRAM bytes per launch from the committed ncu figures (profiles/traffic.json),
    or None when they are for another workload or the kernel's sources changed
    since.  The per-target class times combine + step together, so only the
    encoder and attention classes (one kernel per timed launch) carry a figure."""
    import json
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if kind not in ("encode", "attention") or not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    k = rec.get("kernels", {}).get(kind)
    if rec.get("workload") != config_key or not k:
        return None
    return int(k["dram_bytes_per_launch"]) if k.get("source_sha256_16") == source_hash(kind) else None


def roofline_of(kind, kt, c, wl, peaks, sustained, steps, config_key=None):
    """Roofline object of kernel class `kind` from its live event timings.

    Per launch, the algorithmic work is the class's per-step total divided by
    its launches per step (e.g. the encoder: M N 6 d rd FLOPs and 2 N d s bytes
    per layer; the attention: 4 h d sum_r T_r L_r FLOPs and N d s bytes per layer).
    The tensor-core encoder runs all M layers in one launch and reads X once:
    (M + 1) N d s bytes per launch.
    """
    ms, n = kt[kind]
    if n == 0 or ms <= 0:
        return None
    avg_s = ms / n / 1e3
    per_step = n / steps
    if kind == "encode":
        enc_bytes = (wl.M + 1) * c["N"] * wl.d * c["elem"] if per_step == 1 else \
            c["enc_bytes_per_layer"] * wl.M
        flops, bytes_ = c["enc_flops"] / per_step, enc_bytes / per_step
    elif kind == "attention":
        fl = c["attn_flops_naive"] if c.get("naive") else c["attn_flops"]
        flops, bytes_ = fl / per_step, c["attn_bytes_per_layer"] * wl.M / per_step
    elif kind == "pipe":
        # the two-half pipeline's launches: every attention layer of both halves,
        # beside most of the per-target steps
        flops = (c["attn_flops"] + c["tgt_flops"]) / per_step
        bytes_ = c["attn_bytes_per_layer"] * wl.M / per_step
    else:
        flops, bytes_ = c["tgt_flops"] / per_step, c["io_bytes"] / per_step
    traffic = recorded_traffic(kind, config_key) if wl.dtype == "bf16" else None
    base = {"kernel": kind, "traffic": traffic, "avg_launch_ms": avg_s * 1e3,
            "flops_per_launch": flops, "bytes_per_launch": bytes_}
    if wl.dtype == "f32":
        peak = 148 * 128 * 2 * 1.965e9 / 1e12     # FP32 FFMA lanes x clock (nominal)
        ach = flops / avg_s / 1e12
        return dict(base, bound="alu", achieved=ach, peak=peak, unit="TFLOP/s", frac=ach / peak,
                    peak_source="nominal FP32 FFMA: 148 SMs x 128 lanes x 2 x 1.965 GHz")
    tflops_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    ridge = tflops_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / bytes_ >= ridge:
        ach = flops / avg_s / 1e12
        return dict(base, bound="tensor", achieved=ach, peak=tflops_peak, unit="TFLOP/s",
                    frac=ach / tflops_peak,
                    peak_source="bf16_tflops_sustained" if sustained else "bf16_tflops")
    ach = bytes_ / avg_s / 1e9
    return dict(base, bound="hbm", achieved=ach, peak=peaks["hbm_gbs"], unit="GB/s",
                frac=ach / peaks["hbm_gbs"], peak_source="hbm_gbs")


def measure_train_batch(S, torch, dev, stream, peaks, steps):
    """The sparse-training batch builder on its workload (B = 256 users, L_avg =
    2000, L_max = L_infer = 10000, alpha = 0.02, d = 256 bf16): the host plan,
    the device gather of the packed stream (HBM-bound: every packed row is read
    once and written once, plus a 4-byte user index), and the STCA forward
    (encode + forward, 8 targets per user) over the packed batch."""
    cfg = TRAIN_BATCH
    beta, ss = S.stca_sl_beta(cfg["alpha"], cfg["L_min"], cfg["L_max"], cfg["L_avg"])
    th = make_training_histories(B=cfg["B"], hist=cfg["hist"], d=cfg["d"], alpha=cfg["alpha"],
                                 beta=beta, dtype=cfg["dtype"], seed=cfg["seed"])
    X = torch.from_numpy(th.storage(th.X)).view(torch.int16).view(torch.bfloat16).to(dev)
    args = (cfg["L_min"], cfg["L_max"], cfg["L_avg"], cfg["L_infer"])
    t0 = time.perf_counter()
    for _ in range(steps):
        plan = S.stca_sl_plan(th.hist_offsets, th.s, *args)
    plan_ms = (time.perf_counter() - t0) * 1e3 / steps
    P = int(plan["packed_offsets"][-1])
    src = torch.from_numpy(plan["src_start"]).to(dev)
    poff = torch.from_numpy(plan["packed_offsets"]).to(dev)
    Xp = torch.empty((P, cfg["d"]), dtype=torch.bfloat16, device=dev)
    seg = torch.empty(P, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            S.stca_sl_gather(X, src, poff, Xp, seg, stream)
        evs = []
        for _ in range(steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            S.stca_sl_gather(X, src, poff, Xp, seg, stream)
            b.record(stream)
            evs.append((a, b))
    torch.cuda.synchronize()
    g_ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    nbytes = 2 * P * cfg["d"] * 2 + 4 * P
    ach = nbytes / (g_ms / 1e3) / 1e9
    # the forward over the packed batch
    from gen import make_workload
    wl = make_workload(lengths=plan["lengths"].tolist(), targets=[cfg["targets"]] * cfg["B"],
                       d=cfg["d"], h=cfg["h"], M=cfg["M"], r=cfg["r"], dtype="bf16",
                       seed=cfg["seed"], name=cfg["name"])
    st = S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    xt = to_dev(wl, wl.targets, dev)
    Z = torch.empty((wl.T, wl.M, wl.d), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            st.encode(Xp, plan["packed_offsets"], stream)
            st.forward(xt, wl.target_offsets, Z, stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(steps):
            S.stca_sl_gather(X, src, poff, Xp, seg, stream)
            st.encode(Xp, plan["packed_offsets"], stream)
            st.forward(xt, wl.target_offsets, Z, stream)
        f1.record(stream)
    torch.cuda.synchronize()
    st.status(stream)
    st.close()
    step_ms = f0.elapsed_time(f1) / steps
    return {"workload": cfg["name"], "users": cfg["B"], "packed_rows": P,
            "sequence_sparsity": ss, "beta": beta, "plan_ms_host": plan_ms,
            "gather": {"ms": g_ms, "kernel": "sl_gather_kernel",
                       "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"],
                                    "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                                    "bytes_per_launch": nbytes, "peak_source": "hbm_gbs"}},
            "gather_encode_forward": {"ms": step_ms, "history_tokens_per_s": P / (step_ms / 1e3),
                                      "targets_per_s": wl.T / (step_ms / 1e3)}}


def shard_workload(full, rank, world):
    """Rank `rank`'s part of the batch `full`: whole requests, balanced by work
    with the library's partitioner (target_attention_jagged_b200.shard)."""
    import copy
    from target_attention_jagged_b200.shard import partition_requests, request_work, shard_offsets
    work = request_work(full.lengths, full.target_counts, full.d, full.h, full.M, full.r)
    reqs = partition_requests(work, world)[rank]
    x_rows, t_rows, off, toff = shard_offsets(full.offsets, full.target_offsets, reqs)
    wl = copy.copy(full)
    wl.lengths = full.lengths[reqs]
    wl.target_counts = full.target_counts[reqs]
    wl.offsets, wl.target_offsets = off, toff
    wl.X, wl.targets = full.X[x_rows], full.targets[t_rows]
    return wl


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import target_attention_jagged_b200 as S
    from target_attention_jagged_b200.shard import max_over_ranks

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.strong:
        # strong scaling: every rank draws the same batch and keeps the requests
        # the longest-processing-time partition gives it (no data-path collective)
        full = make_config_workload(args.config, seed=CONFIGS[args.config]["seed"])
        wl = shard_workload(full, rank, world)
        batch_N, batch_T = full.N, full.T
        cfg_wl = full
    else:
        wl = make_config_workload(args.config, seed=CONFIGS[args.config]["seed"] + 1000 * rank)
        batch_N, batch_T = world * wl.N, world * wl.T
        cfg_wl = wl
    c = counts(wl)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    st = S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    if args.attn_form:
        st.set_option(S.STCA_OPT_ATTN_FORM, args.attn_form)
    if args.attn_kernel is not None:
        st.set_option(S.STCA_OPT_ATTN_KERNEL, args.attn_kernel)
    if args.pipeline is not None:
        st.set_option(S.STCA_OPT_PIPELINE, args.pipeline)
    X = to_dev(wl, wl.X, dev)
    xt = to_dev(wl, wl.targets, dev)
    Z = torch.empty((wl.T, wl.M, wl.d), dtype=torch.float32, device=dev)
    s2 = 2 if wl.dtype == "bf16" else 4
    flush = None
    if wl.N * wl.d * s2 * (wl.M + 1) <= L2_BYTES:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    def step():
        if flush is not None:
            flush.fill_(1)
        st.encode_forward(X, wl.offsets, xt, wl.target_offsets, Z, stream)

    def timed_steps(n):
        """n steps on `stream`; device milliseconds of the steps themselves.
        With an L2 flush between steps, each step is bracketed by its own
        events after the flush, so the flush write is not counted."""
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                step()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b)
        evs = []
        for _ in range(n):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st.encode_forward(X, wl.offsets, xt, wl.target_offsets, Z, stream)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    st.status(stream)
    launches_per_step = st.get_option(S.STCA_OPT_LAUNCHES)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    with sampler, torch.cuda.stream(stream):
        local_ms = timed_steps(args.steps)
    if world > 1:
        dist.barrier()
    # per-kernel device times for the roofline: a second pass of the same steps
    # with events around every launch (kept out of the headline pass, where the
    # event records would add a gap at every kernel boundary)
    st.set_option(S.STCA_OPT_TIMING, 1)
    S.stca_kernel_times(st.handle)          # drop anything recorded so far
    with torch.cuda.stream(stream):
        timed_steps(args.steps)
    torch.cuda.synchronize()
    kt = {k: v for k, v in S.stca_kernel_times(st.handle).items() if v[1] > 0}
    st.set_option(S.STCA_OPT_TIMING, 0)
    naive_used = st.get_option(S.STCA_OPT_LAST_FORM) == 1
    c["naive"] = naive_used
    st.status(stream)
    elapsed_ms = max_over_ranks(local_ms, dev)
    sec = elapsed_ms / 1e3
    value = batch_N * args.steps / sec
    targets_per_s = batch_T * args.steps / sec
    sustained = sec > 1.0
    rooflines = {k: roofline_of(k, kt, c, wl, peaks, sustained, args.steps, args.config) for k in kt}
    for r_ in rooflines.values():
        if r_:
            r_["peak_source"] += f" ({peak_src})"
    dom = max(kt, key=lambda k: kt[k][0])
    roof = dict(rooflines[dom])
    tpeak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * 1e12
    t_flop = c["tensor_flops"] / tpeak
    t_bytes = c["bytes_materialised"] / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_flop, t_bytes)
    step_roof = {"t_roof_ms": t_roof * 1e3, "t_step_ms": elapsed_ms / args.steps,
                 "frac": t_roof / (sec / args.steps),
                 "bound": "tensor" if t_flop >= t_bytes else "hbm",
                 "tensor_flops": c["tensor_flops"], "bytes_materialised": c["bytes_materialised"],
                 "bytes_min": c["bytes_min"],
                 "frac_bytes_min": (c["bytes_min"] / (peaks["hbm_gbs"] * 1e9)) / (sec / args.steps)}

    # ---- forward only (the encoded history reused for a new set of targets)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        st.encode(X, wl.offsets, stream)
        st.forward(xt, wl.target_offsets, Z, stream)
        f0.record(stream)
        for _ in range(args.steps):
            st.forward(xt, wl.target_offsets, Z, stream)
        f1.record(stream)
    torch.cuda.synchronize()
    fwd_ms = f0.elapsed_time(f1) / args.steps

    # ---- prediction-head token of Eq. (9) on the forward's Z (outside the step)
    zout = torch.empty((wl.T, wl.d), dtype=torch.float32, device=dev)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        st.forward(xt, wl.target_offsets, Z, stream)
        for _ in range(3):
            st.head(xt, Z, zout, stream)
        h0.record(stream)
        for _ in range(args.steps):
            st.head(xt, Z, zout, stream)
        h1.record(stream)
    torch.cuda.synchronize()
    st.status(stream)
    head_ms = h0.elapsed_time(h1) / args.steps
    # the head fused into the last per-target step (stca_forward_head): its cost
    # is the difference to the plain forward on the same encoded history
    with torch.cuda.stream(stream):
        for _ in range(3):
            S.stca_forward_head(st.handle, xt, wl.target_offsets, Z, zout, stream)
        q0, q1, q2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        q0.record(stream)
        for _ in range(args.steps):
            st.forward(xt, wl.target_offsets, Z, stream)
        q1.record(stream)
        for _ in range(args.steps):
            S.stca_forward_head(st.handle, xt, wl.target_offsets, Z, zout, stream)
        q2.record(stream)
    torch.cuda.synchronize()
    st.status(stream)
    fused_head_ms = (q1.elapsed_time(q2) - q0.elapsed_time(q1)) / args.steps
    head_ach = c["head_flops"] / (head_ms / 1e3) / 1e12
    # bf16 handles with the tensor-core step run the head's products on the
    # tensor cores (step_tc_kernel, head only); the others on the CUDA cores
    head_tc = wl.dtype == "bf16" and wl.d in (128, 256) and wl.r * wl.d <= 512 and wl.M <= 8
    if head_tc:
        head_peak = peaks["bf16_tflops"]
        head_roof = {"bound": "tensor", "achieved": head_ach, "peak": head_peak, "unit": "TFLOP/s",
                     "frac": head_ach / head_peak, "flops_per_launch": c["head_flops"],
                     "peak_source": f"bf16_tflops ({peak_src})"}
    else:
        head_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        head_roof = {"bound": "alu", "achieved": head_ach, "peak": head_peak, "unit": "TFLOP/s",
                     "frac": head_ach / head_peak, "flops_per_launch": c["head_flops"],
                     "peak_source": "nominal FP32 FFMA: 148 SMs x 128 lanes x 2 x 1.965 GHz"}
    head = {"ms_per_head": head_ms, "targets_per_s": batch_T / (head_ms / 1e3),
            "fused_in_last_step_ms": fused_head_ms,
            "kernel": "step_tc_kernel (head products only)" if head_tc else "head_kernel",
            "inputs": "Z and weights L2-resident (back-to-back calls)",
            "roofline": head_roof}

    # ---- backward of layer 1 (history encoding and merged attention), synthetic loss
    backward = None
    if not args.no_backward:
        rng = np.random.default_rng(11)
        dXt = torch.from_numpy(rng.standard_normal((wl.N, wl.d)).astype(np.float32)).to(dev)
        rows = wl.T * wl.h
        Ub = torch.from_numpy((rng.standard_normal((rows, wl.d)) * (2.0 / np.sqrt(wl.d))).astype(np.float32)).to(dev)
        dC = torch.from_numpy(rng.standard_normal((rows, wl.d)).astype(np.float32)).to(dev)
        Qb = torch.from_numpy(rng.standard_normal((wl.T, wl.d)).astype(np.float32)).to(dev)
        dZb = torch.from_numpy(rng.standard_normal((wl.T, wl.d)).astype(np.float32)).to(dev)
        st.encode(X, wl.offsets, stream)
        with torch.cuda.stream(stream):
            for _ in range(2):
                S.stca_encode_backward(st.handle, 0, X, dXt, wl.d, wl.r * wl.d, stream=stream)
                S.stca_attention_backward(st.handle, 0, Ub, wl.target_offsets, dC, wl.N, stream)
                S.stca_output_backward(st.handle, 0, dC, dZb, wl.h, stream)
                S.stca_query_backward(st.handle, 0, Qb, Ub, wl.h, stream)
            b0, b1, b2, b3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
            nrep = max(1, min(args.steps, 5))
            b0.record(stream)
            for _ in range(nrep):
                S.stca_encode_backward(st.handle, 0, X, dXt, wl.d, wl.r * wl.d, stream=stream)
            b1.record(stream)
            for _ in range(nrep):
                S.stca_attention_backward(st.handle, 0, Ub, wl.target_offsets, dC, wl.N, stream)
            b2.record(stream)
            for _ in range(nrep):
                S.stca_output_backward(st.handle, 0, dC, dZb, wl.h, stream)
                S.stca_query_backward(st.handle, 0, Qb, Ub, wl.h, stream)
            b3.record(stream)
            # the query side of the step: the head (block M), the Eq. (7) fusion blocks
            # M-1 .. 1 (accumulating into dZ and dx_t), then the Eq. (3) query init
            dZf = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=dev)
            dxf = torch.zeros((wl.T, wl.d), dtype=torch.float32, device=dev)

            def query_side():
                for blk in range(wl.M, 0, -1):
                    S.stca_fusion_backward(st.handle, blk, Z, xt, dZb, wl.r * wl.d, dZ=dZf, dxt=dxf,
                                           accumulate=True, stream=stream)
                S.stca_query_init_backward(st.handle, xt, dZb, wl.r * wl.d, stream)
            query_side()
            b4 = torch.cuda.Event(enable_timing=True)
            b5 = torch.cuda.Event(enable_timing=True)
            b4.record(stream)
            for _ in range(nrep):
                query_side()
            b5.record(stream)
        torch.cuda.synchronize()
        st.status(stream)
        enc_ms, att_ms = b0.elapsed_time(b1) / nrep, b1.elapsed_time(b2) / nrep
        proj_ms = b2.elapsed_time(b3) / nrep
        qside_ms = b4.elapsed_time(b5) / nrep
        d_, rd_, T_ = wl.d, wl.r * wl.d, wl.T
        qside_fl = sum(6 * T_ * (b + 1) * d_ * d_ + 16 * T_ * d_ * rd_ for b in range(1, wl.M + 1)) + 18 * T_ * d_ * rd_
        rd = wl.r * wl.d
        enc_fl = 18 * wl.N * wl.d * rd              # recomputed forward (6 N d rd) + 6 backward products
        att_tc = wl.dtype == "bf16" and wl.d in (64, 128)
        if att_tc:
            # tensor cores: the forward attention for c and the row statistics (S, P X~),
            # then per (row, key) S, dP, P^T dC, dS^T U and dS X~: 14 d FLOPs
            att_fl = 14 * wl.d * c["TL"] * wl.h
        else:
            att_fl = 18 * wl.d * c["TL"] * wl.h     # per (row, key): 2 passes of 2 dots + dU; 2 dots + dX~
        tf32 = 1100.0
        fp32 = 148 * 128 * 2 * 1.965e9 / 1e12
        enc_bf16 = wl.dtype == "bf16" and wl.d % 64 == 0 and rd % 128 == 0
        backward = {
            "layer": 1, "loss": "synthetic <output, G>, G ~ N(0, 1)",
            "encode": ({"ms": enc_ms, "flops": enc_fl, "tflops": enc_fl / (enc_ms / 1e3) / 1e12,
                        "frac_of_measured_bf16": enc_fl / (enc_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                        "note": "tcgen05 bf16 GEMM (gemm_bf16_kernel, persistent, SwiGLU forward and "
                                "derivative in its epilogues) + the LayerNorm derivative kernel; "
                                "bf16 intermediates"}
                       if enc_bf16 else
                       {"ms": enc_ms, "flops": enc_fl, "tflops": enc_fl / (enc_ms / 1e3) / 1e12,
                        "frac_of_nominal_tf32": enc_fl / (enc_ms / 1e3) / 1e12 / tf32,
                        "note": "cuBLASLt products + SwiGLU / LayerNorm derivative kernels"}),
            "attention": ({"ms": att_ms, "flops": att_fl, "tflops": att_fl / (att_ms / 1e3) / 1e12,
                           "frac_of_measured_bf16": att_fl / (att_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                           "note": "tcgen05: the forward attention for c and the row statistics, delta = dC . c, "
                                   "then S, dP, dX~ = P^T dC + dS^T U and dU = dS X~ per key tile"}
                          if att_tc else
                          {"ms": att_ms, "flops": att_fl, "tflops": att_fl / (att_ms / 1e3) / 1e12,
                           "frac_of_nominal_fp32": att_fl / (att_ms / 1e3) / 1e12 / fp32,
                           "note": "CUDA-core flash-style kernels (softmax recomputed)"}),
            "projections": {"ms": proj_ms, "flops": 20 * wl.T * wl.d * wl.d,
                            "note": "output side (W_V, W_O) and query side (W_Q, W_K): TF32 products on "
                                    "tcgen05 (gemm_tf32_kernel) where both operands are K-major, cuBLASLt "
                                    "TF32 otherwise; the per-head slices as batches"},
            "query_side": {"ms": qside_ms, "flops": qside_fl,
                           "note": "the head (Eq. (9)), the M-1 fusion blocks (Eq. (7)) and the query init "
                                   "(Eq. (3)): TF32 products (gemm_tf32_kernel / cuBLASLt) + SwiGLU / "
                                   "LayerNorm derivative kernels; the query init on the bf16 GEMM"}}

    # ---- the sparse-training batch builder and a forward over its packed batch
    train_batch = None
    if not args.no_train_batch:
        train_batch = measure_train_batch(S, torch, dev, stream, peaks, args.steps)

    # ---- end to end through the host-buffer entry point
    Xh = torch.from_numpy(np.ascontiguousarray(wl.storage(wl.X))).pin_memory()
    th = torch.from_numpy(np.ascontiguousarray(wl.storage(wl.targets))).pin_memory()
    Zh = torch.empty((wl.T, wl.M, wl.d), dtype=torch.float32).pin_memory()
    for _ in range(min(args.warmup, 3)):
        S.stca_run_host(st.handle, Xh, wl.offsets, th, wl.target_offsets, Zh, stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(args.steps):
        S.stca_run_host(st.handle, Xh, wl.offsets, th, wl.target_offsets, Zh, stream)
    g1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(g0.elapsed_time(g1), dev)
    e2e = {"value": batch_N * args.steps / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size() + th.numel() * th.element_size()
                                     + 2 * 8 * (wl.R + 1)),
           "d2h_bytes_per_step": int(Zh.numel() * Zh.element_size()),
           "targets_per_s": batch_T * args.steps / (e2e_ms / 1e3)}
    st.close()

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if args.strong else "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) embeddings, Xavier-uniform weights)",
        "config": dict(workload_config(cfg_wl, world),
                       attn_form="naive (Eq. 12)" if naive_used else "reordered (Eq. 13)"),
        "targets_per_s": targets_per_s,
        "roofline": roof, "roofline_step": step_roof,
        "kernels": {k: {"ms_total": v[0], "launches": v[1]} for k, v in kt.items()},
        "kernel_timing": "second pass of the same steps with CUDA events around every launch",
        "forward_only": {"ms_per_forward": fwd_ms,
                         "targets_per_s": batch_T / (fwd_ms / 1e3),
                         "history_tokens_per_s": batch_N / (fwd_ms / 1e3)},
        "head": head,
        "train_batch": train_batch,
        "backward": backward,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": sampler.summary(),
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(wl, budget_s=args.cpu_budget)
        line["cpu_baseline"]["one_thread"] = oracle_one_thread(wl, budget_s=min(5.0, args.cpu_budget))
    print(json.dumps(line), flush=True)


def _pipe_used(S, st, xt, wl, Z):
    """Whether one forward of this batch ran the two-half pipeline."""
    st.set_option(S.STCA_OPT_TIMING, 1)
    S.stca_kernel_times(st.handle)
    st.forward(xt, wl.target_offsets, Z)
    n = S.stca_kernel_times(st.handle)["pipe"][1]
    st.set_option(S.STCA_OPT_TIMING, 0)
    return n > 0


def attn_paths_sweep():
    """Forward time with the CUDA-core attention path (STCA_OPT_ATTN_PATH 1,
    which also takes the CUDA-core per-target step) against the tensor-core
    path (2), over T_r * h, on bf16 batches shaped like the ragged 32-request
    config (L ~ U[200, 2000]) and like the serving config (L = 10000, 16
    requests); d 128, M 2, r 2.  Prints one JSON line per shape: the whole
    forward (min of 3 x 20 calls) and the attention launches alone (events
    around each launch), in ms, and the normwise difference of the two Z."""
    import torch
    import target_attention_jagged_b200 as S
    from gen import make_workload
    dev = torch.device("cuda:0")
    for shape, R, lengths in (("ragged-L200-2000", 32, ("uniform", 200, 2000)),
                              ("L10000", 16, ("fixed", 10000))):
        for h in (4, 8):
            for Tr in (1, 2, 4, 8, 16, 32):
                wl = make_workload(lengths=lengths, targets=("fixed", Tr), d=128, h=h, M=2, r=2,
                                   dtype="bf16", seed=11, R=R)
                rec = {"shape": shape, "R": R, "h": h, "T_r": Tr, "T_r_h": Tr * h, "N": wl.N}
                zs = {}
                with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
                    X, xt = to_dev(wl, wl.X, dev), to_dev(wl, wl.targets, dev)
                    st.encode(X, wl.offsets)
                    Z = torch.empty((wl.T, wl.M, wl.d), dtype=torch.float32, device=dev)
                    for path, name in ((1, "cuda_cores"), (2, "tensor_cores")):
                        st.set_option(S.STCA_OPT_ATTN_PATH, path)
                        for _ in range(5):
                            st.forward(xt, wl.target_offsets, Z)
                        torch.cuda.synchronize()
                        ts = []
                        for _ in range(3):
                            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                            a.record()
                            for _ in range(20):
                                st.forward(xt, wl.target_offsets, Z)
                            b.record()
                            torch.cuda.synchronize()
                            ts.append(a.elapsed_time(b) / 20)
                        pipelined = _pipe_used(S, st, xt, wl, Z)
                        # the attention launches alone, from a pass with the
                        # two-half pipeline off (its launches mix in the step)
                        st.set_option(S.STCA_OPT_PIPELINE, 0)
                        st.set_option(S.STCA_OPT_TIMING, 1)
                        S.stca_kernel_times(st.handle)
                        for _ in range(20):
                            st.forward(xt, wl.target_offsets, Z)
                        torch.cuda.synchronize()
                        kt = S.stca_kernel_times(st.handle)
                        st.set_option(S.STCA_OPT_TIMING, 0)
                        st.set_option(S.STCA_OPT_PIPELINE, 1)
                        st.status()
                        rec[name] = {"forward_ms": round(min(ts), 4),
                                     "attention_ms": round(kt["attention"][0] / 20, 4),
                                     "pipeline": pipelined}
                        zs[path] = Z.cpu().numpy()
                rec["z_rel_diff"] = float(np.linalg.norm(zs[1] - zs[2]) / np.linalg.norm(zs[2]))
                print(json.dumps(rec), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="c3", choices=sorted(CONFIGS))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attn-form", type=int, default=0, choices=[0, 1, 2],
                    help="attention form: 0 reordered (Eq. 13, default), 1 naive (Eq. 12), 2 auto")
    ap.add_argument("--attn-kernel", type=int, default=None, choices=[0, 1, 2],
                    help="tensor-core attention kernel (STCA_OPT_ATTN_KERNEL): 0 auto, "
                         "1 split-softmax + combine, 2 two-group; default: the library's choice")
    ap.add_argument("--strong", action="store_true",
                    help="strong scaling: one batch partitioned over the ranks by request "
                         "(shard.partition_requests); default: weak, a full batch per rank")
    ap.add_argument("--pipeline", type=int, default=None, choices=[0, 1],
                    help="STCA_OPT_PIPELINE: 1 two-half pipeline where it applies, 0 off; "
                         "default: the library's choice")
    ap.add_argument("--attn-paths", action="store_true",
                    help="only sweep the CUDA-core against the tensor-core attention path over "
                         "T_r * h (one GPU; JSON lines) and exit")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-train-batch", action="store_true",
                    help="skip the sparse-training batch builder measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: WORLD_SIZE={world} but --gpus={args.gpus}; using WORLD_SIZE")
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.attn_paths:
        if rank == 0:               # a one-GPU sweep: other ranks have nothing to do
            attn_paths_sweep()
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
