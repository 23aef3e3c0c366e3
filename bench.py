#!/usr/bin/env python
"""Benchmark of the TwELL sparse ReLU-gated FFN forward pass on B200.

One step = one pass of the whole hybrid forward over one batch of synthetic
tokens: gate GEMM with the TwELL pack in its epilogue, routing, the fused
sparse up/down step for the rows that fit, and the dense branch for the rows
that overflow. Inputs are resident in HBM when the timed region starts; the
L2 is flushed between steps, outside the timed events: a 256 MiB buffer is
written and then read back, so the timed work starts from a cold L2 that holds
no dirty lines (a write alone leaves ~126 MB of the flush's own write-backs to
the first reads of the timed step).

Prints one JSON line (rank 0). Also measured in the same run: the library's
own dense FFN at the same shape (speedup denominator), the same metric end to
end through the C ABI with host buffers, and the CPU oracle on a bounded
sample of the workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 0.5b] [--impl twell|reference]
  python bench.py --sweep            # density x batch sweep, one JSON line per point
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from activation_sparse_gated_gemm_b200 import synth  # noqa: E402

METRIC = "sparse gated-FFN tokens/s"
METRIC_RELU = "sparse non-gated ReLU-FFN tokens/s"
METRIC_BWD = "sparse gated-FFN backward tokens/s"
FLUSH_BYTES = 256 << 20


def layer_config(args):
    """The configured layer, at --tokens tokens when given."""
    cfg = synth.CONFIGS[args.config]
    if getattr(args, "tokens", 0):
        cfg = dataclasses.replace(cfg, T=int(args.tokens), name=f"{cfg.name}-T{int(args.tokens)}")
    return cfg


def flush_l2(buf) -> None:
    """Evict L2: write a buffer larger than L2, then read it back, so the lines
    left in L2 are clean and the timed work pays no write-back of the flush."""
    import torch

    buf.zero_()
    buf.view(torch.int64).sum()
FP32_LANES_PER_SM = 128  # FP32 FMA lanes per SM (4 sub-partitions x 32)
DEFAULT_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                 "sm_max_mhz": 1965.0, "source": "fallback"}


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(DEFAULT_PEAKS)


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML every
    ~10 ms in a background thread (read-only queries)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self.max_mhz = None
        if index is None:  # a sampler that records nothing
            return
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 -- clocks are reported as unavailable
            self.max_mhz = None

    def _run(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), sm, reasons))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        mask = 0
        for _, _, r in self.samples:
            mask |= r
        names = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(s for _, s, _ in self.samples)),
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- helpers


# Device code of the forward kernels whose DRAM traffic profiles/traffic.json
# records (host code and the backward kernels, in other files, do not change
# them): a record taken on other sources is not reported.
FORWARD_SOURCES = ("ptx.cuh", "sparse_ffn.cuh", "umma_gemm.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_sparse_gated_gemm_b200", "csrc")
    for name in FORWARD_SOURCES:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources and this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
    except (OSError, ValueError):
        return None
    if t.get("source_hash") != kernel_source_hash() or t.get("workload") != workload:
        return None
    return t.get("kernels", {}).get(kernel)


UNIT_BYTES = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}


def record_traffic(csv_path: str, workload: str, kernels: list, command: str) -> dict:
    """profiles/traffic.json from an ncu raw-page CSV (`ncu -i rep --page raw
    --csv`): per bench stage, the mean over its captured launches of
    dram__bytes_read.sum + dram__bytes_write.sum, keyed to the current device
    sources. kernels: "stage=substring" pairs naming which captured kernel is
    which stage."""
    import csv

    with open(csv_path, newline="") as fh:
        rows = list(csv.reader(fh))
    head = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    cols = rows[head]
    kn = cols.index("Kernel Name")
    launches = {}  # launch id -> (kernel name, bytes)
    if "Metric Name" in cols:  # one row per (launch, metric): ncu --metrics ... --csv
        idc, mn, mu, mv = (cols.index(c) for c in ("ID", "Metric Name", "Metric Unit", "Metric Value"))
        for r in rows[head + 1:]:
            if len(r) > mv and r[mn] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
                v = float(r[mv].replace(",", "")) * UNIT_BYTES.get(r[mu], 1.0)
                name, b = launches.get(r[idc], (r[kn], 0.0))
                launches[r[idc]] = (name, b + v)
    else:  # one row per launch: ncu -i rep --page raw --csv (second row: units)
        units = rows[head + 1]
        rd, wr = cols.index("dram__bytes_read.sum"), cols.index("dram__bytes_write.sum")
        for i, r in enumerate(rows[head + 2:]):
            if len(r) > max(rd, wr):
                launches[i] = (r[kn], sum(float(r[c].replace(",", "")) * UNIT_BYTES.get(units[c], 1.0)
                                          for c in (rd, wr)))
    out = {}
    for pair in kernels:
        stage, sub = pair.split("=", 1)
        got = [b for name, b in launches.values() if sub in name]
        if not got:
            raise SystemExit(f"no captured launch of {sub!r} in {csv_path}")
        out[stage] = float(np.mean(got))
    rec = {"source_hash": kernel_source_hash(), "workload": workload, "command": command,
           "note": "dram__bytes_read.sum + dram__bytes_write.sum per launch (mean over the captured launches)",
           "kernels": out}
    with open(os.path.join(ROOT, "profiles", "traffic.json"), "w") as fh:
        json.dump(rec, fh, indent=1)
        fh.write("\n")
    return rec


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's value (replicas finish when the last one does)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, local_ms: float, world: int, device: str = "cuda") -> tuple:
    """Whole-job tokens/s of `world` independent replicas: all ranks' tokens
    over the slowest rank's step time. Returns (tokens/s, max ms)."""
    ms = max_over_ranks(local_ms, world, device)
    return job_rate(tokens_per_rank, world, ms), ms


def job_rate(tokens_per_rank: int, world: int, max_ms: float) -> float:
    return world * tokens_per_rank / (max_ms * 1e-3)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


# ---------------------------------------------------------------- CPU oracle


def oracle_step(cfg, L, rows, layer: str, dy=None) -> None:
    """One hybrid forward (or backward, given dy) of the oracle as it stands on the given rows."""
    from oracle import twell_oracle as O

    if dy is not None:
        O.hybrid_ffn_backward(L["x"][rows], L["WgT"], L["WuT"], L["Wd"], dy[rows], cfg.tile, cfg.W)
    elif layer == "relu":
        O.hybrid_relu_ffn(L["x"][rows], L["WgT"], L["Wd"], cfg.tile, cfg.W)
    else:
        O.hybrid_ffn(L["x"][rows], L["WgT"], L["WuT"], L["Wd"], cfg.tile, cfg.W)


def cpu_oracle_rate(cfg, L, sample_rows: int, layer: str = "gated", max_seconds: float = 25.0,
                    dy=None) -> dict:
    """The oracle as it stands (hybrid forward: fp64 gate, pack, route,
    per-token sparse step, dense rows; or the hybrid backward when dy is given)
    on the first rows of the workload."""
    n = min(sample_rows, cfg.T)
    done, t0 = 0, time.perf_counter()
    while done < n and time.perf_counter() - t0 < max_seconds:
        chunk = min(128, n - done)
        oracle_step(cfg, L, slice(done, done + chunk), layer, dy)
        done += chunk
    dt = time.perf_counter() - t0
    what = "hybrid backward" if dy is not None else "gate, pack, route, sparse step, dense rows"
    return {"value": done / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {done} of {cfg.T} tokens of the {cfg.name} {layer} layer, fp64 numpy oracle "
                      f"({what}), {dt:.1f} s"}


# ---------------------------------------------------------------- GPU arm


def algorithmic(cfg, n_ovf: int, nnz_stored: int, union_cols: int, layer: str = "gated") -> dict:
    T, d, f = cfg.T, cfg.d, cfg.f
    nT = f // cfg.tile
    mats = 2 if layer == "relu" else 3         # weight matrices of the layer
    gate_flops = 2.0 * T * d * f
    dense_branch_flops = 2.0 * mats * n_ovf * d * f
    alg_bytes = (2.0 * d * f                  # Wg (W1)
                 + 2.0 * (mats - 1) * d * union_cols  # active Wu columns and Wd rows (W2 rows)
                 + 6.0 * T * d                # x read (bf16), y written (fp32)
                 + 2 * 4.0 * nnz_stored       # TwELL nonzeros written and read (2 B idx + 2 B value)
                 + 2 * 2.0 * T * nT)          # counts written and read
    # up and down for every stored slot (non-overflow rows); down only without the up matrix
    sparse_flops = 2.0 * (mats - 1) * d * nnz_stored
    return {"gate_flops": gate_flops, "dense_branch_flops": dense_branch_flops, "alg_bytes": alg_bytes,
            "sparse_flops": sparse_flops}


def run_gpu(args, world, rank, local):
    import torch

    from activation_sparse_gated_gemm_b200 import twell as tl

    tl.load()
    dev = torch.device("cuda", local)
    cfg = layer_config(args)
    L = synth.make_layer(cfg, seed=args.seed)
    x = tl.to_device_bf16(L["x"], dev)
    WgT = tl.to_device_bf16(L["WgT"], dev)
    WuT = tl.to_device_bf16(L["WuT"], dev)
    Wd = tl.to_device_bf16(L["Wd"], dev)
    compact_info = None
    if args.compact:
        # drop the hidden units that the batch never activates (a one-time model
        # transformation, outside the timed region); the layer then has f_c units
        c = tl.compact_layer(x, {"WgT": WgT, "WuT": WuT, "Wd": Wd}, tl.new_status(dev))
        WgT, WuT, Wd = c["WgT"], c["WuT"], c["Wd"]
        compact_info = {"f_orig": cfg.f, "f_live": c["f_live"], "f_c": c["f_c"],
                        "profile": "the timed batch itself"}
        cfg = dataclasses.replace(cfg, f=c["f_c"])
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    tw = tl.Twell(T, f, W, device=dev)
    y = torch.empty((T, d), dtype=torch.float32, device=dev)
    ovf_rows = torch.empty((T,), dtype=torch.int32, device=dev)
    n_ovf = torch.zeros((1,), dtype=torch.int32, device=dev)
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device=dev)
    ws_dense = torch.empty(tl.dense_workspace_bytes(T, d, f), dtype=torch.uint8, device=dev)
    y_dense = torch.empty_like(y)
    st = tl.new_status(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # The two forms of the hybrid forward: "gate" packs ReLU(z) and runs the
    # fused sparse up+down step; "tc_up" forms u on the tensor cores with the
    # gate and packs h, leaving only the down projection sparse.
    # the down projection of the tc_up and non-gated forms (per token; the
    # union form on the tensor cores is an explicit entry point the forwards
    # do not use)
    def down():
        tl.sparse_down(Wd, tw, y, True, st)

    def stage_fns(variant):
        if variant == "relu":  # the non-gated layer ReLU(x W1) W2 with W1 = Wg, W2 = Wd
            return [lambda: tl.gate_pack(x, WgT, tw, st), lambda: tl.route(tw, ovf_rows, n_ovf), down,
                    lambda: tl.relu_dense_rows_forward(x, WgT, Wd, ovf_rows, n_ovf, y, ws, st)]
        pack = ((lambda: tl.gate_pack(x, WgT, tw, st)) if variant == "gate"
                else (lambda: tl.gate_up_pack(x, WgT, WuT, tw, st)))
        sparse = (lambda: tl.sparse_ffn(x, WuT, Wd, tw, y, True, st)) if variant == "gate" else down
        return [pack, lambda: tl.route(tw, ovf_rows, n_ovf), sparse,
                lambda: tl.dense_rows_forward(x, WgT, WuT, Wd, ovf_rows, n_ovf, y, ws, st)]

    def forward_fn(variant):
        # the library's whole hybrid forward of this form: the timed step
        if variant == "relu":
            return lambda: tl.relu_ffn_hybrid_forward(x, WgT, Wd, tw, y, ovf_rows, n_ovf, ws, st)
        if variant == "gate":
            return lambda: tl.ffn_hybrid_forward(x, WgT, WuT, Wd, tw, y, ovf_rows, n_ovf, ws, st)
        return lambda: tl.ffn_hybrid_forward_tc_up(x, WgT, WuT, Wd, tw, y, ovf_rows, n_ovf, ws, st)

    def timed_steps(fns, sampler=None):
        # K steps of fns in order, an event after each; L2 flushed before each step
        K, Wm = args.steps, args.warmup
        for _ in range(Wm):
            flush_l2(flush)
            for fn in fns:
                fn()
        torch.cuda.synchronize(dev)
        if tl.status_get(st) != 0:
            raise RuntimeError(f"device status {tl.status_get(st)} after warm-up")
        n = len(fns)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize(dev)
        ctx = sampler if sampler is not None else ClockSampler(None)
        with ctx:
            for k in range(K):
                flush_l2(flush)
                evs[k][0].record(stream)
                for i, fn in enumerate(fns):
                    fn()
                    evs[k][i + 1].record(stream)
            torch.cuda.synchronize(dev)
        barrier(world)
        return np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(n)] for k in range(K)])

    def run_variant(variant, sampler=None):
        # median step over the K timed steps of the whole forward
        per = timed_steps([forward_fn(variant)], sampler)
        return max_over_ranks(float(np.median(per[:, 0])), world)

    layer = "relu" if args.layer == "relu" else "gated"
    if layer == "relu":
        variants = ["relu"]
    else:
        variants = ["gate", "tc_up"] if args.variant == "auto" else [args.variant]
    results = {v: run_variant(v) for v in variants} if len(variants) > 1 else {}
    chosen = min(results, key=lambda v: results[v]) if results else variants[0]
    # the reported measurement: the chosen form, timed again with the clocks sampled
    sampler = ClockSampler(local)
    results[chosen] = run_variant(chosen, sampler)
    step_ms = results[chosen]
    # the stage breakdown: the same steps through the stage entry points, one
    # after the other (the tc_up forward's dense branch reuses the gate+up
    # GEMM's h; the separate dense-rows entry point recomputes it)
    stage_ms = np.median(timed_steps(stage_fns(chosen)), axis=0)
    K, Wm = args.steps, args.warmup

    # stats of this batch (for the algorithmic byte and FLOP counts)
    counts = tw.counts.to(torch.int64)
    n_ovf_h = int(n_ovf.item())
    ovf_mask = tw.row_ovf.bool()
    stored = torch.clamp(counts, max=W)
    nnz_stored = int(stored[~ovf_mask].sum())
    g = torch.empty((T, f), dtype=torch.bfloat16, device=dev)
    tl.unpack(tw, g, st)
    keep = ~ovf_mask
    act = (g[keep] != 0).any(dim=0)
    union_cols = int(act.sum())
    del g

    # dense baseline at the same shape
    def dense():
        if layer == "relu":
            tl.relu_dense_ffn_forward(x, WgT, Wd, y_dense, ws_dense, st)
        else:
            tl.dense_ffn_forward(x, WgT, WuT, Wd, y_dense, ws_dense, st)

    for _ in range(Wm):
        flush_l2(flush)
        dense()
    dense_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(world)
    for k in range(K):
        flush_l2(flush)
        dense_ev[k][0].record(stream)
        dense()
        dense_ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = max_over_ranks(float(np.median([a.elapsed_time(b) for a, b in dense_ev])), world)

    # End to end through the C ABI with host buffers: every step copies its x
    # from pinned host memory, runs the hybrid forward and copies y back to
    # pinned host memory. Two device buffer sets and separate copy-in,
    # compute and copy-out streams (ordered by events) let step k+1's input
    # copy and step k-1's output copy run under step k's compute, as a
    # host-fed pipeline would. Timed from the first copy-in to the last
    # copy-out; each step touches ~0.26 GB (> the 126 MB L2), so no flush.
    if layer == "relu":
        def hybrid(x, WgT, WuT, Wd, *rest):
            tl.relu_ffn_hybrid_forward(x, WgT, Wd, *rest)
    else:
        hybrid = tl.ffn_hybrid_forward if chosen == "gate" else tl.ffn_hybrid_forward_tc_up
    x_host = x.cpu().pin_memory()
    xs = [x, torch.empty_like(x)]
    ys = [y, torch.empty_like(y)]
    y_hosts = [torch.empty((T, d), dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipeline(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_cmp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        start = torch.cuda.Event(enable_timing=True)
        start.record(s_in)
        for k in range(nsteps):
            b = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_cmp[k - 2])  # the compute that read xs[b] is done
                xs[b].copy_(x_host, non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if k >= 2:
                stream.wait_event(ev_out[k - 2])  # ys[b] has been copied out
            hybrid(xs[b], WgT, WuT, Wd, tw, ys[b], ovf_rows, n_ovf, ws, st)
            ev_cmp[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[k])
                y_hosts[b].copy_(ys[b], non_blocking=True)
                ev_out[k].record(s_out)
        return start, ev_out[-1]

    torch.cuda.synchronize(dev)
    pipeline(max(2, Wm))
    torch.cuda.synchronize(dev)
    barrier(world)
    a, b_ev = pipeline(K)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b_ev) / K, world)
    status = tl.status_get(st)
    if status != 0:
        raise RuntimeError(f"device status {status} ({tl.status_str(status)})")

    peaks = load_peaks()
    alg = algorithmic(cfg, n_ovf_h, nnz_stored, union_cols, layer)
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops"] * 1e12
    t_tc = (alg["gate_flops"] + alg["dense_branch_flops"]) / tc
    t_hbm = alg["alg_bytes"] / hbm
    t_roof = max(t_tc, t_hbm)
    clocks = sampler.summary()
    fp32_peak = (torch.cuda.get_device_properties(dev).multi_processor_count * FP32_LANES_PER_SM * 2
                 * (clocks["sm_max_mhz"] or peaks.get("sm_max_mhz", 1965.0)) * 1e6)

    if chosen == "relu":
        names = ["gate_pack", "route", "sparse_down", "dense_rows"]
        pack_flops, sparse_flops = alg["gate_flops"], alg["sparse_flops"]
    elif chosen == "gate":
        names = ["gate_pack", "route", "sparse_ffn", "dense_rows"]
        pack_flops, sparse_flops = alg["gate_flops"], alg["sparse_flops"]
    else:
        names = ["gate_up_pack", "route", "sparse_down", "dense_rows"]
        pack_flops, sparse_flops = 2 * alg["gate_flops"], alg["sparse_flops"] / 2
    kern = {
        names[0]: {"bound": "tensor", "work": pack_flops, "peak": tc, "unit": "TFLOP/s", "scale": 1e12},
        names[2]: {"bound": "alu", "work": sparse_flops, "peak": fp32_peak, "unit": "TFLOP/s", "scale": 1e12},
        "dense_rows": {"bound": "tensor", "work": alg["dense_branch_flops"], "peak": tc, "unit": "TFLOP/s",
                       "scale": 1e12},
    }
    sparse_flops_path = alg["sparse_flops"] if chosen in ("gate", "relu") else alg["sparse_flops"] / 2
    # weight rows the sparse step gathers: Wu and Wd rows in the gate form, Wd rows otherwise
    gathered_rows = nnz_stored * (2 if chosen == "gate" else 1)
    dom = max((names[0], names[2], "dense_rows"), key=lambda n: stage_ms[names.index(n)])
    kd = kern[dom]
    ms = float(stage_ms[names.index(dom)])
    achieved = kd["work"] / (ms * 1e-3) / kd["scale"]
    peak = kd["peak"] / kd["scale"]
    traffic = measured_traffic(dom, cfg.name)

    res = {
        "metric": METRIC_RELU if layer == "relu" else METRIC,
        "value": job_rate(T, world, step_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded generator; no dataset or trained weights)",
        "config": {"workload": (f"{cfg.name}-like non-gated ReLU FFN layer forward (W1 = Wg, W2 = Wd), "
                                "hybrid TwELL" if layer == "relu" else
                                f"{cfg.name}-like FFN layer forward, hybrid TwELL")
                               + (f", dead units dropped (f {compact_info['f_orig']} -> {cfg.f})"
                                  if compact_info else ""), "variant": chosen, "compaction": compact_info,
                   "tokens": T, "d": d,
                   "f": f, "tile": cfg.tile, "ell_width": W, "density": cfg.density,
                   "dead_frac": cfg.dead_frac, "l2": "flushed between steps (256 MiB written, then read back so that no dirty line is left; outside events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "roofline": {"kernel": dom, "bound": kd["bound"], "achieved": achieved, "peak": peak, "unit": kd["unit"],
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": ("fp32 FMA lanes x 2 x max SM clock" if kd["bound"] == "alu"
                                     else f"{peaks['source']} bf16 burst"),
                     # the sparse step's real limit: weight rows gathered from L2 (2 bytes x d per
                     # stored slot and gathered matrix)
                     "l2_gather_tbs": (gathered_rows * 2.0 * d / (float(stage_ms[names.index(names[2])]) * 1e-3)
                                       / 1e12)},
        "path_roofline": {"t_tensor_us": t_tc * 1e6, "t_hbm_us": t_hbm * 1e6, "t_roof_us": t_roof * 1e6,
                          "frac": t_roof / (step_ms * 1e-3),
                          # the method's own second bound: the sparse step's FLOPs on the CUDA cores
                          "t_simt_us": sparse_flops_path / fp32_peak * 1e6,
                          "frac_with_simt": max(t_roof, sparse_flops_path / fp32_peak) / (step_ms * 1e-3),
                          "frac_gate_only": (alg["gate_flops"] / tc) / (step_ms * 1e-3),
                          "peaks": f"{peaks['source']}: {peaks['hbm_gbs']} GB/s, {peaks['bf16_tflops']} TF/s"},
        "stages_ms": {n: float(v) for n, v in zip(names, stage_ms)},
        "stages_source": ("the stage entry points called one after the other; the timed step is the library's "
                          "whole hybrid forward (whose tc_up dense branch reuses the gate+up GEMM's h, where the "
                          "separate dense-rows entry point recomputes it)"),
        "variants_ms": {v: results[v] for v in results},
        "dense_ffn_ms": dense_ms,
        "speedup_vs_own_dense": dense_ms / step_ms,
        "batch_stats": {"n_ovf": n_ovf_h, "nnz_stored": nnz_stored, "union_cols": union_cols,
                        "mean_density": float(counts.sum()) / (T * f)},
        "e2e": {"value": job_rate(T, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 4,
                "pipelined": "copy-in, compute and copy-out on three streams, two buffer sets",
                "path": "the library's hybrid forward of the chosen form",
                "l2": "not flushed: each step touches ~0.26 GB, above the 126 MB L2"},
        # per step: zeroing, the pack GEMM, routing, the sparse step, then the dense branch: the gate form's row
        # gather and two GEMMs, or (tc_up and the non-gated layer, which take the routed rows' h from the pack
        # GEMM) the fill of their other tiles and one down GEMM
        "gpu_launches": (7 if chosen == "gate" else 6) * K,
        "down_projection": "fused up+down per token" if chosen == "gate" else "per token",
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_oracle_rate(cfg, L, args.cpu_sample, layer)
    return res


def run_gpu_backward(args, world, rank, local):
    """The backward pass through the hybrid format: dx (per-token sparse pass
    for the rows that fit, tensor-core dense branch for overflow rows) then the
    weight gradients (column sort and per-unit sums, plus the dense branch's
    share). The forward that produces the pack and the routing
    runs once before timing: its outputs are the backward's inputs."""
    import torch

    from activation_sparse_gated_gemm_b200 import twell as tl

    tl.load()
    dev = torch.device("cuda", local)
    cfg = layer_config(args)
    L = synth.make_layer(cfg, seed=args.seed)
    dy_bits = synth.make_dy(cfg.T, cfg.d, args.seed)
    T, d, f, W = cfg.T, cfg.d, cfg.f, cfg.W
    x = tl.to_device_bf16(L["x"], dev)
    WgT = tl.to_device_bf16(L["WgT"], dev)
    WuT = tl.to_device_bf16(L["WuT"], dev)
    Wd = tl.to_device_bf16(L["Wd"], dev)
    dy = tl.to_device_bf16(dy_bits, dev)
    tw = tl.Twell(T, f, W, device=dev)
    y = torch.empty((T, d), dtype=torch.float32, device=dev)
    ovf_rows = torch.empty((T,), dtype=torch.int32, device=dev)
    n_ovf = torch.zeros((1,), dtype=torch.int32, device=dev)
    ws = torch.empty(tl.hybrid_workspace_bytes(T, d, f), dtype=torch.uint8, device=dev)
    st = tl.new_status(dev)
    tl.ffn_hybrid_forward(x, WgT, WuT, Wd, tw, y, ovf_rows, n_ovf, ws, st)
    del ws
    dx = torch.empty((T, d), dtype=torch.float32, device=dev)
    dW = [torch.empty((f, d), dtype=torch.float32, device=dev) for _ in range(3)]
    wsb = torch.empty(tl.backward_workspace_bytes(T, d, f, W), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    K, Wm = args.steps, args.warmup

    def make_dx(tensor_cores):
        return lambda: tl.ffn_hybrid_backward_dx(x, WgT, WuT, Wd, dy, tw, ovf_rows, n_ovf, dx, wsb, st,
                                                 tensor_cores=tensor_cores)

    def time_forms(make):
        out = {}
        for name, tc in (("cuda_cores", False), ("tensor_cores", True)):
            fn = make(tc)
            for _ in range(Wm):
                flush_l2(flush)
                fn()
            ts = []
            for _ in range(max(3, K // 4)):
                flush_l2(flush)
                a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a_ev.record(stream)
                fn()
                b_ev.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(a_ev.elapsed_time(b_ev))
            out[name] = max_over_ranks(float(np.median(ts)), world)
        return out

    # the two forms of dx (per-token axpys on the CUDA cores, or the scattered
    # dz, du through one tensor-core GEMM); the faster is the one the step uses
    dx_forms = time_forms(make_dx)
    dx_form = min(dx_forms, key=dx_forms.get)
    stage_dx = make_dx(dx_form == "tensor_cores")

    def make_dw(tensor_cores):
        return lambda: tl.ffn_hybrid_backward_dw(x, dy, tw, n_ovf, dW[0], dW[1], dW[2], wsb,
                                                 tensor_cores=tensor_cores)

    # the two forms of the weight gradients (per-unit sums on the CUDA cores, or
    # the dense scatter and GEMMs on the tensor cores), timed after a dx pass;
    # the faster is the one the step uses
    stage_dx()
    dw_forms = time_forms(make_dw)
    dw_form = min(dw_forms, key=dw_forms.get)
    stage_dw = make_dw(dw_form == "tensor_cores")

    for _ in range(Wm):
        flush_l2(flush)
        stage_dx()
        stage_dw()
    torch.cuda.synchronize(dev)
    if tl.status_get(st) != 0:
        raise RuntimeError(f"device status {tl.status_get(st)} after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        for k in range(K):
            flush_l2(flush)
            evs[k][0].record(stream)
            stage_dx()
            evs[k][1].record(stream)
            stage_dw()
            evs[k][2].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    per = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(2)] for k in range(K)])
    stage_ms = np.median(per, axis=0)
    step_ms = max_over_ranks(float(np.median(per.sum(axis=1))), world)

    # the library's dense backward at the same shape (tensor cores, bf16 dz/du/h)
    wsd = torch.empty(tl.dense_backward_workspace_bytes(T, d, f), dtype=torch.uint8, device=dev)
    dxd = torch.empty_like(dx)
    dWdn = [torch.empty_like(g) for g in dW]

    def dense_bwd():
        tl.dense_ffn_backward(x, WgT, WuT, Wd, dy, dxd, dWdn[0], dWdn[1], dWdn[2], wsd, st)

    for _ in range(Wm):
        flush_l2(flush)
        dense_bwd()
    dense_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(world)
    for k in range(K):
        flush_l2(flush)
        dense_ev[k][0].record(stream)
        dense_bwd()
        dense_ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = max_over_ranks(float(np.median([a.elapsed_time(b) for a, b in dense_ev])), world)
    del wsd, dxd, dWdn

    # e2e through the C ABI: dy from pinned host memory in, dx and the weight gradients out
    dy_host = dy.cpu().pin_memory()
    dx_host = torch.empty((T, d), dtype=torch.float32).pin_memory()
    dW_host = [torch.empty((f, d), dtype=torch.float32).pin_memory() for _ in range(3)]

    def e2e_step():
        dy.copy_(dy_host, non_blocking=True)
        stage_dx()
        stage_dw()
        dx_host.copy_(dx, non_blocking=True)
        for h, g in zip(dW_host, dW):
            h.copy_(g, non_blocking=True)

    for _ in range(max(1, Wm // 2)):
        e2e_step()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for k in range(K):
        flush_l2(flush)
        e2e_ev[k][0].record(stream)
        e2e_step()
        e2e_ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(float(np.median([a.elapsed_time(b) for a, b in e2e_ev])), world)
    status = tl.status_get(st)
    if status != 0:
        raise RuntimeError(f"device status {status} ({tl.status_str(status)})")

    counts = tw.counts.to(torch.int64)
    ovf_mask = tw.row_ovf.bool()
    n_ovf_h = int(n_ovf.item())
    nnz_fit = int(torch.clamp(counts, max=W)[~ovf_mask].sum())
    nnz_ovf = int(counts[ovf_mask].sum())  # true counts: every active unit of an overflow row
    # CUDA-core work of the rows that fit (the overflow rows' dense branch runs
    # on the tensor cores: 12 n_ovf d f FLOPs, reported beside it)
    flops_dx = 4.0 * d * nnz_fit  # two axpys per stored unit (u and dh come from dense GEMMs)
    flops_dw = 6.0 * d * nnz_fit  # three axpys per stored unit
    clocks = sampler.summary()
    peaks = load_peaks()
    fp32_peak = (torch.cuda.get_device_properties(dev).multi_processor_count * FP32_LANES_PER_SM * 2
                 * (clocks["sm_max_mhz"] or peaks.get("sm_max_mhz", 1965.0)) * 1e6)
    names = ["backward_dx", "backward_dw"]
    work = {"backward_dx": flops_dx, "backward_dw": flops_dw}
    bound = {"backward_dx": "alu", "backward_dw": "alu"}
    peak_tf = {"backward_dx": fp32_peak / 1e12, "backward_dw": fp32_peak / 1e12}
    if dx_form == "tensor_cores":  # one GEMM over all tokens, K = 4 f (values and remainders)
        work["backward_dx"] = 8.0 * T * d * f
        bound["backward_dx"] = "tensor"
        peak_tf["backward_dx"] = peaks["bf16_tflops"]
    if dw_form == "tensor_cores":  # three GEMMs over all tokens (plus the overflow rows' ones)
        work["backward_dw"] = 6.0 * T * d * f
        bound["backward_dw"] = "tensor"
        peak_tf["backward_dw"] = peaks["bf16_tflops"]
    dom = names[int(np.argmax(stage_ms))]
    ms = float(stage_ms[names.index(dom)])
    achieved = work[dom] / (ms * 1e-3) / 1e12
    res = {
        "metric": METRIC_BWD,
        "value": job_rate(T, world, step_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded generator; no dataset or trained weights)",
        "config": {"workload": f"{cfg.name}-like FFN layer backward through the hybrid TwELL format",
                   "tokens": T, "d": d, "f": f, "tile": cfg.tile, "ell_width": W, "density": cfg.density,
                   "dead_frac": cfg.dead_frac, "l2": "flushed between steps (256 MiB written, then read back so that no dirty line is left; outside events)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "roofline": {"kernel": dom, "bound": bound[dom], "achieved": achieved, "peak": peak_tf[dom],
                     "unit": "TFLOP/s", "frac": achieved / peak_tf[dom], "traffic": None,
                     "peak_source": ("fp32 FMA lanes x 2 x max SM clock" if bound[dom] == "alu"
                                     else f"{peaks['source']} bf16 burst")},
        "stages_ms": {n: float(v) for n, v in zip(names, stage_ms)},
        "dx_forms_ms": dx_forms,
        "dx_form": dx_form,
        "weight_gradient_forms_ms": dw_forms,
        "weight_gradient_form": dw_form,
        "batch_stats": {"n_ovf": n_ovf_h, "nnz_fit_rows": nnz_fit, "nnz_overflow_rows": nnz_ovf,
                        "dense_branch_gflop": 12.0 * n_ovf_h * d * f / 1e9},
        "dense_backward_ms": dense_ms,
        "speedup_vs_own_dense": dense_ms / step_ms,
        "e2e": {"value": job_rate(T, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 4 + 3 * f * d * 4},
        # per step, dx: the two slot-epilogue GEMMs (the records), then the tensor-core form's dense rows and
        # dx GEMM, or the CUDA-core form's counter zeroing and dx pass (two passes when Wg and Wu exceed
        # 64 MB), two gathers and three dense-branch GEMMs; weight gradients: the column sort (four launches)
        # and the per-unit sums, or the dense rows, one zeroing and three GEMMs, then the overflow rows' three
        # GEMMs (eight launches either way)
        "gpu_launches": ((9 if dx_form == "tensor_cores" else 9 + (4 * f * d > (64 << 20))) + 8) * K,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_oracle_rate(cfg, L, max(128, args.cpu_sample // 8), "gated", dy=dy_bits)
    return res


# ---------------------------------------------------------------- reference arm


def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, on bounded samples of the
    same workload; same metric and unit as the GPU arm."""
    if rank != 0:
        return None
    cfg = layer_config(args)
    L = synth.make_layer(cfg, seed=args.seed)
    sample = max(1, min(cfg.T, args.cpu_sample // 16))
    layer = "relu" if args.layer == "relu" else "gated"
    backward = args.pass_ == "backward"
    dy = synth.make_dy(cfg.T, cfg.d, args.seed) if backward else None
    if backward:
        sample = max(1, sample // 4)

    def step():
        oracle_step(cfg, L, slice(0, sample), layer, dy)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = sample / dt
    return {
        "impl": "reference",
        "metric": METRIC_BWD if backward else (METRIC_RELU if layer == "relu" else METRIC), "value": v,
        "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
        "config": {"workload": (f"{cfg.name}-like FFN layer backward through the hybrid TwELL format"
                                if backward else
                                f"{cfg.name}-like non-gated ReLU FFN layer forward (W1 = Wg, W2 = Wd), "
                                "hybrid TwELL" if layer == "relu" else
                                f"{cfg.name}-like FFN layer forward, hybrid TwELL"), "tokens": cfg.T,
                   "d": cfg.d, "f": cfg.f, "tile": cfg.tile, "ell_width": cfg.W,
                   "density": cfg.density, "dead_frac": cfg.dead_frac},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{sample} of {cfg.T} tokens per step (fp64 numpy oracle)"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_sweep(args) -> None:
    """Density x batch sweep (d=2048, f=8192): one JSON line per point with the
    hybrid forward's time, the dense FFN's time and the path roofline."""
    import torch

    from activation_sparse_gated_gemm_b200 import twell as tl

    tl.load()
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    Ts = [int(v) for v in args.sweep_T.split(",")] if args.sweep_T else list(synth.SWEEP_T)
    Ps = [float(v) for v in args.sweep_p.split(",")] if args.sweep_p else list(synth.SWEEP_P)
    for T in Ts:
        for pden in Ps:
            cfg = synth.sweep_config(T, pden)
            if args.sweep_w:
                cfg = dataclasses.replace(cfg, W=args.sweep_w)
            L = synth.make_layer(cfg, seed=args.seed)
            x, WgT, WuT, Wd = (tl.to_device_bf16(L[k], dev) for k in ("x", "WgT", "WuT", "Wd"))
            tw = tl.Twell(T, cfg.f, cfg.W, device=dev)
            y = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
            ovf_rows = torch.empty((T,), dtype=torch.int32, device=dev)
            n_ovf = torch.zeros((1,), dtype=torch.int32, device=dev)
            ws = torch.empty(tl.hybrid_workspace_bytes(T, cfg.d, cfg.f), dtype=torch.uint8, device=dev)
            wsd = torch.empty(tl.dense_workspace_bytes(T, cfg.d, cfg.f), dtype=torch.uint8, device=dev)
            st = tl.new_status(dev)

            def timed(fn, k):
                """Median device time of fn; replayed from a CUDA graph when the
                calls capture (they are stream-ordered and never sync), so
                small batches are not measured as launch gaps."""
                for _ in range(args.warmup):
                    flush_l2(flush)
                    fn()
                torch.cuda.synchronize(dev)
                run = fn
                if not args.sweep_eager:
                    try:
                        graph = torch.cuda.CUDAGraph()
                        with torch.cuda.graph(graph):
                            fn()
                        run = graph.replay
                    except Exception:  # noqa: BLE001 -- measured eagerly instead
                        torch.cuda.synchronize(dev)
                        run = fn
                ts = []
                for _ in range(k):
                    flush_l2(flush)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    run()
                    b.record()
                    torch.cuda.synchronize(dev)
                    ts.append(a.elapsed_time(b))
                timed.graph = run is not fn
                return float(np.median(ts))

            ms_gate = timed(lambda: tl.ffn_hybrid_forward(x, WgT, WuT, Wd, tw, y, ovf_rows, n_ovf, ws, st),
                            args.steps)
            ms_tc = timed(lambda: tl.ffn_hybrid_forward_tc_up(x, WgT, WuT, Wd, tw, y, ovf_rows, n_ovf, ws, st),
                          args.steps)
            ms, form = (ms_gate, "gate") if ms_gate <= ms_tc else (ms_tc, "tc_up")
            ms_dense = timed(lambda: tl.dense_ffn_forward(x, WgT, WuT, Wd, y, wsd, st), args.steps)
            status = tl.status_get(st)
            counts = tw.counts.to(torch.int64)
            n_o = int(n_ovf.item())
            nnz = int(torch.clamp(counts, max=cfg.W)[~tw.row_ovf.bool()].sum())
            g = torch.empty((T, cfg.f), dtype=torch.bfloat16, device=dev)
            tl.unpack(tw, g, st)
            union = int((g[~tw.row_ovf.bool()] != 0).any(dim=0).sum())
            del g
            alg = algorithmic(cfg, n_o, nnz, union)
            t_roof = max((alg["gate_flops"] + alg["dense_branch_flops"]) / (peaks["bf16_tflops"] * 1e12),
                         alg["alg_bytes"] / (peaks["hbm_gbs"] * 1e9))
            # the dense layer's own bound: 6 T d f FLOPs at the tensor peak, or its
            # three weight matrices, x, y and the bf16 h round trip at the HBM peak
            dense_bytes = 3 * 2.0 * cfg.d * cfg.f + 6.0 * T * cfg.d + 4.0 * T * cfg.f
            t_dense_roof = max(6.0 * T * cfg.d * cfg.f / (peaks["bf16_tflops"] * 1e12),
                               dense_bytes / (peaks["hbm_gbs"] * 1e9))
            print(json.dumps({"sweep": True, "T": T, "density": pden, "W": cfg.W, "d": cfg.d, "f": cfg.f,
                              "ms": ms, "form": form, "ms_gate_form": ms_gate, "ms_tc_up_form": ms_tc,
                              "tokens_per_s": T / (ms * 1e-3), "dense_ms": ms_dense,
                              "speedup_vs_own_dense": ms_dense / ms, "roofline_frac": t_roof / (ms * 1e-3),
                              "t_roof_us": t_roof * 1e6, "dense_roofline_frac": t_dense_roof / (ms_dense * 1e-3),
                              "t_dense_roof_us": t_dense_roof * 1e6, "n_ovf": n_o,
                              "measured_density": float(counts.sum()) / (T * cfg.f), "status": status,
                              "cuda_graph": bool(getattr(timed, "graph", False))}),
                  flush=True)
            del x, WgT, WuT, Wd, tw, y, ws, wsd
            torch.cuda.empty_cache()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="twell", choices=["twell", "reference"])
    ap.add_argument("--config", default="2b", choices=sorted(synth.CONFIGS),
                    help="layer shape (default: the 2B-like hybrid layer, the largest that fits one GPU)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the configured layer on this many tokens instead (small cases for profiler captures)")
    ap.add_argument("--cpu-sample", type=int, default=12288)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", default="auto", choices=["auto", "gate", "tc_up"],
                    help="hybrid form: gate (sparse up+down) or tc_up (up on tensor cores); auto times both")
    ap.add_argument("--layer", default="gated", choices=["gated", "relu"],
                    help="gated: (ReLU(x Wg) * x Wu) Wd; relu: the non-gated ReLU(x W1) W2")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "backward"],
                    help="forward (the default) or the backward pass through the hybrid format")
    ap.add_argument("--compact", action="store_true",
                    help="drop the hidden units the batch never activates before timing")
    ap.add_argument("--sweep", action="store_true", help="density x batch sweep, one JSON line per point")
    ap.add_argument("--sweep-T", default="", help="comma-separated token counts (default: the full sweep)")
    ap.add_argument("--sweep-p", default="", help="comma-separated densities (default: the full sweep)")
    ap.add_argument("--sweep-eager", action="store_true", help="time sweep points without CUDA graphs")
    ap.add_argument("--sweep-w", type=int, default=0,
                    help="ELL width for every sweep point (0: the smallest that stores the pure sparse path); "
                         "a fixed W such as 32 measures the hybrid route, dense branch included")
    ap.add_argument("--record-traffic", default="",
                    help="write profiles/traffic.json from this ncu raw-page CSV and exit")
    ap.add_argument("--record-kernel", action="append", default=[],
                    help="stage=kernel-name substring, for --record-traffic (repeatable)")
    ap.add_argument("--record-command", default="", help="the ncu command the CSV came from")
    args = ap.parse_args(argv)
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.config, args.record_kernel,
                                        args.record_command)))
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.sweep:
        run_sweep(args)
        return 0

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    world, rank, local = dist_setup(args)
    try:
        res = (run_gpu_backward if args.pass_ == "backward" else run_gpu)(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
