#!/usr/bin/env python
"""Throughput of blockwise packed causal RoPE attention on B200.

One step = one pass of the whole path over one batch of synthetic input:
the forward (RoPE table, block metadata, longest-first order, attention
kernel) and, for workloads with a backward, the backward (delta, metadata,
attention backward kernel, dQ conversion), all through the C ABI.

Prints ONE JSON line (rank 0). `value` is mask-aware attention TFLOP/s of
the whole job (forward 4*D*pairs*H, backward 10*D*pairs*H, pairs = exact
count of visible (query, key) pairs of the generated segments); tokens/s
and the forward / backward split ride along.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed

Multi-GPU: one process per GPU (torchrun); every rank runs its own
independent copy of the workload (weak scaling, no data-path collective);
timing is the max over ranks of CUDA-event time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_blockwise_causal_b200 import workloads as wl  # noqa: E402

METRIC = ("attention TFLOP/s and tokens/s (fwd, fwd+bwd) at 1 B200; "
          "% of bf16 tensor peak")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# sources whose change invalidates a recorded DRAM capture: the kernel's
# own file and the metadata and scheduling kernels that decide which units
# it runs in which order (its traffic depends on both)
TRAFFIC_SOURCES = {"fwd_tc_kernel": ("fwd_tc.cu", "aux_kernels.cu"),
                   "bwd_tc_kernel": ("bwd_tc.cu", "aux_kernels.cu")}


def traffic_source_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for src in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(ROOT, "long_context_blockwise_causal_b200",
                               "csrc", src), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` from the committed one-pass ncu
    capture (profiles/traffic_<workload>.json), or None when there is no
    capture for this workload or the sources it depends on changed since."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(kernel)
    if not rec:
        return None
    if traffic_source_hash(kernel) != rec.get("source_sha256_16"):
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.lines = []
        self.sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else
                        "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ oracle sample

def oracle_sample(w, t_host, budget_s, backward):
    """Time the fp64 oracle on a prefix of the workload's first row (head 0),
    sized so one run takes about budget_s. Returns (TFLOP/s, info)."""
    import oracle
    from threadpoolctl import threadpool_info

    def run(L):
        q = t_host["q"][:1, :L, :1]
        k = t_host["k"][:1, :L, :1]
        v = t_host["v"][:1, :L, :1]
        seg = t_host["segment_ids"][:1, :L]
        pos = t_host["positions"][:1, :L]
        t0 = time.perf_counter()
        if backward:
            g = t_host["dout"][:1, :L, :1]
            oracle.attn_bwd(q, k, v, g, seg, pos, w.theta)
        else:
            oracle.attn_fwd(q, k, v, seg, pos, w.theta)
        dt = time.perf_counter() - t0
        segn = seg[0].numpy()
        runs = np.diff(np.r_[0, np.flatnonzero(np.diff(segn)) + 1, L])
        pairs = int((runs * (runs + 1) // 2).sum())
        flop = (14 if backward else 4) * w.D * pairs
        return dt, flop

    avail = t_host["q"].shape[1]   # the host copy may be a prefix
    L = min(1024, avail)
    dt, _ = run(L)
    scale = math.sqrt(max(budget_s, 0.1) / max(dt, 1e-3))
    L = int(min(avail, max(128, (L * scale) // 128 * 128)))
    dt, flop = run(L)
    threads = max((i.get("num_threads", 1) for i in threadpool_info()),
                  default=1)
    info = {"sample": f"oracle {'fwd+bwd' if backward else 'fwd'} (fp64, "
                      f"dense row-blocked) on the first {L} tokens of batch "
                      f"row 0, head 0 of {w.name}; mask-aware FLOP of that "
                      f"prefix / wall time",
            "cores": int(threads), "host_cores": os.cpu_count(),
            "seconds": dt}
    return flop / dt / 1e12, info


# ------------------------------------------------------------------ e2e

def pipelined_e2e(dev, h_in, make_set, run, outputs, h_out, steps):
    """Time `steps` end-to-end steps through the public API: every step
    copies its inputs from pinned host buffers (h_in: name -> tensor), runs
    run(set) on the device and copies its results back (outputs(set) ->
    h_out). Copies go on their own streams into two buffer sets, so step
    i+1's inputs arrive and step i-1's results leave while step i computes.
    Returns ms per step (CUDA events on the compute stream; the first
    step's upload and the last step's download are inside the interval)."""
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [make_set(), make_set()]
    ev = lambda: torch.cuda.Event()
    uploaded = [ev(), ev()]
    computed = [ev(), ev()]
    downloaded = [ev(), ev()]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(comp)
    up.wait_event(start)
    for i in range(steps):
        b = i % 2
        ds = sets[b]
        if i >= 2:
            up.wait_event(computed[b])        # set b's inputs are free
            comp.wait_event(downloaded[b])    # set b's outputs are free
        with torch.cuda.stream(up):
            for n, hb in h_in.items():
                ds[n].copy_(hb, non_blocking=True)
            uploaded[b].record(up)
        comp.wait_event(uploaded[b])
        run(ds)
        computed[b].record(comp)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            for hb, db in zip(h_out, outputs(ds)):
                hb.copy_(db, non_blocking=True)
            downloaded[b].record(down)
    comp.wait_event(downloaded[(steps - 1) % 2])
    if steps >= 2:
        comp.wait_event(downloaded[(steps - 2) % 2])
    end.record(comp)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / steps


def pipelined_e2e_phased(dev, h_in_phases, make_set, run_phases,
                         output_phases, h_out_phases, steps):
    """pipelined_e2e for a step made of phases (forward, then backward):
    phase k's inputs (h_in_phases[k]) are uploaded in order on the upload
    stream, its compute (run_phases[k]) waits only for them, and its
    results (output_phases[k] -> h_out_phases[k]) leave as soon as it is
    done, while the next phase computes. Same two device buffer sets and
    the same events-on-the-compute-stream timing as pipelined_e2e."""
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [make_set(), make_set()]
    nph = len(run_phases)
    ev = lambda: torch.cuda.Event()
    uploaded = [[ev() for _ in range(nph)] for _ in range(2)]
    phase_done = [[ev() for _ in range(nph)] for _ in range(2)]
    downloaded = [ev(), ev()]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(comp)
    up.wait_event(start)
    for i in range(steps):
        b = i % 2
        ds = sets[b]
        if i >= 2:
            up.wait_event(phase_done[b][nph - 1])  # set b's inputs are free
            comp.wait_event(downloaded[b])         # set b's outputs are free
        with torch.cuda.stream(up):
            for k in range(nph):
                for n, hb in h_in_phases[k].items():
                    ds[n].copy_(hb, non_blocking=True)
                uploaded[b][k].record(up)
        for k in range(nph):
            comp.wait_event(uploaded[b][k])
            run_phases[k](ds)
            phase_done[b][k].record(comp)
            down.wait_event(phase_done[b][k])
            with torch.cuda.stream(down):
                for hb, db in zip(h_out_phases[k], output_phases[k](ds)):
                    hb.copy_(db, non_blocking=True)
        downloaded[b].record(down)
    comp.wait_event(downloaded[(steps - 1) % 2])
    if steps >= 2:
        comp.wait_event(downloaded[(steps - 2) % 2])
    end.record(comp)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / steps


# ------------------------------------------------------------------ main

def init_dist(impl):
    from long_context_blockwise_causal_b200 import dist
    # the reference arm runs on host cores only: no NCCL, no GPU
    return dist.init_from_env("gloo" if impl == "reference" else "nccl")


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x, ws, dev):
    from long_context_blockwise_causal_b200 import dist
    return dist.max_over_ranks(x, ws, dev)


REF_PREFIX_TOKENS = 32768


def reference_arm(args, ws, rank):
    """The oracle, timed as it stands on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    # the oracle runs on a prefix of row 0: draw only that much of the
    # inputs (the same values as the full draw)
    t_host = wl.make_inputs(w, args.seed, device="cpu",
                            with_dout=w.backward, prefix=REF_PREFIX_TOKENS)
    times, flops, info = [], [], None
    for i in range(args.warmup + args.steps):
        tf, info = oracle_sample(w, t_host, args.ref_budget, w.backward)
        if i >= args.warmup:
            times.append(info["seconds"])
            flops.append(tf)
    value = float(np.mean(flops))
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": float(np.mean(times)) * 1e3,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H,
                       "D": w.D, "theta": w.theta},
            "cpu_baseline": {"kind": "oracle", "value": value,
                             "unit": "TFLOP/s", "cores": info["cores"],
                             "sample": info["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


DECODE_WORKLOADS = {
    # one query token per (row, head) against a cache of L keys, one example
    "decode1m": {"B": 1, "L": 1 << 20, "H": 32, "theta": 5e7},
    "decode128k_b16": {"B": 16, "L": 1 << 17, "H": 32, "theta": 1e7},
}


DECODE_METRIC = ("decode attention HBM GB/s (1 query token per row and "
                 "head against the cache)")


def decode_oracle_sample(cfg, seed, budget_s):
    """Time the fp64 oracle on one decode query (batch row 0, head 0) against
    a prefix of the cache, sized so one run takes about budget_s. The
    metric counts the key and value rows read, as on the device. Returns
    (GB/s, info)."""
    import oracle
    from threadpoolctl import threadpool_info
    D = 128

    def run(L):
        scale = 1.0 / math.sqrt(D)
        k = wl.random_tensor((1, L, 1, D), seed * 16 + 2, scale,
                             torch.bfloat16, "cpu")
        v = wl.random_tensor((1, L, 1, D), seed * 16 + 3, scale,
                             torch.bfloat16, "cpu")
        # only the last row is the query; the others are never read
        q = wl.random_tensor((1, 1, 1, D), seed * 16 + 1, scale,
                             torch.bfloat16, "cpu").expand(1, L, 1, D)
        seg = torch.zeros((1, L), dtype=torch.int32)
        pos = torch.arange(L, dtype=torch.int32)[None]
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(q, k, v, seg, pos, cfg["theta"], 0, 0, [L - 1])
        return time.perf_counter() - t0

    L = min(1 << 15, cfg["L"])
    dt = run(L)
    L = int(min(cfg["L"], max(4096, (L * max(budget_s, 0.05) / max(dt, 1e-4))
                              // 4096 * 4096)))
    dt = run(L)
    threads = max((i.get("num_threads", 1) for i in threadpool_info()),
                  default=1)
    info = {"sample": f"oracle decode (fp64) of batch row 0, head 0 against "
                      f"the first {L} cached keys; key and value bytes read "
                      f"/ wall time",
            "cores": int(threads), "host_cores": os.cpu_count(),
            "seconds": dt}
    return L * D * 2 * 2 / dt / 1e9, info


def decode_reference(args):
    """The oracle's decode as the reference arm (rank 0, host cores)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    cfg = DECODE_WORKLOADS[args.workload]
    vals, secs, info = [], [], None
    for i in range(args.warmup + args.steps):
        gbs, info = decode_oracle_sample(cfg, args.seed, args.ref_budget)
        if i >= args.warmup:
            vals.append(gbs)
            secs.append(info["seconds"])
    value = float(np.mean(vals))
    print(json.dumps({
        "impl": "reference", "metric": DECODE_METRIC, "value": value,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": float(np.mean(secs)) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": cfg["B"], "L": cfg["L"],
                   "H": cfg["H"], "D": 128},
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": "GB/s",
                         "cores": info["cores"], "sample": info["sample"]},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def bench_decode(args):
    """Decode attention: HBM-bound (every visible key and value row is read
    once). Prints one JSON line with GB/s against the measured copy
    bandwidth."""
    if args.impl == "reference":
        decode_reference(args)
        return
    from long_context_blockwise_causal_b200 import ops
    cfg = DECODE_WORKLOADS[args.workload]
    B, L, H, D = cfg["B"], cfg["L"], cfg["H"], 128
    dev = torch.device("cuda", 0)
    scale = 1.0 / math.sqrt(D)
    k = wl.random_tensor((B, L, H, D), args.seed * 16 + 2, scale,
                         torch.bfloat16, dev)
    v = wl.random_tensor((B, L, H, D), args.seed * 16 + 3, scale,
                         torch.bfloat16, dev)
    q = wl.random_tensor((B, 1, H, D), args.seed * 16 + 1, scale,
                         torch.bfloat16, dev)[:, 0].contiguous()
    pos = torch.arange(L, dtype=torch.int32, device=dev).repeat(B, 1)
    table = ops.rope_table(cfg["theta"], L, device=dev)
    k_rot = ops.rope_apply(k, pos, table)
    del k
    kv_start = torch.zeros(B, dtype=torch.int32, device=dev)
    kv_len = torch.full((B,), L, dtype=torch.int32, device=dev)
    q_pos = torch.full((B,), L - 1, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    ws = torch.empty(ops.decode_workspace_size(B, H, L), dtype=torch.uint8,
                     device=dev)
    step = lambda: ops.decode(q, k_rot, v, kv_start, kv_len, q_pos, table,
                              out=out, lse=lse, workspace=ws)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    l0 = ops.kernel_launches()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    launches = ops.kernel_launches() - l0
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    nbytes = B * H * L * D * 2 * 2 + B * H * D * 4  # K, V rows + q, out
    gbs = nbytes / (ms / 1e3) / 1e9
    pk = peaks()
    line = {"metric": DECODE_METRIC,
            "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "B": B, "L": L, "H": H,
                       "D": D, "l2": "cache larger than L2"},
            "tokens_per_s": B / (ms / 1e3),
            "roofline": {"bound": "hbm", "kernel": "decode_split_kernel",
                         "achieved": gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": None,
                         "peak_kind": f"copy bandwidth ({pk['source']})"},
            "gpu_launches": int(launches), "device_status": ops.last_status(),
            "clocks": clk}
    if not args.no_e2e:
        # through the public call with host buffers: each step's query
        # tokens and their positions in, the outputs and lse out; the cache
        # is serving state resident in HBM
        qh = q.cpu().pin_memory()
        ph = q_pos.cpu().pin_memory()
        h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                 torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]

        def make_set():
            # the workspace is used by the compute stream only: shared
            return {"q": torch.empty_like(q), "q_pos": torch.empty_like(q_pos),
                    "out": torch.empty_like(out),
                    "lse": torch.empty_like(lse)}

        def run(d):
            ops.decode(d["q"], k_rot, v, kv_start, kv_len, d["q_pos"], table,
                       out=d["out"], lse=d["lse"], workspace=ws)

        h_in = {"q": qh, "q_pos": ph}
        outs = lambda d: [d["out"], d["lse"]]
        pipelined_e2e(dev, h_in, make_set, run, outs, h_out, 2)
        ems = pipelined_e2e(dev, h_in, make_set, run, outs, h_out,
                            max(2, args.steps))
        nbytes_in = qh.numel() * qh.element_size() + ph.numel() * 4
        nbytes_out = sum(x.numel() * x.element_size() for x in h_out)
        line["e2e"] = {"value": nbytes / (ems / 1e3) / 1e9, "unit": "GB/s",
                       "ms_per_step": ems, "h2d_bytes_per_step": nbytes_in,
                       "d2h_bytes_per_step": nbytes_out,
                       "note": "query tokens and positions in, out and lse "
                               "back per step (copy streams overlapped with "
                               "the neighbouring steps' compute); the "
                               "rotated key cache and the values stay in "
                               "HBM"}
    if not args.no_cpu_baseline:
        gbs_cpu, info = decode_oracle_sample(cfg, args.seed, args.cpu_budget)
        line["cpu_baseline"] = {"value": gbs_cpu, "unit": "GB/s",
                                "kind": "oracle", **info}
    print(json.dumps(line), flush=True)


FFN_METRIC = ("blockwise SwiGLU FFN TFLOP/s, forward + backward (3 + 8 "
              "products of T x Dm x F: the backward recomputes x Wg^T and "
              "x Wu^T per chunk) at 1 B200; % of bf16 tensor peak")


def ffn_oracle_sample(t_host, budget_s):
    """Time the fp64 oracle MLP on the first R tokens (full weights), R
    sized so one run takes about budget_s. Returns (TFLOP/s, info)."""
    import oracle
    from threadpoolctl import threadpool_info
    w = {k: v.float().numpy().astype(np.float64) for k, v in t_host.items()
         if k != "x"}
    x = t_host["x"]
    Dm, F = x.shape[1], w["w_gate"].shape[0]

    def run(R):
        xs = x[:R].float().numpy().astype(np.float64)
        dy = np.ones((R, Dm))
        t0 = time.perf_counter()
        oracle.swiglu_mlp(xs, w["w_gate"], w["w_up"], w["w_down"])
        oracle.swiglu_mlp_bwd(xs, w["w_gate"], w["w_up"], w["w_down"], dy)
        return time.perf_counter() - t0

    R = 32
    dt = run(R)
    R = int(min(x.shape[0], max(32, R * max(budget_s, 0.1) / max(dt, 1e-3))))
    dt = run(R)
    threads = max((i.get("num_threads", 1) for i in threadpool_info()),
                  default=1)
    info = {"sample": f"oracle SwiGLU MLP forward + backward (fp64 numpy) "
                      f"on the first {R} tokens, full {Dm}x{F} weights; "
                      f"FLOP of those rows (3 + 8 products) / wall time",
            "cores": int(threads), "host_cores": os.cpu_count(),
            "seconds": dt}
    return wl.ffn_flops(R, Dm, F) // 3 * 11 / dt / 1e12, info


def bench_ffn(args):
    """Blockwise FFN: three dense projections on the tensor cores."""
    w = wl.FFN_WORKLOADS[args.workload]
    f_fwd = wl.ffn_flops(w.T, w.Dm, w.F)          # 3 products
    f_bwd = f_fwd // 3 * 8                         # 8 products
    flop = f_fwd + f_bwd
    cfg = {"workload": w.name, "T": w.T, "Dm": w.Dm, "F": w.F,
           "chunk": w.chunk, "weights": "N(0, 0.02^2) bf16",
           "l2": "inputs and weights larger than L2 (no flush)"}
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        t_host = wl.make_ffn_inputs(w.T, w.Dm, w.F, args.seed, device="cpu",
                                    w_std=w.w_std)
        vals, secs = [], []
        for i in range(args.warmup + args.steps):
            tf, info = ffn_oracle_sample(t_host, args.ref_budget)
            if i >= args.warmup:
                vals.append(tf)
                secs.append(info["seconds"])
        value = float(np.mean(vals))
        print(json.dumps({
            "impl": "reference", "metric": FFN_METRIC, "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": float(np.mean(secs)) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"kind": "oracle", "value": value,
                             "unit": "TFLOP/s", "cores": info["cores"],
                             "sample": info["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
            flush=True)
        return
    from long_context_blockwise_causal_b200 import ops
    dev = torch.device("cuda", 0)
    t = wl.make_ffn_inputs(w.T, w.Dm, w.F, args.seed, device=dev,
                           w_std=w.w_std)
    y = torch.empty_like(t["x"])
    g = torch.Generator(device=dev).manual_seed(args.seed * 16 + 9)
    dy = torch.randn(t["x"].shape, generator=g, device=dev).to(torch.bfloat16)
    ws = torch.empty(ops.ffn_workspace_size(w.chunk, w.F), dtype=torch.uint8,
                     device=dev)
    wsb = torch.empty(ops.ffn_bwd_workspace_size(w.chunk, w.F),
                      dtype=torch.uint8, device=dev)
    grads = (torch.empty_like(t["x"]),
             torch.empty((w.F, w.Dm), dtype=torch.float32, device=dev),
             torch.empty((w.F, w.Dm), dtype=torch.float32, device=dev),
             torch.empty((w.Dm, w.F), dtype=torch.float32, device=dev))
    fwd = lambda: ops.ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"],
                              chunk=w.chunk, y=y, workspace=ws)
    bwd = lambda: ops.ffn_bwd(t["x"], t["w_gate"], t["w_up"], t["w_down"],
                              dy, chunk=w.chunk, dx=grads[0],
                              dw_gate=grads[1], dw_up=grads[2],
                              dw_down=grads[3], workspace=wsb)
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    l0 = ops.kernel_launches()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    t_f = t_b = 0.0
    for _ in range(args.steps):
        ev[0].record()
        fwd()
        ev[1].record()
        bwd()
        ev[2].record()
        torch.cuda.synchronize()
        t_f += ev[0].elapsed_time(ev[1])
        t_b += ev[1].elapsed_time(ev[2])
    launches = ops.kernel_launches() - l0
    clk = clocks.stop()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ms = (t_f + t_b) / args.steps
    ms_f, ms_b = t_f / args.steps, t_b / args.steps
    tflops = flop / (ms / 1e3) / 1e12
    tf_b = f_bwd / (ms_b / 1e3) / 1e12
    pk = peaks()
    line = {"metric": FFN_METRIC, "value": tflops, "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": cfg, "tokens_per_s": w.T / (ms / 1e3),
            "fwd": {"ms": ms_f, "tflops": f_fwd / (ms_f / 1e3) / 1e12},
            "bwd": {"ms": ms_b, "tflops": tf_b},
            "roofline": {"bound": "tensor",
                         "kernel": "mlp_gemm_kernel (backward launches)",
                         "achieved": tf_b, "peak": pk["bf16_tflops_sustained"],
                         "unit": "TFLOP/s",
                         "frac": tf_b / pk["bf16_tflops_sustained"],
                         "frac_of_burst_peak": tf_b / pk["bf16_tflops"],
                         "traffic": None,
                         "peak_kind": f"bf16 sustained ({pk['source']})"},
            "gpu_launches": int(launches), "device_status": ops.last_status(),
            "clocks": clk}
    if not args.no_e2e:
        # through the public call with host buffers: x in, y out per step
        xh = t["x"].cpu().pin_memory()
        dyh = dy.cpu().pin_memory()
        h_out = [torch.empty_like(xh).pin_memory(),
                 torch.empty_like(xh).pin_memory()]

        def make_set():
            # the workspaces are used by the compute stream only: shared
            return {"x": torch.empty_like(t["x"]), "dy": torch.empty_like(dy),
                    "y": torch.empty_like(y), "dx": torch.empty_like(y)}

        def run(d):
            ops.ffn_fwd(d["x"], t["w_gate"], t["w_up"], t["w_down"],
                        chunk=w.chunk, y=d["y"], workspace=ws)
            ops.ffn_bwd(d["x"], t["w_gate"], t["w_up"], t["w_down"], d["dy"],
                        chunk=w.chunk, dx=d["dx"], dw_gate=grads[1],
                        dw_up=grads[2], dw_down=grads[3], workspace=wsb)

        h_in = {"x": xh, "dy": dyh}
        outs = lambda d: [d["y"], d["dx"]]
        pipelined_e2e(dev, h_in, make_set, run, outs, h_out, 2)
        ems = pipelined_e2e(dev, h_in, make_set, run, outs, h_out,
                            max(2, min(args.steps, 6)))
        nb = xh.numel() * xh.element_size()
        line["e2e"] = {"value": flop / (ems / 1e3) / 1e12, "unit": "TFLOP/s",
                       "ms_per_step": ems, "h2d_bytes_per_step": 2 * nb,
                       "d2h_bytes_per_step": 2 * nb,
                       "note": "x and dy in, y and dx out per step (copy "
                               "streams overlapped with the neighbouring "
                               "steps' compute); weights and weight "
                               "gradients stay on the device"}
    if not args.no_cpu_baseline:
        t_host = {k: v.cpu() for k, v in t.items()}
        tf, info = ffn_oracle_sample(t_host, args.cpu_budget)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s",
                                "kind": "oracle", **info}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="packed128k",
                    choices=sorted(wl.WORKLOADS) + sorted(DECODE_WORKLOADS)
                    + sorted(wl.FFN_WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--N", type=int, default=None,
                    help="override the workload's sequence length (profiling)")
    ap.add_argument("--H", type=int, default=None,
                    help="override the workload's head count (profiling)")
    ap.add_argument("--B", type=int, default=None,
                    help="override the workload's batch rows (profiling)")
    ap.add_argument("--shard", default="replica", choices=["replica", "heads"],
                    help="N>1: each rank runs a full replica (weak scaling) or "
                         "a slice of the heads of one job (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=4.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.workload in DECODE_WORKLOADS:
        bench_decode(args)
        return
    if args.workload in wl.FFN_WORKLOADS:
        bench_ffn(args)
        return
    if args.impl == "reference":
        # host cores only: rank 0 runs the oracle, other ranks have no work
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    bench_attention(args)


L2_BYTES = 126e6


def tile_counts(ops, segment_ids):
    """Tiles the forward kernel visits and, of those, the ones it takes
    mask-free, from the very metadata it runs on (lwm_blockattn_visibility:
    key blocks [kv_lo, kv_hi] per query block, FULL iff every row's key
    range covers the block)."""
    v = ops.visibility(segment_ids, key_view=False)
    lo, hi = v["kv_lo"].long(), v["kv_hi"].long()
    lo_max, hi_min = v["lo_max"].long(), v["hi_min"].long()
    visited = (hi - lo + 1).clamp(min=0)
    blk = ops.BLOCK
    first_full = torch.maximum(lo, (lo_max + blk - 1).div(blk,
                                                          rounding_mode="floor"))
    last_full = torch.minimum(hi, (hi_min - (blk - 1)).div(
        blk, rounding_mode="floor"))
    full = (last_full - first_full + 1).clamp(min=0)
    full = torch.where(lo_max > hi_min, torch.zeros_like(full), full)
    return int(visited.sum().item()), int(full.sum().item())


def copy_floor(dev, h_in, d_in, h_out, d_out):
    """Host<->device copy time of one step's bytes over this box's link:
    uploads alone, downloads alone and both at once on two streams (ms,
    CUDA events, after one untimed round)."""
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def once(do_up, do_down):
        comp = torch.cuda.current_stream(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        up.wait_stream(comp)
        down.wait_stream(comp)
        if do_up:
            with torch.cuda.stream(up):
                for n, hb in h_in.items():
                    d_in[n].copy_(hb, non_blocking=True)
        if do_down:
            with torch.cuda.stream(down):
                for hb, db in zip(h_out, d_out):
                    hb.copy_(db, non_blocking=True)
        comp.wait_stream(up)
        comp.wait_stream(down)
        e1.record(comp)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    once(True, True)
    return {"h2d_ms": once(True, False), "d2h_ms": once(False, True),
            "both_ms": once(True, True)}


def bench_attention(args):
    ws, rank, local = init_dist(args.impl)

    from long_context_blockwise_causal_b200 import ops

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS[args.workload]
    qkp = "bf16x3" if w.scale == 1.0 else "bf16"
    if args.N or args.H or args.B:
        w = wl.Workload(w.name + "-reduced", args.B or w.B, args.N or w.N,
                        args.H or w.H, w.D, w.theta, w.segments, w.scale,
                        w.backward, seg_args=w.seg_args)
    job_heads = w.H
    if args.shard == "heads" and ws > 1:
        from long_context_blockwise_causal_b200 import dist
        h0, h1 = dist.head_shard(w.H, ws, rank)
        t = wl.make_inputs(w, args.seed, device=dev, H=h1 - h0,
                           with_dout=w.backward)
    else:
        t = wl.make_inputs(w, args.seed + 1000 * rank, device=dev,
                           with_dout=w.backward)
    B, N, H, D = t["q"].shape
    pairs_per_head = wl.visible_pairs(t["lengths"])
    tiles_visited, tiles_full = tile_counts(ops, t["segment_ids"])
    fwd_flop = 4.0 * D * pairs_per_head * H
    bwd_flop = 10.0 * D * pairs_per_head * H if w.backward else 0.0
    elem = t["q"].element_size()
    # forward algorithmic bytes: q, k, v in, out and lse out, ids and
    # positions in
    fwd_bytes = 4 * B * N * H * D * elem + B * H * N * 4 + 8 * B * N
    strong = args.shard == "heads" and ws > 1
    # whole-job work: replicas multiply it by the rank count, a head-sharded
    # job is one workload split across the ranks
    job_scale = (job_heads / H) if strong else ws
    max_pos = int(t["positions"].max().item()) + 1
    ws_bytes = max(ops.fwd_workspace_size(B, N, H, max_pos,
                                          qk_precision=qkp),
                   ops.bwd_workspace_size(B, N, H, max_pos,
                                          qk_precision=qkp)
                   if w.backward else 0)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    grads = [torch.empty_like(t["q"]) for _ in range(3)] if w.backward \
        else None
    stream = torch.cuda.current_stream(dev)
    # inputs smaller than L2 would be re-read from it: flush it (a write
    # larger than L2) before every timed step, outside the step's events
    small = 3 * t["q"].numel() * elem < L2_BYTES
    flush = torch.empty(int(2 * L2_BYTES), dtype=torch.uint8, device=dev) \
        if small else None

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                w.theta, max_pos=max_pos, qk_precision=qkp, out=out, lse=lse,
                workspace=workspace, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if w.backward:
            ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                    t["segment_ids"], t["positions"], w.theta,
                    max_pos=max_pos, qk_precision=qkp, dq=grads[0],
                    dk=grads[1], dv=grads[2], workspace=workspace,
                    stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        if small:
            flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if ops.last_status() != ops.OK:
        raise SystemExit("device status not OK after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    barrier(ws)
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    launches0 = ops.kernel_launches()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        if small:
            flush.zero_()
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = ops.kernel_launches() - launches0
    barrier(ws)
    clk = clocks.stop() if clocks else None
    status = ops.last_status()
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs])) \
        if w.backward else 0.0
    # with flushes in between, a step is its own events; else the whole
    # bracketed interval over the steps
    ms = (fwd_ms + bwd_ms) if small else \
        start.elapsed_time(end) / args.steps
    ms = max_over_ranks(ms, ws, dev)

    # a small (launch-bound) forward also as a CUDA graph replay of the same
    # call, L2 flushed before each replay like the timed calls above
    graph_us = None
    if small and not w.backward:
        gs = torch.cuda.Stream(dev)
        with torch.cuda.stream(gs):
            step_fwd = lambda: ops.fwd(
                t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                w.theta, max_pos=max_pos, qk_precision=qkp, out=out, lse=lse,
                workspace=workspace, stream=gs)
            step_fwd()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            step_fwd()
        torch.cuda.synchronize(dev)
        gt = []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            graph.replay()
            g1.record(stream)
            torch.cuda.synchronize(dev)
            gt.append(g0.elapsed_time(g1))
        graph_us = float(np.mean(gt)) * 1e3
        del graph

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "segment_ids", "positions"] + \
            (["dout"] if w.backward else [])
        hin = {n: t[n].cpu().pin_memory() for n in names}
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                torch.empty(lse.shape, dtype=lse.dtype).pin_memory()]
        if w.backward:
            hout += [torch.empty(out.shape, dtype=out.dtype).pin_memory()
                     for _ in range(3)]
        h2d = sum(x.numel() * x.element_size() for x in hin.values())
        d2h = sum(x.numel() * x.element_size() for x in hout)

        def make_set():
            d = {n: torch.empty_like(t[n]) for n in names}
            d["out"] = torch.empty_like(out)
            d["lse"] = torch.empty_like(lse)
            if w.backward:
                d["grads"] = [torch.empty_like(g) for g in grads]
            return d

        def outputs(d):
            return [d["out"], d["lse"]] + (d["grads"] if w.backward else [])

        # phases: the forward needs q, k, v, ids and positions and yields
        # out and lse; the backward also needs dO and yields the gradients.
        # Each phase's copies go as soon as they can: dO uploads while the
        # forward runs, out and lse download while the backward runs.
        fwd_names = ["q", "k", "v", "segment_ids", "positions"]
        in_phases = [{n: hin[n] for n in fwd_names}]
        out_phases = [hout[:2]]
        run_phases = [lambda d: ops.fwd(
            d["q"], d["k"], d["v"], d["segment_ids"], d["positions"],
            w.theta, max_pos=max_pos, qk_precision=qkp, out=d["out"],
            lse=d["lse"], workspace=workspace)]
        res_phases = [lambda d: [d["out"], d["lse"]]]
        if w.backward:
            in_phases.append({"dout": hin["dout"]})
            out_phases.append(hout[2:])
            run_phases.append(lambda d: ops.bwd(
                d["q"], d["k"], d["v"], d["out"], d["dout"], d["lse"],
                d["segment_ids"], d["positions"], w.theta, max_pos=max_pos,
                qk_precision=qkp, dq=d["grads"][0], dk=d["grads"][1],
                dv=d["grads"][2], workspace=workspace))
            res_phases.append(lambda d: d["grads"])

        def e2e_run(nsteps):
            return pipelined_e2e_phased(dev, in_phases, make_set, run_phases,
                                        res_phases, out_phases, nsteps)

        e2e_run(2)  # warm-up
        s0 = make_set()
        link = copy_floor(dev, hin, s0, hout, outputs(s0))
        del s0
        barrier(ws)
        ems = max_over_ranks(e2e_run(max(2, args.steps)), ws, dev)
        compute_ms = fwd_ms + bwd_ms
        e2e = {"value": (fwd_flop + bwd_flop) * job_scale / (ems / 1e3) / 1e12,
               "unit": "TFLOP/s", "ms_per_step": ems,
               "steps": max(2, args.steps),
               "tokens_per_s": B * N * (1 if strong else ws) / (ems / 1e3),
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "link": {**link,
                        "h2d_gbs": h2d / link["h2d_ms"] / 1e6,
                        "d2h_gbs": d2h / link["d2h_ms"] / 1e6},
               "floor_ms": max(link["both_ms"], compute_ms),
               "over_floor": ems / max(link["both_ms"], compute_ms),
               "copies": "every step uploads its inputs and downloads its "
                         "results through pinned host buffers, on copy "
                         "streams overlapped with the neighbouring steps' "
                         "compute (two device buffer sets) and, within a "
                         "step, dO uploaded during the forward and out/lse "
                         "downloaded during the backward; floor = the "
                         "slower of one step's uploads and downloads run "
                         "together on this link and the step's compute"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        t_host = {k_: (v_.cpu() if torch.is_tensor(v_) else v_)
                  for k_, v_ in t.items()}
        tf, info = oracle_sample(w, t_host, args.cpu_budget, w.backward)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": info["cores"],
               "kind": "oracle", "sample": info["sample"],
               "seconds": info["seconds"], "host_cores": info["host_cores"],
               "cpu_model": cpu_model(),
               "extrapolated_full_step_s":
                   (fwd_flop + bwd_flop) / (tf * 1e12) if tf > 0 else None,
               "extrapolated_note": "extrapolated: the whole step's "
                                    "mask-aware FLOP at the sampled rate"}

    if rank == 0:
        pk = peaks()
        total_flop = (fwd_flop + bwd_flop) * job_scale
        value = total_flop / (ms / 1e3) / 1e12
        peak_burst = pk["bf16_tflops"]
        peak_sus = pk.get("bf16_tflops_sustained", peak_burst)
        fwd_tf = fwd_flop / (fwd_ms / 1e3) / 1e12
        bwd_tf = bwd_flop / (bwd_ms / 1e3) / 1e12 if w.backward else None
        fwd_gbs = fwd_bytes / (fwd_ms / 1e3) / 1e9
        dom = "bwd" if w.backward and bwd_ms > fwd_ms else "fwd"
        ach = bwd_tf if dom == "bwd" else fwd_tf
        kernel = f"{dom}_tc_kernel"
        if small:
            # a few MB per call: launch- and memory-latency-bound, reported
            # against HBM bandwidth
            roof = {"bound": "hbm", "kernel": "forward call (all kernels)",
                    "achieved": fwd_gbs, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": fwd_gbs / pk["hbm_gbs"],
                    "peak_kind": f"copy bandwidth ({pk['source']})",
                    "algorithmic_bytes": fwd_bytes, "traffic": None,
                    "us_per_call": fwd_ms * 1e3,
                    "graph_replay_us_per_call": graph_us}
        else:
            # the timed region is well under a second of back-to-back
            # launches: the burst peak applies
            roof = {"bound": "tensor", "kernel": kernel, "achieved": ach,
                    "peak": peak_burst,
                    "peak_kind": f"bf16 burst ({pk['source']})",
                    "unit": "TFLOP/s", "frac": ach / peak_burst,
                    "frac_of_sustained_peak": ach / peak_sus,
                    "traffic": recorded_traffic(w.name, kernel),
                    "traffic_unit": "bytes per launch (ncu, dram "
                                    "read+write)"}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if strong else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "N": N, "H": job_heads,
                       "heads_per_rank": H, "D": D,
                       "theta": w.theta, "qk_precision": qkp,
                       "segments": w.segments,
                       "passes": "fwd+bwd" if w.backward else "fwd",
                       "visible_pairs_per_head": pairs_per_head,
                       "tiles_visited_per_head": tiles_visited // B,
                       "tiles_full_per_head": tiles_full // B,
                       "executed_tile_pairs_over_visible":
                           tiles_visited * 128 * 128 / max(1, B *
                                                          pairs_per_head),
                       "l2": "inputs smaller than L2: L2 flushed (256 MB "
                             "write) before every timed step" if small else
                             "inputs larger than L2 (no flush)",
                       "parallelism": (f"heads split over {ws} GPUs" if strong
                                       else f"replicas x{ws}")},
            "tokens_per_s": B * N * (1 if strong else ws) / (ms / 1e3),
            "fwd": {"ms": fwd_ms, "tflops": fwd_tf,
                    "frac_of_burst_peak": fwd_tf / peak_burst,
                    "frac_of_sustained_peak": fwd_tf / peak_sus,
                    "hbm_gbs_algorithmic": fwd_gbs,
                    "tokens_per_s": B * N / (fwd_ms / 1e3)},
            "bwd": ({"ms": bwd_ms, "tflops": bwd_tf,
                     "frac_of_burst_peak": bwd_tf / peak_burst,
                     "frac_of_sustained_peak": bwd_tf / peak_sus}
                    if w.backward else None),
            "roofline": roof,
            "gpu_launches": int(launches),
            "device_status": status,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
