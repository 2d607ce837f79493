"""Benchmark of sparse-graph causal attention on B200.

    python bench.py --gpus N --steps K --warmup W [--workload NAME] [--impl reference]

One step = the whole hot path over one batch of synthetic input on its fixed
neighbour graph: forward (out, lse) and backward (dq, dk, dv).  The default
workload is the 16,384-token layer of "SpatialLM-Mini ..." (B1 H4 T16384 D64
bf16, window 32 + distance links 2^k, k = 0..13); its structured graph is
built once before the timed region (it has no device work: the kernels
enumerate it from the window and the distances), and the end-to-end pass
rebuilds it every step.  The headline value is query-key edges per second of
fwd+bwd, summed over all ranks; every rank runs its own replica (the heads of
a batch are independent problems: weak scaling, no collective on the data
path).

Timing: W untimed warm-up steps; then K steps, each bracketed by its own CUDA
events on the launching stream, with a 256 MiB buffer written between steps
so that no step finds its inputs in the 126 MB L2; barrier + synchronize on
both sides; the max over ranks.  A second pass records per-kernel events for
the roofline of the dominant kernel; a third measures the same step end to
end from pinned host buffers (copies inside the timed region).  nvidia-smi
samples the clocks during the timed region.

The same line also carries, under "workloads", the other named workloads at
a few steps each (same timing rules, own roofline and clocks): the W = 4096
band (fwd+bwd), the graph-view CSR mask at T = 2^20 (fwd, with the timed
CSR normalise + transpose build), the T = 2^27 sequence (fwd), the 16K layer
with grouped-query attention and with learned-coordinate scores (fwd+bwd),
and decode against 16K caches.  The end-to-end pass streams the (b, h)
slices through separate upload, kernel and download streams.

``--impl reference`` times the CPU oracle (the plain fp64 statement of the
method) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sparse-attn query-key edges/s (fwd, fwd+bwd) at T=16K and % of roofline"

# Algorithmic (compulsory) bytes of each kernel per (b, h) slice: every input
# row read once and every output row written once.  es = element size.
#   fwd                      q, k, v read; out written; lse written
#   bwd, dQ (+ Delta)        q, k, v, out, dout read; dq written; lse read; Delta written
#   bwd, dK/dV               q, k, v, dout read; dk, dv written; lse, Delta read
KERNEL_BYTES = {
    "fwd": lambda T, D, es: 4 * T * D * es + 4 * T,
    "bwd_dq": lambda T, D, es: 6 * T * D * es + 8 * T,
    "bwd_dkdv": lambda T, D, es: 6 * T * D * es + 8 * T,
}


def kernel_bytes(kc: str, w) -> int:
    """KERNEL_BYTES over the whole job, with k, v, dk, dv on the key/value heads
    (grouped-query attention: Hkv <= H)."""
    B, H, Hk, T, D, es = w.B, w.H, w.kv_heads, w.T, w.D, w.elem_size
    rows = {"fwd": (2 * H + 2 * Hk, 4 * H), "bwd_dq": (4 * H + 2 * Hk, 8 * H),
            "bwd_dkdv": (2 * H + 4 * Hk, 8 * H)}[kc]
    return B * T * (rows[0] * D * es + rows[1])
# Algorithmic FLOPs per edge: forward 4D (q.k and p.v); backward 10D split as
# dQ kernel 6D (S recompute, dP, dQ) and dK/dV kernel 4D (dV, dK); the dK/dV
# kernel's own recomputation of S and dP is not counted.
KERNEL_FLOPS_PER_EDGE = {"fwd": lambda D: 4 * D, "bwd_dq": lambda D: 6 * D,
                         "bwd_dkdv": lambda D: 4 * D}


def kernel_class(name: str) -> str:
    if name.endswith("bwd_dq"):
        return "bwd_dq"
    if name.endswith("bwd_dkdv"):
        return "bwd_dkdv"
    return "fwd"


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` at `workload` from the committed ncu
    summary (profiles/traffic.json), or None when there is none or the
    kernel's source changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(p))[workload][kernel]
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None
    if hashlib.sha256(src).hexdigest() != rec["source_sha256"]:
        return None
    return rec["bytes"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def edge_count(w: synth.Workload, g) -> int:
    return int(g.nnz) * w.B * w.H


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    mhz.append(float(f[1]))
                    mx = float(f[2])
                except ValueError:
                    continue
                for n, val in zip(names, f[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(n)
            os.unlink(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


def dist_setup(n_gpus):
    if n_gpus > 1 or "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
        return dist, dist.get_rank(), dist.get_world_size()
    return None, 0, 1


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ CPU oracle

def cpu_oracle_run(w: synth.Workload, seconds: float, seed_rows: int = 7):
    """Time the oracle as it stands on rows of slice 0 of the workload (fwd +
    bwd), growing the row sample until about `seconds` of CPU work.  Returns
    (edges/s, edges, seconds, description)."""
    import oracle
    o = oracle.get()
    x = synth.make_qkv(w, device="cpu", with_dout=True)
    D, T = w.D, w.T

    def host(name, rows):
        t = x[name].view(w.B * w.H, T, D)[0][torch.as_tensor(rows)]
        if w.dtype == "bf16":
            return t.contiguous().view(torch.int16).numpy().view(np.uint16)
        return t.contiguous().numpy()

    n_rows, done_edges, done_s = 256, 0, 0.0
    rng = np.random.default_rng(seed_rows)
    while done_s < seconds and n_rows <= T:
        rows = np.sort(rng.choice(T, size=n_rows, replace=False)).astype(np.int64)
        rp, ci = o.structured_rows(rows, w.W, w.exps)
        keys, local = np.unique(ci, return_inverse=True)
        q, do = host("q", rows), host("dout", rows)
        k, v = host("k", keys), host("v", keys)
        t0 = time.perf_counter()
        o.fwd(q, k, v, rp, local.astype(np.int32), w.scale, dtype=w.dtype)
        o.bwd(q, k, v, do, rp, local.astype(np.int32), w.scale, dtype=w.dtype)
        done_s += time.perf_counter() - t0
        done_edges += int(rp[-1])
        n_rows = min(T, n_rows * 2)  # whole slices again once the sample reaches T rows
    desc = (f"fwd+bwd of {done_edges} edges: random query rows of slice 0 of {w.name}, "
            f"oracle single-threaded fp64 C")
    return done_edges / done_s, done_edges, done_s, desc


def run_reference(args, dist, rank, world):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    per_step = min(args.cpu_seconds, max(0.5, min(3.0, 150.0 / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        cpu_oracle_run(w, per_step / 4)
    edges, secs = 0, 0.0
    for _ in range(args.steps):
        _, e, s, desc = cpu_oracle_run(w, per_step)
        edges += e
        secs += s
    v = edges / secs
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "edges/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "D": w.D, "W": w.W,
                       "dilation_exps": list(w.exps), "pass": "fwd+bwd",
                       "parallelism": "replicas"},
            "cpu_baseline": {"value": v, "unit": "edges/s", "cores": 1, "kind": "oracle",
                             "sample": desc, **host_info()},
            "e2e": {"value": v, "unit": "edges/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU arm

# Workloads timed besides the headline one (few steps each): name -> pass.
EXTRA_WORKLOADS = ("band_32k", "csr_1m", "extreme_128m", "gqa_16k", "dist_16k", "decode_16k")


def host_info():
    """CPU model and logical core count of this host (for the CPU baseline)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def gather_model_bytes(w: synth.Workload, g, dev) -> tuple:
    """Bytes a forward must move from HBM when the gathered rows that cannot
    stay in L2 miss it: the compulsory bytes plus one K and one V row per such
    edge, plus the CSR lists.  CSR workload: the edges outside the window and
    the 16 global keys (random keys drawn from the whole history).  Structured
    graph: the distance links o whose rows were last streamed more than an
    L2 ago (o * 4 D es > L2 bytes).  Returns (bytes per replica, description)."""
    es = w.elem_size
    comp = kernel_bytes("fwd", w)
    row2 = 2 * w.D * es
    if w.csr:
        rp, ci, _, _ = sa_export(g)
        deg = rp[1:] - rp[:-1]
        rows = torch.repeat_interleave(torch.arange(w.T, device=rp.device), deg)
        far = (ci.long() >= 16) & (ci.long() <= rows - w.band_hint)
        n_far = int(far.sum())
        del rp, ci, rows, far
        lists = 8 * (w.T + 1) + 4 * int(g.nnz)
        return (comp + lists + row2 * n_far * w.B * w.H,
                f"compulsory + CSR lists + {row2} B per edge outside the window and the 16 "
                f"global keys ({n_far} per slice)")
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_far = sum(w.T - (1 << e) for e in w.exps
                if (1 << e) >= w.W and (1 << e) < w.T and (1 << e) * 4 * w.D * es > l2)
    return (comp + row2 * n_far * w.B * w.H,
            f"compulsory + {row2} B per distance-link edge reaching back more than "
            f"L2 ({l2} B) / {4 * w.D * es} B per row ({n_far} per slice)")


def two_pass_model_bytes(w: synth.Workload) -> tuple:
    """Bytes of the two-pass forward (band kernel, then the link pass over the
    links of at least 2^13 rows in class order, which keeps their rows in
    L2): the compulsory bytes, plus the link pass's own q read, out and lse
    read and written, and one more read of K and V (each class's rows once).
    The first pass's links are all shorter than 2^13 rows and hit L2."""
    es = w.elem_size
    BH, BHkv = w.B * w.H, w.B * w.kv_heads
    extra = BH * (3 * w.T * w.D * es + 8 * w.T) + BHkv * 2 * w.T * w.D * es
    return (kernel_bytes("fwd", w) + extra,
            "two passes: compulsory + the link pass's q, out and lse once more and K and V once "
            "more (the class order keeps the long links' rows in L2)")


def sa_export(g):
    import sparse_graph_causal_b200 as sa
    return sa.sparse_attn_graph_export(g)


def time_workload(sa, w: synth.Workload, dev, rank, world, dist, steps, warmup, fwd_only,
                  use_graph=True, want_e2e=False, args=None):
    """Time one workload: K steps with CUDA events (L2 flushed between steps),
    per-kernel events for the roofline, a fwd-only pass, optionally the
    end-to-end pass.  Returns a dict of results (rank-max times)."""
    stream = torch.cuda.current_stream()
    x = synth.make_qkv(w, device=dev, seed=w.seed + 17 * rank, with_dout=w.bwd and not fwd_only)
    q, k, v = x["q"], x["k"], x["v"]
    dout = x.get("dout")
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    do_bwd = w.bwd and not fwd_only
    dq = torch.empty_like(q) if do_bwd else None
    dk = torch.empty_like(k) if do_bwd else None
    dv = torch.empty_like(v) if do_bwd else None
    graph_build_ms = None
    builds, builds_host = [], []
    if w.csr:
        # graph view: raw CSR rows -> normalised lists + transpose, timed alone
        rp_h, ci_h = synth.csr_random_rows(w.T, seed=w.graph_seed)
        rp_d, ci_d = torch.from_numpy(rp_h).to(dev), torch.from_numpy(ci_h).to(dev)
        del rp_h, ci_h
        g0 = None
        for _ in range(3):
            if g0 is not None:
                g0.close()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0 = time.perf_counter()
            a.record(stream)
            g0 = sa.sparse_attn_graph_build_csr(rp_d, ci_d, band_hint=w.band_hint)
            b.record(stream)
            torch.cuda.synchronize()
            builds_host.append(1e3 * (time.perf_counter() - t0))
            builds.append(a.elapsed_time(b))
        graph_build_ms = max_over_ranks(dist, min(builds))
        del rp_d, ci_d
    else:
        g0 = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    ws = (torch.empty(sa.sparse_attn_bwd_workspace_size(q, g0), dtype=torch.uint8, device=dev)
          if do_bwd else None)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    E = edge_count(w, g0)

    def eager_step():
        sa.sparse_attn_fwd(q, k, v, g0, w.scale, out=out, lse=lse)
        if do_bwd:
            sa.sparse_attn_bwd(q, k, v, out, lse, dout, g0, w.scale, dq=dq, dk=dk, dv=dv,
                               workspace=ws)

    for _ in range(max(3, warmup)):
        flush.fill_(1)
        eager_step()
    sa.sparse_attn_check_device()
    torch.cuda.synchronize()

    # The timed step replays fwd (+ bwd) captured once in a CUDA graph (the
    # neighbour graph is fixed in advance and built outside the step).
    cuda_graph = None
    launches_per_step = None
    if use_graph:
        cuda_graph = torch.cuda.CUDAGraph()
        n0 = sa.sparse_attn_launch_count()
        with torch.cuda.graph(cuda_graph):
            eager_step()
        launches_per_step = sa.sparse_attn_launch_count() - n0
        torch.cuda.synchronize()

    def step():
        if cuda_graph is not None:
            cuda_graph.replay()
        else:
            eager_step()

    for _ in range(3):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()

    # ---- timed region: K steps, L2 flushed between steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    launches0 = sa.sparse_attn_launch_count()
    with ClockSampler(dev.index or 0) as clk:
        barrier(dist)
        torch.cuda.synchronize()
        for a, b in evs:
            flush.fill_(1)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        barrier(dist)
    launches = sa.sparse_attn_launch_count() - launches0
    if cuda_graph is not None:
        launches = launches_per_step * steps
    sa.sparse_attn_check_device()
    ms = [a.elapsed_time(b) for a, b in evs]
    ms_step = max_over_ranks(dist, sum(ms)) / steps

    # ---- per-kernel event timing (separate pass) for the roofline
    sa.sparse_attn_profile_begin(True)
    for _ in range(steps):
        flush.fill_(1)
        eager_step()
    prof = sa.sparse_attn_profile_end()
    kt = {n: (c, t) for n, (c, t) in prof.items() if not n.startswith("graph_")}
    dom = max(kt, key=lambda n: kt[n][1])
    cnt, tot = kt[dom]
    avg_ms = max_over_ranks(dist, tot / cnt)
    es = w.elem_size
    kc = kernel_class(dom)
    alg_bytes = kernel_bytes(kc, w)
    alg_flops = KERNEL_FLOPS_PER_EDGE[kc](w.D) * E
    hbm, tflops, src = peaks()
    shares = {n: round(t / sum(tt for _, tt in kt.values()), 4) for n, (_, t) in kt.items()}
    # the kernel's bound: compulsory intensity against the machine balance
    tensor_bound = alg_flops / alg_bytes > (tflops * 1e12) / (hbm * 1e9) and w.dtype == "bf16"
    if tensor_bound:
        achieved = alg_flops / (avg_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tflops, "unit": "TFLOP/s",
                    "frac": achieved / tflops, "peak_source": f"{src} bf16_tflops"}
    else:
        achieved = alg_bytes / (avg_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "peak_source": f"{src} hbm_gbs"}
    roofline.update({"traffic": ncu_traffic(w.name, dom), "kernel": dom, "kernel_ms": avg_ms,
                     "algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops,
                     "kernel_shares": shares,
                     "kernel_ms_all": {n: t / c for n, (c, t) in kt.items()}})
    if not tensor_bound and kc == "fwd" and (w.csr or any((1 << e) >= w.W for e in w.exps)):
        if "link_pass" in kt:
            # two forward passes: the model covers both kernels
            mb, desc = two_pass_model_bytes(w)
            fwd_ms = max_over_ranks(dist, sum(kt[n][1] / kt[n][0] for n in ("band_fwd", "link_pass")))
        else:
            mb, desc = gather_model_bytes(w, g0, dev)
            fwd_ms = avg_ms
        roofline["gather_model"] = {"bytes": mb, "achieved": mb / (fwd_ms * 1e-3) / 1e9,
                                    "frac": mb / (fwd_ms * 1e-3) / 1e9 / hbm, "model": desc,
                                    "ms": fwd_ms}

    # ---- fwd-only throughput
    fwd_ev = []
    for _ in range(min(steps, 50)):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sa.sparse_attn_fwd(q, k, v, g0, w.scale, out=out, lse=lse)
        b.record(stream)
        fwd_ev.append((a, b))
    torch.cuda.synchronize()
    fwd_ms = max_over_ranks(dist, sum(a.elapsed_time(b) for a, b in fwd_ev) / len(fwd_ev))

    e2e = None
    if want_e2e:
        e2e = measure_e2e(sa, w, x, out, lse, dq, dk, dv, ws, g0, flush, stream, do_bwd, E,
                          world, dist, args)
    res = {
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "D": w.D, "W": w.W,
                   "dilation_exps": list(w.exps), "csr": w.csr, "edges_per_replica": E,
                   "pass": "fwd+bwd" if do_bwd else "fwd",
                   "l2": "256 MiB buffer written between timed steps",
                   "timed_step": ("CUDA-graph replay of " if cuda_graph is not None else
                                  "eager ") + ("fwd+bwd" if do_bwd else "fwd"),
                   "link_pass": args.link_pass if args is not None else "auto",
                   "parallelism": f"replicas x{world}"},
        "steps": steps, "ms_per_step": ms_step, "edges_per_s": E * world / (ms_step * 1e-3),
        "fwd_ms": fwd_ms, "fwd_edges_per_s": E * world / (fwd_ms * 1e-3),
        "tokens_per_s": w.B * w.T * world / (ms_step * 1e-3), "graph_build_ms": graph_build_ms,
        "graph_build_ms_each": [round(b, 3) for b in builds] if builds else None,
        "graph_build_host_ms_each": [round(b, 3) for b in builds_host] if builds else None,
        "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary(),
    }
    del cuda_graph
    g0.close()
    return res


def _timed_steps(step, steps, flush, stream, dist, dev):
    """K steps bracketed by CUDA events, L2 flushed between steps; returns
    (rank-max mean ms, clocks)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with ClockSampler(dev.index or 0) as clk:
        barrier(dist)
        torch.cuda.synchronize()
        for a, b in evs:
            flush.fill_(1)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        barrier(dist)
    return max_over_ranks(dist, sum(a.elapsed_time(b) for a, b in evs)) / steps, clk.summary()


def _roofline_bytes(sa, step, steps, flush, kernel_bytes_of, dist):
    """Per-kernel events of `steps` eager steps; the dominant kernel against
    the measured HBM bandwidth with its compulsory bytes."""
    sa.sparse_attn_profile_begin(True)
    for _ in range(steps):
        flush.fill_(1)
        step()
    prof = sa.sparse_attn_profile_end()
    dom = max(prof, key=lambda n: prof[n][1])
    cnt, tot = prof[dom]
    avg_ms = max_over_ranks(dist, tot / cnt)
    hbm, _, src = peaks()
    b = kernel_bytes_of(dom)
    achieved = b / (avg_ms * 1e-3) / 1e9
    tot_all = sum(t for _, t in prof.values())
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": f"{src} hbm_gbs", "traffic": None,
            "kernel": dom, "kernel_ms": avg_ms, "algorithmic_bytes": b,
            "kernel_shares": {n: round(t / tot_all, 4) for n, (_, t) in prof.items()},
            "kernel_ms_all": {n: t / c for n, (c, t) in prof.items()}}


def time_dist(sa, w, dev, rank, world, dist, steps, warmup, fwd_only, **_):
    """Learned-coordinate scoring (s = -scale |a_i - c_j|^2) on the workload's
    graph, fwd+bwd, CUDA-graph replay."""
    stream = torch.cuda.current_stream()
    x = synth.make_qkv(w, device=dev, seed=w.seed + 17 * rank)
    v, dout = x["v"], x["dout"]
    a_, c_ = synth.make_coords(w, device=dev, seed=w.seed + 7 + 17 * rank)
    g0 = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    out = torch.empty_like(v)
    lse = torch.empty(v.shape[:3], dtype=torch.float32, device=dev)
    da, dc, dv = torch.empty_like(a_), torch.empty_like(c_), torch.empty_like(v)
    ws = torch.empty(sa.sparse_attn_dist_bwd_workspace_size(v, g0), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    E = edge_count(w, g0)

    def eager():
        sa.sparse_attn_dist_fwd(a_, c_, v, g0, w.scale, out=out, lse=lse)
        sa.sparse_attn_dist_bwd(a_, c_, v, out, lse, dout, g0, w.scale, da=da, dc=dc, dv=dv,
                                workspace=ws)

    for _ in range(max(3, warmup)):
        eager()
    sa.sparse_attn_check_device()
    cg = torch.cuda.CUDAGraph()
    n0 = sa.sparse_attn_launch_count()
    with torch.cuda.graph(cg):
        eager()
    per_step = sa.sparse_attn_launch_count() - n0
    for _ in range(3):
        cg.replay()
    ms, clk = _timed_steps(cg.replay, steps, flush, stream, dist, dev)
    sa.sparse_attn_check_device()
    B, H, T, D, es = w.B, w.H, w.T, w.D, w.elem_size
    # compulsory bytes per kernel: value rows, coordinates (12 B per row),
    # lse / Delta (4 B per row), outputs
    kb = {"dist_fwd": B * H * T * (2 * D * es + 24 + 4),
          "dist_bwd_da": B * H * T * (3 * D * es + 24 + 12 + 8),
          "dist_bwd_dcdv": B * H * T * (3 * D * es + 24 + 12 + 8)}
    roof = _roofline_bytes(sa, eager, steps, flush, lambda n: kb[n], dist)
    del cg
    g0.close()
    return {"config": {"workload": w.name, "B": B, "H": H, "T": T, "D": D, "W": w.W,
                       "dilation_exps": list(w.exps), "scale": w.scale, "pass": "fwd+bwd",
                       "score": "-scale |a_i - c_j|^2, 3-D coordinates",
                       "l2": "256 MiB buffer written between timed steps",
                       "timed_step": "CUDA-graph replay of fwd+bwd",
                       "parallelism": f"replicas x{world}"},
            "steps": steps, "ms_per_step": ms, "edges_per_s": E * world / (ms * 1e-3),
            "tokens_per_s": B * T * world / (ms * 1e-3), "roofline": roof,
            "gpu_launches": per_step * steps, "clocks": clk}


def time_decode(sa, w, dev, rank, world, dist, steps, warmup, fwd_only, **_):
    """One new token per sequence (B sequences, H query heads over Hkv cache
    heads, caches of T rows) at positions drawn in [T/2, T)."""
    stream = torch.cuda.current_stream()
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 17 * rank)
    B, H, Hk, T, D = w.B, w.H, w.kv_heads, w.T, w.D
    q = torch.empty((B, H, 1, D), dtype=torch.float32, device=dev).normal_(
        generator=g).to(w.torch_dtype)
    kc = torch.empty((B, Hk, T, D), dtype=torch.float32, device=dev).normal_(
        generator=g).to(w.torch_dtype)
    vc = torch.empty((B, Hk, T, D), dtype=torch.float32, device=dev).normal_(
        generator=g).to(w.torch_dtype)
    pos = torch.randint(T // 2, T, (B,), generator=g, device=dev, dtype=torch.int64)
    g0 = sa.sparse_attn_graph_build_structured(T, w.W, list(w.exps))
    out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def eager():
        sa.sparse_attn_decode(q, kc, vc, pos, g0, w.scale, out=out, lse=lse)

    for _ in range(max(3, warmup)):
        eager()
    sa.sparse_attn_check_device()
    # the timed step replays the decode call captured once in a CUDA graph,
    # as a serving loop would run it (eager, the host's launch path shows up
    # in a kernel of ~10 us)
    cg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cg):
        eager()
    torch.cuda.synchronize()
    for _ in range(3):
        cg.replay()
    ms, clk = _timed_steps(cg.replay, steps, flush, stream, dist, dev)
    sa.sparse_attn_check_device()
    # neighbours per query: min(p + 1, W) + #{2^k : W <= 2^k <= p}
    ps = pos.cpu().tolist()
    offs = sorted({1 << e for e in w.exps if (1 << e) >= w.W})
    deg = [min(p + 1, w.W) + sum(1 for o in offs if o <= p) for p in ps]
    edges = sum(deg) * H
    es = w.elem_size
    # compulsory bytes: q and out rows, lse, one K and one V row per edge of
    # each query head (rows shared by the heads of a group are counted once)
    bytes_ = B * H * (2 * D * es + 4) + sum(deg) * Hk * 2 * D * es
    roof = _roofline_bytes(sa, eager, steps, flush, lambda n: bytes_, dist)
    g0.close()
    return {"config": {"workload": w.name, "B": B, "H": H, "Hkv": Hk, "T_cache": T, "D": D,
                       "W": w.W, "dilation_exps": list(w.exps), "positions": "uniform in [T/2, T)",
                       "pass": "decode (one query per sequence and head)",
                       "timed_step": "CUDA-graph replay of the decode call",
                       "l2": "256 MiB buffer written between timed steps",
                       "parallelism": f"replicas x{world}"},
            "steps": steps, "ms_per_step": ms, "edges_per_s": edges * world / (ms * 1e-3),
            "queries_per_s": B * H * world / (ms * 1e-3), "roofline": roof,
            "gpu_launches": steps, "clocks": clk}


def run_gpu(args, dist, rank, world):
    import sparse_graph_causal_b200 as sa
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    sa.sparse_attn_set_link_pass({"auto": sa.SA_LINKS_AUTO, "split": sa.SA_LINKS_SPLIT,
                                  "one": sa.SA_LINKS_ONE_PASS}[args.link_pass])
    r = time_workload(sa, w, dev, rank, world, dist, args.steps, args.warmup, args.fwd_only,
                      use_graph=not args.no_graph, want_e2e=not args.no_e2e, args=args)
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_extra:
        chosen = set(filter(None, args.extra.split(",")))
        for name in EXTRA_WORKLOADS:
            if name == w.name or name not in chosen:
                continue
            wx = synth.WORKLOADS[name]
            timer = {"attn": time_workload, "dist": time_dist, "decode": time_decode}[wx.kind]
            extra[name] = timer(sa, wx, dev, rank, world, dist, args.extra_steps, 3, False,
                                args=args)
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and not w.csr:
        v_cpu, e_cpu, s_cpu, desc = cpu_oracle_run(w, args.cpu_seconds)
        cpu = {"value": v_cpu, "unit": "edges/s", "cores": 1, "kind": "oracle",
               "sample": f"{desc}; {s_cpu:.1f} s", **host_info()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": r["edges_per_s"], "unit": "edges/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic", "config": r["config"],
            "fwd_edges_per_s": r["fwd_edges_per_s"], "fwd_ms": r["fwd_ms"],
            "tokens_per_s": r["tokens_per_s"], "graph_build_ms": r["graph_build_ms"],
            "graph_build_ms_each": r["graph_build_ms_each"],
            "graph_build_host_ms_each": r["graph_build_host_ms_each"],
            "roofline": r["roofline"], "cpu_baseline": cpu, "e2e": r["e2e"],
            "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
            "workloads": extra,
        }
        print(json.dumps(line), flush=True)


def measure_e2e(sa, w, x, out, lse, dq, dk, dv, ws, g0, flush, stream, do_bwd, E, world, dist,
                args):
    """Same step through the public API from pinned host memory: H2D of the
    inputs and D2H of the results inside the timed region.  The (b, h) slices
    are independent problems on the same graph, so the step runs slice by
    slice through an upload, a kernel and a download stream: the copies of
    one slice overlap the kernels of another (and uploads overlap downloads),
    as a user streaming heads from host memory would run it."""
    BH, T, D = w.B * w.H, w.T, w.D
    names_in = ("q", "k", "v") + (("dout",) if do_bwd else ())
    names_out = ("out",) + (("dq", "dk", "dv") if do_bwd else ())
    dev_out = {"out": out, "dq": dq, "dk": dk, "dv": dv}
    hx = {n: x[n].cpu().pin_memory() for n in names_in}
    hout = {n: torch.empty(x["q"].shape, dtype=x["q"].dtype).pin_memory() for n in names_out}
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in hout.values())

    def sl(t, c):  # slice c of a [B, H, T, D] tensor as a contiguous [1, 1, T, D] view
        return t.view(BH, T, D)[c].view(1, 1, T, D)

    # three streams: uploads, kernels, downloads; slice c's kernels wait for
    # its upload and its download for its kernels, so the copy engines stream
    # continuously in both directions while the kernels run in between
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ws_c = (torch.empty(sa.sparse_attn_bwd_workspace_size(sl(x["q"], 0), g0), dtype=torch.uint8,
                        device=x["q"].device) if do_bwd else None)
    lse2 = lse.view(BH, T)

    def e2e_step(start):
        g = g0 if w.csr else sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
        for s_ in (up, comp, down):
            s_.wait_event(start)
        for c in range(BH):
            # the forward's inputs first, dout after them; out leaves as soon
            # as the forward is done, the gradients after the backward
            ev = {}
            with torch.cuda.stream(up):
                for n in names_in:
                    sl(x[n], c).copy_(sl(hx[n], c), non_blocking=True)
                    if n in ("v", "dout"):
                        ev[n] = torch.cuda.Event()
                        ev[n].record(up)
            comp.wait_event(ev["v"])
            with torch.cuda.stream(comp):
                qc, kc, vc = sl(x["q"], c), sl(x["k"], c), sl(x["v"], c)
                oc, lc = sl(out, c), lse2[c].view(1, 1, T)
                sa.sparse_attn_fwd(qc, kc, vc, g, w.scale, out=oc, lse=lc, stream=comp)
                ev["fwd"] = torch.cuda.Event()
                ev["fwd"].record(comp)
                if do_bwd:
                    comp.wait_event(ev["dout"])
                    sa.sparse_attn_bwd(qc, kc, vc, oc, lc, sl(x["dout"], c), g, w.scale,
                                       dq=sl(dq, c), dk=sl(dk, c), dv=sl(dv, c), workspace=ws_c,
                                       stream=comp)
                    ev["bwd"] = torch.cuda.Event()
                    ev["bwd"].record(comp)
            with torch.cuda.stream(down):
                for n in names_out:
                    down.wait_event(ev["fwd" if n == "out" else "bwd"])
                    sl(hout[n], c).copy_(sl(dev_out[n], c), non_blocking=True)
        for s_ in (up, comp, down):
            done = torch.cuda.Event()
            done.record(s_)
            stream.wait_event(done)

    for _ in range(3):
        st = torch.cuda.Event()
        st.record(stream)
        e2e_step(st)
    torch.cuda.synchronize()
    e_evs = []
    n_e2e = min(args.steps, 50)
    barrier(dist)
    for _ in range(n_e2e):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step(a)
        b.record(stream)
        e_evs.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, sum(a.elapsed_time(b) for a, b in e_evs) / n_e2e)
    return {"value": E * world / (e2e_ms * 1e-3), "unit": "edges/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "graph": "built per step" if not w.csr else "CSR graph built once",
            "pipelining": f"{BH} slices through upload, kernel and download streams (the "
                          "copies of one slice overlap the kernels of another)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    # the main line times a dot-product workload; the learned-coordinate and
    # decode workloads are timed under "workloads"
    ap.add_argument("--workload", default="spatiallm_16k",
                    choices=sorted(n for n, x in synth.WORKLOADS.items() if x.kind == "attn"))
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls, no CUDA graph")
    ap.add_argument("--no-e2e", action="store_true", help="skip the pinned-host end-to-end pass")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload, not the other named workloads")
    ap.add_argument("--extra", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated subset of the other named workloads to time")
    ap.add_argument("--extra-steps", type=int, default=5,
                    help="timed steps of each of the other named workloads")
    ap.add_argument("--link-pass", default="auto", choices=["auto", "split", "one"],
                    help="long distance links in a second forward pass: the library's "
                         "automatic choice, always, or never (sparse_attn_set_link_pass)")
    args = ap.parse_args()
    unknown = set(filter(None, args.extra.split(","))) - set(EXTRA_WORKLOADS)
    if unknown:
        ap.error(f"--extra: unknown workloads {sorted(unknown)}")
    dist, rank, world = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, dist, rank, world)
        else:
            run_gpu(args, dist, rank, world)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
