#!/usr/bin/env python
"""Benchmark of the HHR decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hhr|reference]
                    [--workload NAME] [--no-extra] [--no-dense] [--no-cpu-baseline]

One step = one decode token of the workload: hhr_decode_step on every layer
in order (32 layers of Llama-3.1-8B shape at 128K context by default),
captured in one CUDA graph.  Inputs are resident in HBM before timing; the
headline KV cache (17.5 GB) is far larger than L2, so every layer's bytes are
evicted by the other 31 layers before they are read again (no L2 flush).
The other workloads (`per_config`) are timed step by step with CUDA events,
L2 flushed (a 2 x L2 write) between steps outside the timed events; their
figure is the median over the steps.

Rank 0 prints one JSON line.  Under torchrun every rank runs its own replica
of the workload (independent sequences, no collective on the data path);
`value` counts the tokens of all ranks over the slowest rank's time.
`--impl reference` times the fp64 CPU oracle instead (bounded sample).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HHR decode-attention tokens/s at 128K ctx; achieved HBM GB/s vs ~8 TB/s peak"


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["hhr", "reference"], default="hhr")
    p.add_argument("--workload", default="llama_32l_128k")
    p.add_argument("--layers", type=int, default=None, help="fewer layers (profiling runs only)")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="only the headline workload")
    p.add_argument("--extra-steps", type=int, default=60)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--cpu-workers", type=int, default=0, help="all-cores oracle workers (0: every core, at most 64)")
    p.add_argument("--soak-seconds", type=float, default=1.0)
    return p.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (host side; CPU-testable with gloo)
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def dist_init(backend: str):
    import datetime
    import torch.distributed as dist
    rank, _, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
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


def whole_job_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / max_seconds


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must touch per decode step)
# ---------------------------------------------------------------------------

def hhr_bytes_per_head(L: int, P: int, N: int, k: int, G: int, nb: int, d: int = 128) -> dict:
    """Bytes one (sequence, KV head) decode must move: page metadata, codes of
    the candidate rows, the kept K'/V rows, q and out, and R_h, W_h."""
    np_ = -(-L // P)
    Neff = min(N, np_)
    # candidate rows: exact when every kept page is full (L a multiple of P, or
    # the partial last page not kept); otherwise over by fewer than P rows
    cand = min(Neff * P, L)
    keff = min(k, cand)
    return dict(meta=np_ * 2 * d * 2, codes=cand * (nb // 8), gather=keff * 2 * d * 2,
                qo=G * (d * 2 + d * 4), rw=d * d * 4 + nb * d * 2, cand=cand, keff=keff, pages=Neff)


def dense_bytes_per_head(L: int, G: int, d: int = 128) -> int:
    return L * 2 * d * 2 + G * (d * 2 + d * 4) + d * d * 4


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def kernel_source_hash() -> str:
    """sha256 over the CUDA sources of the library (any edit changes it)."""
    import hashlib
    csrc = os.path.join(ROOT, "hash_sparse_attention_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per hhr_sparse_kernel launch from the committed ncu summary,
    when that summary was taken on the current sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"hhr_sparse_kernel_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ": " in line:
                k, v = line[2:].split(": ", 1)
                fields[k.strip()] = v.strip().strip("`")
    try:
        if fields.get("sources_sha256") != kernel_source_hash() or fields.get("workload") != workload:
            return None
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk.get("bf16_tflops", 1590.0)),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def oracle_units(w, n_heads: int, layer: int = 0):
    """Oracle-built caches of the first n_heads KV heads of one layer (sequence
    0), generated on the CPU (the oracle's timing never touches the GPU)."""
    from hash_sparse_attention_b200.synth import make_layer
    from oracle import hhr_oracle as O
    li = make_layer(w, layer=layer, device="cpu")
    L = int(li.seq_lens[0])
    G, P = w.group, w.page_size
    R32 = li.R.double().numpy()
    Wn = li.W.double().numpy()
    units = []
    for h in range(n_heads):
        K = (li.K_logical if w.paged else li.K)[0, h, :L].double().numpy()
        V = (li.V_logical if w.paged else li.V)[0, h, :L].double().numpy()
        Q = li.q[0, h * G:(h + 1) * G].double().numpy()
        Kp, mn, mx, codes = O.build_head(K, R32[h], Wn[h], L, P)
        units.append(dict(Q=Q, R=R32[h], W=Wn[h], Kp=Kp, V=V, mn=mn, mx=mx, codes=codes, L=L, P=P,
                          N=int(li.n_keep[0]), k=int(li.top_k[0])))
    del li
    return units


def oracle_decode_unit(u):
    from oracle import hhr_oracle as O
    return O.decode_head(u["Q"], u["R"], u["W"], u["Kp"], u["V"], u["mn"], u["mx"], u["codes"], u["L"], u["P"],
                         u["N"], u["k"])


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_ARRAYS = ("Q", "R", "W", "Kp", "V", "mn", "mx", "codes")


def _cpu_worker(path, n_units, seconds, go, q):
    """All-cores oracle leg: one process, one thread, decodes the shared units
    (memory-mapped .npy files) until `seconds` have passed."""
    import json as _json
    import numpy as _np
    from threadpoolctl import threadpool_limits
    with open(os.path.join(path, "meta.json")) as f:
        meta = _json.load(f)
    units = []
    for i in range(n_units):
        u = {k: _np.load(os.path.join(path, f"u{i}_{k}.npy"), mmap_mode="r") for k in _ARRAYS}
        u.update(meta[i])
        units.append(u)
    with threadpool_limits(1):
        go.wait()
        t0 = time.perf_counter()
        done = 0
        while True:
            oracle_decode_unit(units[done % n_units])
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    q.put((done, el))


def cpu_baseline(w, seconds: float, workers: int = 0) -> dict:
    """The fp64 oracle's decode step on whole (layer, KV head) units of the
    workload, on the host cores: one thread, then one process per core (each
    single-threaded), every unit's cache built beforehand (untimed).  Runs
    before the GPU is touched."""
    import multiprocessing as mp
    import shutil
    import tempfile
    from threadpoolctl import threadpool_limits
    import numpy as np
    units = oracle_units(w, min(2, w.num_kv_heads))
    heads_per_token = w.layers * w.num_kv_heads * w.batch
    done = 0
    with threadpool_limits(1):
        t0 = time.perf_counter()
        while True:
            oracle_decode_unit(units[done % len(units)])
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    single = (done / heads_per_token) / el
    out = {"value": single, "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "cpu_model": cpu_model(), "host_cores": host_cores(),
           "sample": f"{done} (layer 0, KV head) decode units of {heads_per_token} per token, "
                     f"{el:.1f} s of fp64 CPU work on one thread; cache build untimed"}
    n = workers if workers > 0 else min(64, host_cores())
    if n > 1:
        base = "/dev/shm" if os.path.isdir("/dev/shm") else None
        tmp = tempfile.mkdtemp(prefix="hhr_oracle_", dir=base)
        try:
            meta = []
            for i, u in enumerate(units):
                for k in _ARRAYS:
                    np.save(os.path.join(tmp, f"u{i}_{k}.npy"), np.ascontiguousarray(u[k]))
                meta.append({k: u[k] for k in ("L", "P", "N", "k")})
            with open(os.path.join(tmp, "meta.json"), "w") as f:
                json.dump(meta, f)
            ctx = mp.get_context("spawn")
            go, q = ctx.Event(), ctx.Queue()
            procs = [ctx.Process(target=_cpu_worker, args=(tmp, len(units), seconds, go, q)) for _ in range(n)]
            for p_ in procs:
                p_.start()
            time.sleep(min(20.0, 2.0 + 0.05 * n))  # workers map the units
            go.set()
            res = [q.get(timeout=seconds + 600) for _ in procs]
            for p_ in procs:
                p_.join(timeout=60)
            total = sum(d / e for d, e in res) / heads_per_token
            out["all_cores"] = {"value": total, "unit": "tokens/s", "cores": n, "kind": "oracle",
                                "sample": f"{sum(d for d, _ in res)} units in {n} single-threaded processes, "
                                          f"{seconds:.0f} s each"}
        finally:
            shutil.rmtree(tmp, ignore_errors=True)
    return out


# ---------------------------------------------------------------------------
# the HHR arm
# ---------------------------------------------------------------------------

def _config_of(hhr, w, li):
    if w.paged:
        return hhr.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.page_size, w.hash_bits, w.context,
                               paged=True, num_blocks=li.K.shape[0], max_blocks_per_seq=li.block_table.shape[1])
    return hhr.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.page_size, w.hash_bits, w.context)


def build_layers(w, dev):
    """Every layer's inputs, drawn on the device, and its cache built in place
    by the library (each build timed with CUDA events)."""
    import torch
    from hash_sparse_attention_b200 import hhr
    from hash_sparse_attention_b200.synth import make_layer
    layers, events = [], []
    for l in range(w.layers):
        li = make_layer(w, layer=l, device=dev)
        cfg = _config_of(hhr, w, li)
        cache = hhr.alloc_cache(cfg, dev, Krot=li.K, V=li.V)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        hhr.build_cache(cfg, li.K, li.V, li.R, li.W, li.seq_lens, li.block_table, cache)
        e1.record()
        events.append((e0, e1))
        lens = [int(x) for x in li.seq_lens.cpu()]
        layers.append(dict(cfg=cfg, cache=cache, R=li.R, W=li.W, q=li.q, seq=li.seq_lens, table=li.block_table,
                           lens=lens, n_keep=li.n_keep, top_k=li.top_k,
                           nk=[int(x) for x in li.n_keep.cpu()], tk=[int(x) for x in li.top_k.cpu()]))
        li.K_logical = li.V_logical = None
        del li
    return layers, events


def with_budgets(w, layers, dev):
    """The same caches with another workload's page and key budgets."""
    import torch
    out = []
    for L in layers:
        nk = [w.keep_for(x) for x in L["lens"]]
        tk = [w.topk_for(x) for x in L["lens"]]
        out.append(dict(L, nk=nk, tk=tk, n_keep=torch.tensor(nk, dtype=torch.int32, device=dev),
                        top_k=torch.tensor(tk, dtype=torch.int32, device=dev)))
    return out


def step_bytes(w, layers, Nmax, Kmax):
    """Algorithmic bytes of one decode step per layer (see hhr_bytes_per_head)."""
    d, Hkv = w.head_dim, w.num_kv_heads
    per_layer = []
    for L in layers:
        tot = 0
        for b, Lb in enumerate(L["lens"]):
            hb = hhr_bytes_per_head(Lb, w.page_size, min(L["nk"][b], Nmax), min(L["tk"][b], Kmax), w.group,
                                    w.hash_bits)
            tot += Hkv * (hb["meta"] + hb["codes"] + hb["gather"] + hb["qo"])
        tot += Hkv * (d * d * 4 + w.hash_bits * d * 2)
        per_layer.append(tot)
    return per_layer


def capture(fn, dev):
    """fn warmed up on a side stream, then captured in a CUDA graph."""
    import torch
    fn()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def timed_steps(graph, steps, world, dev, flush=None):
    """Replays `graph` `steps` times with an event pair around each replay on
    the launching stream.  Without `flush` the replays run back to back and
    the total is the span from the first start to the last end; with it, L2
    is flushed between steps outside the events and the total is the sum.
    Returns (total seconds, per-step milliseconds)."""
    import torch
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world, dev)
    torch.cuda.synchronize()
    for e0, e1 in ev:
        if flush is not None:
            flush.add_(1)
        e0.record(st)
        graph.replay()
        e1.record(st)
    torch.cuda.synchronize()
    barrier(world, dev)
    per = [e0.elapsed_time(e1) for e0, e1 in ev]
    total = sum(per) / 1e3 if flush is not None else ev[0][0].elapsed_time(ev[-1][1]) / 1e3
    return total, per


def measure_workload(w, layers, dev, args, world, flush, with_dense):
    """Decode-step (and dense) throughput of one workload on prepared caches."""
    import torch
    from hash_sparse_attention_b200 import hhr
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    Nmax = max(max(L["nk"]) for L in layers)
    Kmax = max(max(L["tk"]) for L in layers)
    cfg0 = layers[0]["cfg"]
    ws = hhr.decode_workspace(cfg0, Nmax, Kmax, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty(len(layers), B, Hq, d, dtype=torch.float32, device=dev)

    def step():
        for l, L in enumerate(layers):
            hhr.decode_step(L["cfg"], L["q"], L["R"], L["W"], L["cache"], L["seq"], L["table"], L["n_keep"],
                            L["top_k"], Nmax, Kmax, out[l], ws, status=status)
    step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"{w.name}: device status {int(status.item())}"
    g = capture(step, dev)
    for _ in range(max(3, args.warmup)):
        g.replay()
    steps = max(50, args.extra_steps)
    total, per = timed_steps(g, steps, world, dev, flush)
    med = statistics.median(per) / 1e3
    per_layer = step_bytes(w, layers, Nmax, Kmax)
    pk = peaks()
    res = {"tokens_per_s": whole_job_throughput(B, world, max_over_ranks(med, world, dev)),
           "ms_per_step_median": med * 1e3, "steps": steps, "layers": len(layers),
           "bytes_per_step": sum(per_layer), "achieved_gbs": sum(per_layer) / med / 1e9,
           "frac": sum(per_layer) / med / 1e9 / pk["hbm_gbs"],
           "keep_pages": Nmax, "top_k": Kmax,
           "l2": "flushed between steps" if flush is not None else "not flushed (the cache is far larger than L2)"}
    if with_dense:
        dws = hhr.dense_workspace(cfg0, dev)
        dout = torch.empty_like(out)

        def dstep():
            for l, L in enumerate(layers):
                hhr.dense_decode(L["cfg"], L["q"], L["R"], L["cache"], L["seq"], L["table"], dout[l], dws,
                                 status=status)
        dg = capture(dstep, dev)
        for _ in range(3):
            dg.replay()
        _, dper = timed_steps(dg, max(10, steps // 4), world, dev, flush)
        dmed = statistics.median(dper) / 1e3
        dbytes = sum(dense_bytes_per_head(Lb, w.group) for L in layers for Lb in L["lens"] for _ in range(w.num_kv_heads))
        res["dense"] = {"tokens_per_s": whole_job_throughput(B, world, max_over_ranks(dmed, world, dev)),
                        "ms_per_step_median": dmed * 1e3, "achieved_gbs": dbytes / dmed / 1e9,
                        "frac": dbytes / dmed / 1e9 / pk["hbm_gbs"]}
        res["sparse_over_dense"] = dmed / med
        del dg, dws
    del g, ws
    assert int(status.item()) == 0, f"{w.name}: device status {int(status.item())}"
    return res


def run_hhr(args, rank, world):
    import torch
    from hash_sparse_attention_b200 import hhr
    from hash_sparse_attention_b200.synth import WORKLOADS, scaled

    _, local_rank, _ = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    if args.layers is not None:
        w = scaled(w, layers=args.layers)
    B, Hq, Hkv, d, P = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size

    # ---- setup: every layer's cache built in place by the library (each build timed) ----
    layers, build_events = build_layers(w, dev)
    torch.cuda.synchronize()
    q_all = torch.stack([L["q"] for L in layers])
    out_all = torch.empty(w.layers, B, Hq, d, dtype=torch.float32, device=dev)
    cfg0 = layers[0]["cfg"]
    Nmax = max(max(L["nk"]) for L in layers)
    Kmax = max(max(L["tk"]) for L in layers)
    ws = hhr.decode_workspace(cfg0, Nmax, Kmax, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        for l, L in enumerate(layers):
            hhr.decode_step(L["cfg"], q_all[l], L["R"], L["W"], L["cache"], L["seq"], L["table"], L["n_keep"],
                            L["top_k"], Nmax, Kmax, out_all[l], ws, status=status)

    step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    graph = capture(step, dev)

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(local_rank))
    if getattr(props, "uuid", None) is not None:
        u = str(props.uuid)
        sampler.gpu_id = u if u.startswith("GPU-") else f"GPU-{u}"
    sampler.start()
    st = torch.cuda.current_stream()
    # warm-up, plus a short soak so that clocks settle under load
    for _ in range(max(3, args.warmup)):
        graph.replay()
    t_end = time.time() + args.soak_seconds
    while time.time() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    secs, per_step = timed_steps(graph, args.steps, world, dev)
    clocks = sampler.stop()
    secs_max = max_over_ranks(secs, world, dev)

    # e2e: q from pinned host memory, out back to pinned host memory, every step
    q_host = q_all.cpu().pin_memory()
    out_host = torch.empty(out_all.shape, dtype=out_all.dtype).pin_memory()
    for _ in range(3):
        q_all.copy_(q_host, non_blocking=True)
        graph.replay()
        out_host.copy_(out_all, non_blocking=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        q_all.copy_(q_host, non_blocking=True)
        graph.replay()
        out_host.copy_(out_all, non_blocking=True)
    e1.record(st)
    e1.synchronize()
    e2e_secs = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    del graph

    # ---- algorithmic bytes and the roofline of the decode kernel ----
    per_layer_bytes = step_bytes(w, layers, Nmax, Kmax)
    step_total = sum(per_layer_bytes)
    t_step = secs_max / args.steps
    pk = peaks()
    # the timed graph holds only the per-layer decode launches, back to back:
    # the average duration of one layer's launch is the timed region / layers
    mean_layer_s = t_step / len(layers)
    achieved = statistics.mean(per_layer_bytes) / mean_layer_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": profiled_traffic(w.name),
                "algorithmic_bytes_per_launch": statistics.mean(per_layer_bytes),
                "kernel": "hhr_sparse_kernel (one launch per layer; one group of CTAs per KV head: query prep, "
                          "page scan, radix page select, Hamming scores and key select, tensor-core sparse "
                          "attention, merge of the group's CTA partials)",
                "peak_source": pk["source"], "peak_note": "of measured" if pk["source"] == "measured" else "of fallback",
                "step_gbs": step_total / t_step / 1e9, "step_frac": step_total / t_step / 1e9 / pk["hbm_gbs"]}
    build = build_report(w, layers, build_events, clocks, props.multi_processor_count, pk)
    result = {
        "metric": METRIC,
        "value": whole_job_throughput(B * args.steps, world, secs_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step * 1e3,
        "ms_per_step_median": statistics.median(per_step),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "head_dim": d,
                   "context": w.context, "layers": len(layers), "page_size": P, "hash_bits": w.hash_bits,
                   "keep_pages": Nmax, "top_k": Kmax, "kv_dtype": "bf16",
                   "parallelism": f"replicas x{world}" if world > 1 else "single",
                   "l2": "not flushed: the KV cache (all layers) is far larger than L2 and each layer's bytes "
                         "are evicted by the other layers before reuse",
                   "bytes_per_step": step_total},
        "e2e": {"value": whole_job_throughput(B * args.steps, world, e2e_secs), "unit": "tokens/s",
                "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size()},
        "gpu_launches": len(layers) * args.steps,
        "roofline": roofline,
        "clocks": clocks,
        "build": build,
        "achieved_gbs": step_total / t_step / 1e9,
    }
    del ws
    # ---- the dense kernel at the same context, and the other workloads ----
    flush = torch.zeros(l2_flush_elems(dev), dtype=torch.float32, device=dev)
    if not args.no_dense:
        m = measure_workload(w, layers, dev, args, world, None, True)
        result["dense"] = dict(m["dense"], sparse_over_dense=m["sparse_over_dense"])
    per_config = {}
    if not args.no_extra and w.name == "llama_32l_128k" and args.layers is None:
        w3b = WORKLOADS["llama_32l_128k_keep8"]
        per_config[w3b.name] = measure_workload(w3b, with_budgets(w3b, layers, dev), dev, args, world, None,
                                                not args.no_dense)
    del layers, q_all, out_all
    torch.cuda.empty_cache()
    if not args.no_extra and args.layers is None:
        for name in ("tiny_4k", "llama_layer_32k", "paged_b16_ragged", "qwen_gqa7_128k"):
            if name == w.name:
                continue
            wx = WORKLOADS[name]
            lx, _ = build_layers(wx, dev)
            torch.cuda.synchronize()
            per_config[name] = measure_workload(wx, lx, dev, args, world, flush, not args.no_dense)
            del lx
            torch.cuda.empty_cache()
    if per_config:
        result["per_config"] = per_config
    return result, w


def l2_flush_elems(dev) -> int:
    import torch
    props = torch.cuda.get_device_properties(dev)
    return 2 * int(getattr(props, "L2_cache_size", 128 << 20)) // 4


def build_report(w, layers, build_events, clocks, sms, pk):
    """The cache build (rotation, page metadata and key codes of every valid
    row; not part of the timed step), timed with CUDA events around each
    layer's hhr_build_cache call during setup.  The median over layers after
    the first (which pays one-time costs) is reported against its two
    ceilings: HBM (the bytes the build must move; the binding one) and the
    tensor cores (the projections K R^T and K W^T run as tcgen05 MMAs; the
    kernel executes R as three bf16 terms, so it issues 2 d (3 d + nb) flops
    per row for the method's 2 d (d + nb))."""
    try:
        ms = [e0.elapsed_time(e1) for e0, e1 in build_events]
        t = statistics.median(ms[1:] if len(ms) > 1 else ms) / 1e3
        d, nb, P = w.head_dim, w.hash_bits, w.page_size
        rows = sum(w.num_kv_heads * Lb for Lb in layers[0]["lens"])
        pages = sum(w.num_kv_heads * (-(-Lb // P)) for Lb in layers[0]["lens"])
        # K read, K' written, codes written, page min/max written, R and W read (V is aliased)
        nbytes = rows * (2 * d * 2 + nb // 8) + pages * 2 * d * 2 + w.num_kv_heads * (d * d * 4 + nb * d * 2)
        flops = 2 * rows * d * (d + nb)
        issued = 2 * rows * d * (3 * d + nb)
        gbs = nbytes / t / 1e9
        return {"kernel": "build_cache_kernel (one launch per layer; tcgen05 MMAs, accumulators in TMEM)",
                "ms_per_layer": t * 1e3, "rows_per_layer": rows, "bound": "hbm", "achieved": gbs,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                "peak_source": pk.get("source", "measured"),
                "algorithmic_bytes_per_layer": nbytes,
                "tensor": {"algorithmic_tflops": flops / t / 1e12, "issued_tflops": issued / t / 1e12,
                           "peak": pk["bf16_tflops"], "frac": flops / t / 1e12 / pk["bf16_tflops"],
                           "flops_per_layer": flops, "issued_flops_per_layer": issued}}
    except Exception as e:  # reporting only: never fails the bench
        return {"error": repr(e)}


def run_reference(args, rank, world):
    """fp64 CPU oracle, rank 0 only: each step decodes one (layer 0, KV head) unit."""
    from threadpoolctl import threadpool_limits
    from hash_sparse_attention_b200.synth import WORKLOADS
    w = WORKLOADS[args.workload]
    units = oracle_units(w, min(2, w.num_kv_heads))
    heads_per_token = w.layers * w.num_kv_heads * w.batch
    with threadpool_limits(1):
        for i in range(max(3, args.warmup)):
            oracle_decode_unit(units[i % len(units)])
        t0 = time.perf_counter()
        for i in range(args.steps):
            oracle_decode_unit(units[i % len(units)])
        el = time.perf_counter() - t0
    value = (args.steps / heads_per_token) / el
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "batch": w.batch, "context": w.context, "layers": w.layers,
                   "note": "each step is one (layer, KV head) unit of the oracle; value scales by the "
                           f"{heads_per_token} units of one token"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} timed (layer 0, KV head) decode units, one thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, 1)))
        return 0
    from hash_sparse_attention_b200.synth import WORKLOADS, scaled
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the host leg first, before the GPU is touched (its processes are spawned)
        cpu = cpu_baseline(WORKLOADS[args.workload], args.cpu_seconds, args.cpu_workers)
    import torch
    rank, world = dist_init("nccl" if torch.cuda.is_available() else "gloo")
    result, w = run_hhr(args, rank, world)
    if cpu is not None:
        result["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
