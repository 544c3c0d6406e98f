"""Host-side logic of bench.py (no GPU): byte accounting and rank aggregation."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_algorithmic_bytes_of_the_128k_layer():
    # per (layer, KV head) at 128K: metadata 8192 pages x 512 B, codes of the
    # 8192 candidate rows x 16 B, 8192 kept K'/V rows x 512 B, q and out of
    # 4 query heads (256 B + 512 B each), R_h (64 KiB) and W_h (32 KiB)
    hb = bench.hhr_bytes_per_head(131072, 16, 512, 13108, 4, 128)
    assert hb["meta"] == 4_194_304
    assert hb["codes"] == 131_072
    assert hb["gather"] == 4_194_304
    assert hb["qo"] == 3_072
    assert hb["rw"] == 98_304
    assert sum(hb[k] for k in ("meta", "codes", "gather", "qo", "rw")) == 8_621_056
    assert hb["keff"] == 8192  # k clamped to the candidates
    # keep 1/8 of pages: 16384 candidates, k = 13108 rows gathered
    hb8 = bench.hhr_bytes_per_head(131072, 16, 1024, 13108, 4, 128)
    assert hb8["gather"] == 13108 * 512 and hb8["codes"] == 16384 * 16
    # ragged tail: every page kept
    hr = bench.hhr_bytes_per_head(17, 16, 10, 100, 4, 128)
    assert hr["cand"] == 17 and hr["keff"] == 17 and hr["meta"] == 2 * 512


def test_dense_bytes():
    assert bench.dense_bytes_per_head(131072, 4) == 131072 * 512 + 3072 + 65536


def test_whole_job_throughput():
    assert bench.whole_job_throughput(100, 4, 2.0) == 200.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w = bench.dist_init("gloo")
    bench.barrier(w)
    m = bench.max_over_ranks(1.0 + r, w)
    q.put((r, m))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2.0), (1, 2.0)]


def test_build_report_counts_rows_bytes_and_flops():
    """The cache-build line: median over layers after the first, the HBM
    ceiling from the bytes the build must move and the tensor-core ceiling
    from the projection flops (no GPU needed)."""
    import bench
    from hash_sparse_attention_b200.synth import WORKLOADS

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    w = WORKLOADS["llama_32l_128k"]
    ev = [(Ev(0.0), Ev(9.0)), (Ev(0.0), Ev(4.0)), (Ev(0.0), Ev(2.0)), (Ev(0.0), Ev(3.0))]
    r = bench.build_report(w, [{"lens": [131072]}], ev, {"sm_max_mhz": 2000.0}, 100,
                           {"hbm_gbs": 1000.0, "bf16_tflops": 500.0, "source": "measured"})
    assert r["ms_per_layer"] == 3.0  # median of 4, 2, 3 (the first layer is left out)
    rows = 8 * 131072
    assert r["rows_per_layer"] == rows
    pages = 8 * 131072 // 16
    nbytes = rows * (512 + 16) + pages * 512 + 8 * (128 * 128 * 4 + 128 * 128 * 2)
    assert r["algorithmic_bytes_per_layer"] == nbytes
    assert r["bound"] == "hbm" and r["peak"] == 1000.0
    assert abs(r["achieved"] - nbytes / 3e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 1000.0) < 1e-12
    t = r["tensor"]
    assert t["flops_per_layer"] == 2 * rows * 128 * (128 + 128)
    assert t["issued_flops_per_layer"] == 2 * rows * 128 * (3 * 128 + 128)
    assert abs(t["frac"] - t["flops_per_layer"] / 3e-3 / 1e12 / 500.0) < 1e-12


def test_profiled_traffic_only_for_matching_sources_and_workload(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed profile summary only when it
    was taken on the current kernel sources and the same workload."""
    import bench

    prof = tmp_path / "profiles"
    prof.mkdir()
    f = prof / "hhr_sparse_kernel_llama_32l_128k.md"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("llama_32l_128k") is None  # no summary
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc123")
    f.write_text("- workload: `llama_32l_128k`\n- dram_bytes_per_launch: `1234`\n- sources_sha256: `abc123`\n")
    assert bench.profiled_traffic("llama_32l_128k") == 1234.0
    assert bench.profiled_traffic("qwen_gqa7_128k") is None  # another workload (no summary of its own)
    f.write_text("- workload: `llama_32l_128k`\n- dram_bytes_per_launch: `1234`\n- sources_sha256: `def456`\n")
    assert bench.profiled_traffic("llama_32l_128k") is None  # sources changed since the capture
    f.write_text("- workload: `llama_32l_128k`\n- sources_sha256: `abc123`\n")
    assert bench.profiled_traffic("llama_32l_128k") is None  # no figure


def test_kernel_source_hash_tracks_the_sources():
    import bench
    h1 = bench.kernel_source_hash()
    assert len(h1) == 64 and h1 == bench.kernel_source_hash()


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the fp64 oracle on the host (no GPU)
    and prints one JSON line with the contract's keys."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "llama_32l_128k"


def test_cpu_baseline_single_and_all_cores():
    """The oracle leg: one thread, then single-threaded spawned processes over
    memory-mapped unit caches; both report tokens/s, the core count and the CPU
    model."""
    from hash_sparse_attention_b200.synth import WORKLOADS, scaled
    w = scaled(WORKLOADS["tiny_4k"], context=1024)
    out = bench.cpu_baseline(w, 0.5, workers=2)
    assert out["kind"] == "oracle" and out["cores"] == 1 and out["value"] > 0
    assert out["cpu_model"] and out["host_cores"] >= 1
    ac = out["all_cores"]
    assert ac["cores"] == 2 and ac["value"] > 0 and ac["kind"] == "oracle"

