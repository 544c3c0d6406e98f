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
