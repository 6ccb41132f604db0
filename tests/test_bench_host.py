"""Host-side logic of bench.py that needs no GPU: the multi-rank reductions
(world size 2 over gloo), per-rank workloads, profiling trims and the
traffic record's staleness check."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world) and dist.get_backend() == "gloo"
    mx = bench.max_over_ranks(float(10 + rank), w)
    sm = bench.sum_over_ranks(float(1 + rank), w)
    wl = bench.rank_workload(2, r)
    bench.barrier(w)
    out[rank] = (mx, sm, wl.seed, wl.batch)
    dist.destroy_process_group()


def test_two_rank_reductions_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0          # max over ranks
    assert out[0][1] == out[1][1] == 3.0           # sum over ranks
    assert out[0][2] != out[1][2]                  # each rank serves its own sequences
    assert out[0][3] == out[1][3] == 4             # same per-rank batch: weak scaling


def test_trim_keeps_shared_layer():
    import gen
    w = gen.config(3)

    class A:
        compose_layers = 1
        cross_layers = 2
    comp, cross = bench.trim(w, A)
    assert comp == [w.shared_layer] and cross == w.cross_layers[:2]

    class Z:
        compose_layers = 0
        cross_layers = 0
    comp, cross = bench.trim(w, Z)
    assert comp == w.composed_layers and cross == w.cross_layers


def test_traffic_record_goes_stale(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    h = bench.source_hash(bench.KERNEL_SOURCES["decode_split_kernel"])
    (prof / "traffic.json").write_text(json.dumps({"decode_split_kernel": {
        "w": {"source_hash": h, "bytes_per_launch": 123},
        "x": {"source_hash": "0" * 16, "bytes_per_launch": 456}}}))
    for k, paths in bench.KERNEL_SOURCES.items():
        for p in paths:
            os.makedirs(tmp_path / os.path.dirname(p), exist_ok=True)
            with open(os.path.join(ROOT, p), "rb") as src, open(tmp_path / p, "wb") as dst:
                dst.write(src.read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("decode_split_kernel", "w") == 123
    assert bench.ncu_traffic("decode_split_kernel", "x") is None
    assert bench.ncu_traffic("compose_append_kernel", "w") is None


def test_peak_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6441.9}))
    assert bench.hbm_peak() == (6441.9, "measured")


def test_causal_pair_count():
    # whole-prompt causal prefill: a sequence of n rows scores n (n + 1) / 2 (query, key) pairs
    assert bench.causal_pairs([]) == 0
    assert bench.causal_pairs([1]) == 1
    assert bench.causal_pairs([3, 1, 0]) == 6 + 1
    n = 8191
    assert bench.causal_pairs([n] * 32) == 32 * n * (n + 1) // 2
    # brute-force count of u <= t for a small case
    assert bench.causal_pairs([7, 5]) == sum(1 for n in (7, 5) for t in range(n) for u in range(n) if u <= t)


def test_tensor_peak_reads_measured_file(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1000.0, "bf16_tflops_sustained": 900.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.tensor_peak() == (1000.0, 900.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").unlink()
    burst, sustained, kind = bench.tensor_peak()
    assert kind == "fallback" and burst > sustained > 0
