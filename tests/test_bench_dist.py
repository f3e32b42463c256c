"""Host logic of bench.py on CPU: the multi-rank plumbing (world size 2, gloo)
and the algorithmic byte accounting of a step."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = bench.dist_env()
    dist = bench.dist_init(w, "gloo")
    # each rank a replica of the workload with its own seed (weak scaling)
    spec = bench.rank_spec(W.small("opt13b"), r)
    sc = W.scenario(spec)
    t_ms = 1.0 + r                     # per-rank step time
    units = float(sc.context_lens.sum())
    bench.barrier(w)
    tmax = bench.reduce_max(t_ms, w)
    usum = bench.reduce_sum(units, w)
    q.put((r, spec.seed, tmax, usum, units))
    dist.destroy_process_group()


def test_two_rank_replicas_reduce_max_time_and_sum_units():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = {r[1] for r in res}
    assert len(seeds) == world                 # replicas draw different batches
    for r in res:
        assert r[2] == 2.0                     # max over ranks of 1.0, 2.0
        assert r[3] == pytest.approx(res[0][4] + res[1][4])


def test_single_rank_helpers_are_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.reduce_sum(2.0, 1) == 2.0
    assert bench.rank_spec(W.TINY, 0) is W.TINY


def test_step_bytes_unique_and_logical():
    spec = W.Spec("t", "bf16", 8, 2, 128, 16, "independent", 3, seed=1)
    # two sequences share their first block (id 5); the third is separate
    tables = np.array([[5, 6], [5, 7], [9, -1]], dtype=np.int32)
    lens = np.array([20, 18, 16], dtype=np.int32)
    unique, logical, other = bench.step_bytes(spec, tables, lens)
    row = 2 * 2 * 128 * 2                      # K and V, 2 kv heads, D 128, bf16
    assert logical == (20 + 18 + 16) * row
    assert unique == (16 + 4 + 2 + 16) * row   # block 5 once, 6: 4 tokens, 7: 2, 9: 16
    assert other == 2 * 3 * 8 * 128 * 2 + (2 + 2 + 1) * 4 + 3 * 4


def test_profile_digest_gates_traffic(tmp_path, monkeypatch):
    import json
    d = bench.source_digest(bench.KERNEL_SOURCES["decode_partition_tc_kernel"])
    prof = tmp_path / "profiles"
    prof.mkdir()
    k = "decode_partition_tc_kernel"
    caps = [dict(workload="x", kernel=k, partition_size=512, source_digest=d,
                 dram_bytes_per_launch=123, how="full launch"),
            dict(workload="y", kernel=k, partition_size=512, source_digest="0000",
                 dram_bytes_per_launch=123)]
    (prof / "dram_traffic.json").write_text(json.dumps({"captures": caps}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digest is computed from the sources under ROOT; point it back at the repo
    monkeypatch.setattr(bench, "source_digest", lambda files=None: d)
    assert bench.profiled_traffic("x", k, 512) == (123.0, "full launch")
    assert bench.profiled_traffic("x", k, 4096)[0] is None     # another launch configuration
    assert bench.profiled_traffic("x", "decode_partition_kernel", 512)[0] is None
    assert bench.profiled_traffic("y", k, 512)[0] is None      # kernel changed since
    assert bench.profiled_traffic("z", k, 512)[0] is None


def test_record_traffic_sums_one_call_and_replaces_its_entry(tmp_path, monkeypatch):
    import json
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.json").write_text(json.dumps({"captures": [
        dict(workload="w", kernel="decode_grouped", partition_size=512, source_digest="old",
             dram_bytes_per_launch=1),
        dict(workload="other", kernel="decode_grouped", partition_size=512,
             source_digest="keep", dram_bytes_per_launch=7)]}))
    csv_path = tmp_path / "cap.csv"
    hdr = '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
    rows = ['"0","span","dram__bytes_read.sum","byte","1,000"', '"0","span","dram__bytes_write.sum","byte","24"',
            '"0","span","gpu__time_duration.sum","nsecond","5"',
            '"1","rest","dram__bytes_read.sum","byte","2000"', '"1","rest","dram__bytes_write.sum","byte","6"']
    csv_path.write_text("==PROF== Connected\n" + hdr + "\n".join(rows) + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda files=None: "new")
    e = bench.record_traffic(str(csv_path), "w", "decode_grouped", 512)
    assert e["dram_bytes_per_launch"] == 1000 + 24 + 2000 + 6 and e["source_digest"] == "new"
    caps = json.loads((prof / "dram_traffic.json").read_text())["captures"]
    assert sorted(c["workload"] for c in caps) == ["other", "w"]
    assert bench.profiled_traffic("w", "decode_grouped", 512)[0] == 3030.0
    # the raw page of a report: one row per launch after a row of units
    csv_path.write_text('"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum"\n'
                        '"","","byte","byte"\n"0","k","433997568","4872192"\n')
    e = bench.record_traffic(str(csv_path), "w", "decode_grouped", 1024)
    assert e["dram_bytes_per_launch"] == 433997568 + 4872192
    # values not in bytes are refused rather than mis-scaled
    csv_path.write_text(hdr + '"0","span","dram__bytes_read.sum","Mbyte","1.5"\n')
    with pytest.raises(SystemExit):
        bench.record_traffic(str(csv_path), "w", "decode_grouped", 512)


def test_partition_kernel_choice():
    assert bench.partition_kernel(W.GQA70B, 512) == "decode_partition_tc_kernel"
    assert bench.partition_kernel(W.LONG_PREFIX, 512) == "decode_partition_tc_kernel"
    assert bench.partition_kernel(W.OPT13B, 512) == "decode_partition_kernel"
    assert bench.partition_kernel(W.GQA70B, 96) == "decode_partition_kernel"
    assert bench.partition_kernel(W.TINY, 512) == "decode_partition_kernel"
    assert bench.partition_kernel(W.fp8(W.GQA70B), 2048) == "decode_partition_tc8_kernel"
    assert bench.partition_kernel(W.fp8(W.OPT13B), 512) == "decode_partition_kernel"


def test_fp8_workloads_count_one_byte_per_element():
    spec = W.fp8(W.Spec("t", "bf16", 8, 2, 128, 16, "independent", 3, seed=1))
    tables = np.array([[5, 6], [5, 7], [9, -1]], dtype=np.int32)
    lens = np.array([20, 18, 16], dtype=np.int32)
    unique, logical, other = bench.step_bytes(spec, tables, lens)
    row = 2 * 2 * 128 * 1                      # K and V, 2 kv heads, D 128, one byte each
    assert logical == (20 + 18 + 16) * row and unique == (16 + 4 + 2 + 16) * row
    assert other == 2 * 3 * 8 * 128 * 2 + (2 + 2 + 1) * 4 + 3 * 4   # q / out stay bf16
    s = bench.workload_spec("opt13b_fp8")
    assert s.fp8 and s.dtype == "f16" and s.num_seqs == W.OPT13B.num_seqs
    assert "E4M3" in bench.workload_text("gqa70b_fp8")
