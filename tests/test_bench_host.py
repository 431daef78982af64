"""Host-side pieces of bench.py: byte accounting, replica aggregation over ranks, the reference arm."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench
import oracle
from synth import configs

from _dist_helpers import free_port

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_llama70b():
    g = configs.llama70b()
    B = bench.alg_bytes(g, oracle.layout(g.world, g.shapes))
    assert B["rs"] == 13_690_470_400 + 3_422_617_600 == 17_113_088_000
    assert B["ag"] == 2 * 855_654_400 + 2 * 855_654_400
    assert B["stage"] == 2 * 8 * 855_654_400 * 2


def test_algorithmic_bytes_count_pads_on_the_write_side():
    g = configs.wan14b()
    L = oracle.layout(g.world, g.shapes)
    B = bench.alg_bytes(g, L)
    N = sum(g.numel(i) for i in range(g.n_params))
    assert B["N"] == N and B["Npad"] == g.world * L.Ns > N      # modulation rows 6..15 are pad
    assert B["rs"] == 2 * g.world * N + 4 * g.world * L.Ns


def _agg_worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank], "cpu")
        with open(os.path.join(out_dir, f"agg_{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_replica_aggregation_takes_the_slowest_rank(tmp_path):
    mp.spawn(_agg_worker, args=(2, free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert json.load(open(tmp_path / f"agg_{r}.json")) == [2.0, 5.0, 0.25]
    # whole-job throughput: both replicas' bytes over the slowest rank's step time
    assert bench.replica_throughput(2, 10**9, 2.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks([3.0], "cpu") == [3.0]          # no process group: identity


def _run_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "2", "--warmup", "1", "--gpus", "2"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank0_prints_one_line_other_ranks_exit_quietly():
    r1 = _run_reference(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0)
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["higher_is_better"] is True


def test_jsonl_rows_flatten_a_bench_line():
    """One row per timed entry, with (op, mode, ctas), bytes, time and the bit check."""
    res = {
        "kernels": {
            "rs_reduce_kernel": {"ms": 2.5, "GB/s": 6900.0, "frac_of_peak": 1.05, "alg_bytes": 17,
                                 "ctas": 296, "kernel": "rs_v32", "traffic": 17},
            "ag_place_kernel": {"ms": 0.5, "GB/s": 6600.0, "frac_of_peak": 1.0, "alg_bytes": 3,
                                "ctas": 592, "traffic": None}},
        "variants": {
            "ag_place_ce": {"ms": 0.7, "GB/s": 5000.0, "frac_of_peak": 0.76, "alg_bytes": 3,
                            "kernel_launches": 0, "kernel": "copy engines", "ctas": 0,
                            "same_bits_as_plain": True},
            "slot_reuse_pipelined_seg4": {"ms": 6.8, "GB/s": 6500.0, "frac_of_peak": 0.99,
                                          "alg_bytes": 44, "kernel_launches": 4, "kernel": "slot_rs_v32",
                                          "ctas": 296, "same_bits_as_plain": False}},
        "cpu_baseline": {"value": 1.9, "cores": 1},
        "clocks": {"sm_mhz": 1965},
    }
    rows = bench.jsonl_rows(res, "llama70b", 8)
    assert [r["entry"] for r in rows] == ["rs_reduce_kernel", "ag_place_kernel", "ag_place_ce",
                                          "slot_reuse_pipelined_seg4"]
    by = {r["entry"]: r for r in rows}
    assert by["rs_reduce_kernel"]["op"] == "rs_reduce" and by["rs_reduce_kernel"]["ctas"] == 296
    assert by["rs_reduce_kernel"]["dram_bytes_per_launch"] == 17
    assert by["ag_place_ce"]["mode"] == "copy engines" and by["ag_place_ce"]["same_bits_as_plain"] is True
    assert by["slot_reuse_pipelined_seg4"]["mode"] == "pipelined, 4 segments"
    assert by["slot_reuse_pipelined_seg4"]["same_bits_as_plain"] is False
    assert all(r["config"] == "llama70b" and r["world"] == 8 and r["oracle_GB/s"] == 1.9 for r in rows)
    assert all(json.loads(json.dumps(r)) == r for r in rows)


def test_rs_sm_time_counts_sms_held_times_duration():
    import bench
    v = {"stock_torch_pack_reduce": {"ms": 30.0}, "slot_reduce": {"ms": 2.5, "ctas": 296}}
    r = bench.rs_sm_time(2.4, 296, v, 148)
    assert r["stock_pack_reduce"] == 148 * 30.0
    assert r["tide_rs_reduce"] == round(148 * 2.4, 2)          # 296 CTAs hold the 148 SMs
    assert r["tide_slot_reuse_ce"] == 148 * 2.5                 # the staging holds none
    assert r["stock_over_tide"] == round(30.0 / 2.4, 2)
    capped = bench.rs_sm_time(40.0, 4, v, 148)                 # 4 CTAs hold 4 SMs
    assert capped["tide_rs_reduce"] == 160.0


def test_traffic_record_is_current_and_close_to_the_algorithmic_bytes():
    """profiles/ncu_traffic.txt holds one small-case capture per kernel, keyed by a digest of
    its sources: every entry matches the sources as they are now (so the bench reports its
    traffic), and the scaled traffic of a 70B launch is within 0.5 % of the algorithmic bytes
    (a kernel that re-read its inputs would show up here)."""
    import bench
    for kernel, sources in (("rs_v32", bench.RS_SOURCES), ("rs_tree_v32", bench.RS_SOURCES),
                            ("ag", bench.AG_SOURCES)):
        rd, wr = (13690208256, 3422552064) if kernel.startswith("rs") else (3422552064, 3422552064)
        traffic, note = bench.ncu_traffic(kernel, sources, rd, wr)
        assert traffic is not None, (kernel, note)
        assert abs(traffic / (rd + wr) - 1.0) < 0.005, (kernel, traffic)
