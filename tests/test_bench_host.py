"""Host-side logic of bench.py that the GPU runs rely on (no GPU needed)."""
import hashlib
import os
import shutil

import pytest

import bench
from h2o_kv_cache_step_b200 import synth

WL = synth.WORKLOADS["qwen3-4b-c2048-t1024-n64k"]


def test_schedule_fills_then_stays_full():
    sched = bench.sequence_schedule(WL)
    assert len(sched) == WL.n_chunks
    assert sched[:3] == [(0, WL.T), (WL.T, WL.T), (2 * WL.T, WL.T)]
    assert all(n == WL.C for n, _ in sched[2:])


def test_kernel_work_counts_visible_pairs():
    # a steady step of the bench layer: 32 heads x (1024 x 2048 + 1024 x 1025 / 2) pairs
    pairs = bench.step_pairs(WL, WL.C, WL.T)
    assert pairs == 32 * (1024 * 2048 + 1024 * 1025 // 2)
    assert bench.kernel_work(WL, "sdpa_tc_kernel", WL.C, WL.T) == (4.0 * 128 * pairs, "flop", "tensor")
    assert bench.kernel_work(WL, "wsum_tc_kernel", WL.C, WL.T)[0] == 2.0 * 128 * pairs


def test_profiled_traffic_needs_matching_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "h2o_kv_cache_step_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("tc.cu", "tc_ptx.cuh", "common.cuh"):
        shutil.copy(os.path.join(bench.ROOT, "h2o_kv_cache_step_b200", "csrc", f), csrc / f)
    # a record written for the sources as they are now (the committed record
    # may predate the current kernel; what is tested here is the rule)
    h = hashlib.sha256()
    for fn in sorted(("tc.cu", "tc_ptx.cuh", "common.cuh")):
        h.update(fn.encode())
        h.update(open(csrc / fn, "rb").read())
    rec = ["sdpa_tc_kernel", WL.name, str(WL.C), str(WL.T), "21048320", "256", "tc.cu,tc_ptx.cuh,common.cuh",
           h.hexdigest()[:16]]
    (root / "profiles" / "dram_traffic.txt").write_text("# kernel workload n T read write sources sha\n" +
                                                        " ".join(rec) + "\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    sched = [(WL.C, WL.T)]  # the captured steady-state step itself: no scaling
    assert bench.profiled_traffic(WL, "sdpa_tc_kernel", sched) == pytest.approx(float(rec[4]) + float(rec[5]))
    # launches that read less (a filling cache) are scaled by their compulsory bytes
    small = bench.profiled_traffic(WL, "sdpa_tc_kernel", [(0, WL.T)])
    assert small < float(rec[4])
    # any change to the kernel's sources voids the record
    with open(csrc / "tc.cu", "a") as fh:
        fh.write("\n// changed\n")
    assert bench.profiled_traffic(WL, "sdpa_tc_kernel", sched) is None
    assert bench.profiled_traffic(WL, "scatter_kernel", sched) is None  # no record


def test_job_throughput_is_all_ranks_over_the_slowest():
    assert bench.job_throughput(65536, 4, 8.0) == pytest.approx(65536 * 4 / 0.008)


def test_sdpa_pieces_follow_the_split_rule():
    """The SDPA splits a unit's cache blocks only when its units fill less than
    half of the SMs; every piece keeps at least one cache block (the last one
    also takes the chunk's blocks), and no more CTAs than SMs are launched."""
    big = synth.WORKLOADS["qwen3-4b-c16384-t512-n128k"]
    assert bench.sdpa_pieces(WL, WL.C, WL.T) == 1                 # 128 units: no split
    assert bench.sdpa_pieces(big, big.C, big.T) == 2              # 64 units on 148 SMs
    assert bench.sdpa_pieces(big, 3 * 128, big.T) == 1            # fewer than 4 cache blocks
    for wl in synth.WORKLOADS.values():
        for n in range(0, wl.C + 1, 97):
            ns = bench.sdpa_pieces(wl, n, wl.T)
            nbc = -(-n // 128)
            units = -(-wl.T // 128) * wl.B * wl.Hkv * ((wl.G + 1) // 2)
            assert 1 <= ns <= 8
            if ns > 1:
                assert units * ns <= 148
                cb = -(-nbc // ns)
                assert (ns - 1) * cb < nbc                       # the last piece has a cache block too


def test_kernel_work_of_the_other_kernels():
    e = 2  # bf16
    groups = WL.B * WL.Hkv
    # the split SDPA's merge reads every piece's fp32 partial row and writes bf16 rows
    big = synth.WORKLOADS["qwen3-4b-c16384-t512-n128k"]
    rows = big.B * big.Hq * big.T
    assert bench.kernel_work(big, "sdpa_combine_kernel", big.C, big.T) == (
        float(rows * 2 * (big.d + 2) * 4 + rows * big.d * e), "byte", "hbm")
    # decode: the split kernel reads the cache's K and V once (plus the chunk)
    b, unit, bound = bench.kernel_work(WL, "decode_split_kernel", WL.C, 1)
    assert (unit, bound) == ("byte", "hbm")
    assert b == groups * (2 * WL.C * WL.d * e + (WL.G + 2) * WL.d * e)
    for name in ("decode_combine_kernel", "decode_wsum_kernel"):
        assert bench.kernel_work(WL, name, WL.C, 1)[1:] == ("byte", "hbm")
        assert bench.kernel_work(WL, name, WL.C, 1)[0] > 0
