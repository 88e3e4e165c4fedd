"""The multi-rank path of the benchmark, on CPU with two gloo ranks.

The chunked H2O step shards by sequence: every rank prefills its own
sequence and no collective touches the data path; the ranks only agree on
the timing (the slowest rank's time) and the job's throughput is all ranks'
tokens over that time. These tests run that host logic as two processes
without a GPU, with the oracle standing in for the device step.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from h2o_kv_cache_step_b200 import synth

WORLD = 2
CHUNKS = 2  # chunks of the tiny workload each rank prefills


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _prefill_oracle(wl, chunks: int):
    """Outputs and final H2O state of the first `chunks` chunk steps."""
    from oracle import oracle
    st = oracle.State.empty(wl.B, wl.Hkv, wl.C, wl.d)
    outs = []
    for c in range(chunks):
        q, k, v = (x.astype(np.float64) for x in synth.chunk(wl, c))
        outs.append(oracle.step(st, q, k, v).out)  # advances st in place
    return np.stack(outs), st


def _worker(rank: int, port: int, result_dir: str):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        wl = bench.rank_workload(synth.WORKLOADS["tiny-fp32"], rank, WORLD)
        out, st = _prefill_oracle(wl, CHUNKS)
        # a per-rank "device time": the slowest must win on every rank
        ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(ms)
        value = bench.job_throughput(wl.B * wl.T * CHUNKS, WORLD, ms_max)
        np.savez(os.path.join(result_dir, f"rank{rank}.npz"), out=out, scores=st.phi, pos=st.pos,
                 seed=wl.seed, ms_max=ms_max, value=value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def rank_results(tmp_path_factory, oracle_lib):
    d = str(tmp_path_factory.mktemp("ranks"))
    mp.start_processes(_worker, args=(_free_port(), d), nprocs=WORLD, join=True, start_method="spawn")
    return [dict(np.load(os.path.join(d, f"rank{r}.npz"))) for r in range(WORLD)]


def test_ranks_run_distinct_sequences(rank_results):
    seeds = [int(r["seed"]) for r in rank_results]
    assert len(set(seeds)) == WORLD
    assert not np.allclose(rank_results[0]["out"], rank_results[1]["out"])


def test_each_rank_matches_a_single_process_run(rank_results):
    # sharding by sequence couples nothing: rank r's result is exactly what a
    # single process computes for rank r's sequence
    for r, res in enumerate(rank_results):
        wl = bench.rank_workload(synth.WORKLOADS["tiny-fp32"], r, WORLD)
        out, st = _prefill_oracle(wl, CHUNKS)
        np.testing.assert_array_equal(res["out"], out)
        np.testing.assert_array_equal(res["scores"], st.phi)
        np.testing.assert_array_equal(res["pos"], st.pos)


def test_timing_is_the_max_over_ranks(rank_results):
    for res in rank_results:
        assert float(res["ms_max"]) == 10.0 + 5.0 * (WORLD - 1)


def test_throughput_counts_all_ranks(rank_results):
    wl = synth.WORKLOADS["tiny-fp32"]
    want = wl.B * wl.T * CHUNKS * WORLD / ((10.0 + 5.0 * (WORLD - 1)) / 1e3)
    for res in rank_results:
        assert float(res["value"]) == pytest.approx(want)


def test_single_rank_is_the_identity():
    wl = synth.WORKLOADS["tiny-fp32"]
    assert bench.rank_workload(wl, 0, 1) is wl
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1000, 1, 500.0) == 2000.0
