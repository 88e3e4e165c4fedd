"""GPU parity: the CUDA step through the C ABI against the fp64 oracle.

Small cases compare every element; full-size cases (the benchmark's
workloads and launch configuration) compare sampled rows, one whole group's
scores, and the selection of every group."""
import numpy as np
import pytest
import torch

from h2o_kv_cache_step_b200 import H2OCache, synth
from oracle import oracle
from parity_util import (TOL_LSE, TOL_OUT, TORCH_DTYPE, check_selection_replay, compare_scores,
                         gpu_step, lockstep_full, oracle_state_from_device, record_errors, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def run_sequence_lockstep(wl, n_chunks=None, cache=None):
    cache = cache or H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, TORCH_DTYPE[wl.dtype], max_T=wl.T)
    stats = []
    for c in range(n_chunks or wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        stats.append(lockstep_full(cache, q, k, v, wl.dtype, wl.C))
    return cache, stats


def test_tiny_fp32_workload_lockstep():
    """The tiny fp32 workload end to end (12 chunks, 4 filling, 8 evicting)."""
    wl = synth.WORKLOADS["tiny-fp32"]
    cache, stats = run_sequence_lockstep(wl)
    assert cache.counters() == (wl.N, wl.C)
    assert all(s["same_selection"] for s in stats)


@pytest.mark.parametrize("dtype,d,B,Hq,Hkv,C,T,chunks", [
    ("bf16", 128, 2, 8, 2, 384, 200, 4),     # ragged T and C, GQA 4
    ("bf16", 128, 1, 4, 4, 256, 128, 4),     # MHA, tile-aligned
    ("bf16", 64, 1, 8, 1, 300, 130, 4),      # d = 64, one KV head, G = 8
    ("bf16", 128, 1, 4, 2, 100, 300, 3),     # chunk longer than the cache
    ("fp32", 128, 1, 4, 2, 200, 96, 4),
    ("fp32", 64, 2, 2, 1, 130, 33, 6),
    ("bf16", 128, 1, 8, 2, 1500, 200, 9),    # few units, long cache: SDPA split into 2..6 pieces
    ("bf16", 64, 1, 8, 1, 1100, 130, 10),    # the same at d = 64, ragged last piece
])
def test_small_shapes_lockstep(dtype, d, B, Hq, Hkv, C, T, chunks):
    wl = synth.Workload("small", dtype, B=B, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * chunks,
                        seed=11, recipe="heavy", hh_frac=0.05)
    run_sequence_lockstep(wl)


@pytest.mark.parametrize("T", [1, 2, 17])
def test_short_chunks_lockstep(T):
    """T = 1 is classic per-token H2O; short chunks stress the causal tail."""
    wl = synth.Workload("short", "bf16", B=1, Hq=8, Hkv=2, d=128, C=40, T=T, N=T * 6, seed=3,
                        recipe="iid")
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, torch.bfloat16, max_T=64)
    # start from a full cache with scattered positions so eviction happens at once
    K, V, S, pos = synth.random_state(wl, n=wl.C, P=500, seed=T)
    cache.set_state(to_dev(K, "bf16"), to_dev(V, "bf16"), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=500, n=wl.C)
    for c in range(wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        lockstep_full(cache, q, k, v, "bf16", wl.C)


@pytest.mark.parametrize("dtype,d,B,Hq,Hkv,C,T,chunks", [
    ("fp32", 64, 1, 4, 2, 256, 64, 8),       # the tiny workload's shape, 4 evicting steps
    ("bf16", 128, 2, 8, 2, 384, 200, 4),     # ragged T and C, GQA 4
    ("bf16", 64, 1, 8, 1, 300, 130, 4),      # d = 64, one KV head, G = 8
    ("bf16", 128, 1, 4, 2, 100, 300, 3),     # chunk longer than the cache
])
def test_normalized_policy_lockstep(dtype, d, B, Hq, Hkv, C, T, chunks):
    """Eviction ranked by score / age (H2O_POLICY_NORMALIZED): outputs and
    scores against the oracle under the same policy, selection bit-exact on
    replay with the device's fp32 key."""
    from h2o_kv_cache_step_b200._lib import H2O_POLICY_NORMALIZED
    wl = synth.Workload("norm", dtype, B=B, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * chunks,
                        seed=13, recipe="heavy", hh_frac=0.05)
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, TORCH_DTYPE[dtype], max_T=wl.T)
    cache.set_policy(H2O_POLICY_NORMALIZED)
    differs = False
    for c in range(wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        pre = oracle_state_from_device(cache)
        lockstep_full(cache, q, k, v, dtype, wl.C, policy=oracle.POLICY_NORMALIZED)
        # the policy matters: the sum policy would keep another set somewhere
        r_sum = oracle.step(pre.copy(), q, k, v, policy=oracle.POLICY_SUM)
        r_norm = oracle.step(pre.copy(), q, k, v, policy=oracle.POLICY_NORMALIZED)
        differs |= not np.array_equal(r_sum.cand_kept, r_norm.cand_kept)
    assert differs


@pytest.mark.parametrize("dtype,d,B,Hq,Hkv,C,T,chunks,full", [
    ("bf16", 128, 2, 8, 2, 256, 96, 5, False),   # fills, then evicts before attending (tensor cores)
    ("bf16", 128, 1, 8, 2, 200, 200, 3, False),  # T = C: the whole cache turns over every step
    ("fp32", 64, 1, 4, 2, 130, 33, 6, False),    # CUDA-core path
    ("bf16", 128, 1, 8, 2, 300, 4, 4, True),     # short chunks on a full cache: decode path
])
def test_insert_always_lockstep(dtype, d, B, Hq, Hkv, C, T, chunks, full):
    """H2O_POLICY_INSERT_ALWAYS against the oracle's insert-always step from
    the device's own state each step: outputs and LSE within tolerance, token
    slots and positions exact, scores within tolerance, the chunk's rows in
    their slots."""
    from h2o_kv_cache_step_b200._lib import H2O_POLICY_INSERT_ALWAYS
    wl = synth.Workload("insert", dtype, B=B, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * chunks, seed=17,
                        recipe="heavy", hh_frac=0.05)
    cache = H2OCache(B, Hq, Hkv, d, C, TORCH_DTYPE[dtype], max_T=T)
    cache.set_policy(H2O_POLICY_INSERT_ALWAYS)
    if full:
        K, V, S, pos = synth.random_state(wl, n=C, P=2000, seed=3)
        cache.set_state(to_dev(K, dtype), to_dev(V, dtype), torch.from_numpy(S).cuda(),
                        torch.from_numpy(pos).cuda(), P=2000, n=C)
    for c in range(chunks):
        q, k, v = synth.chunk(wl, c)
        pre = oracle_state_from_device(cache)
        st = pre.copy()
        out_ref, lse_ref, ts_ref = oracle.step_insert_always(st, q, k, v)
        g = gpu_step(cache, q, k, v, dtype)
        assert np.abs(g["out"] - out_ref).max() <= TOL_OUT[dtype]
        assert np.abs(g["lse"] - lse_ref).max() <= TOL_LSE[dtype]
        assert np.array_equal(g["token_slot"], ts_ref)
        assert np.array_equal(g["Pos"], st.pos.astype(np.int32))
        compare_scores(g["S"], st.phi, "insert-always scores")
        for b in range(B):
            for gg in range(Hkv):
                assert np.array_equal(g["K"][b, gg, ts_ref[b, gg]], np.asarray(k, np.float32)[b, gg])


def test_insert_always_rejects_chunks_longer_than_the_cache():
    from h2o_kv_cache_step_b200._lib import H2O_POLICY_INSERT_ALWAYS, H2OError
    cache = H2OCache(1, 2, 1, 64, 8, torch.float32, max_T=16)
    cache.set_policy(H2O_POLICY_INSERT_ALWAYS)
    x = torch.zeros((1, 2, 9, 64), device="cuda")
    with pytest.raises(H2OError):
        cache.step(x, x[:, :1].contiguous(), x[:, :1].contiguous())


def test_set_policy_rejects_unknown():
    from h2o_kv_cache_step_b200._lib import H2OError
    cache = H2OCache(1, 2, 1, 64, 8, torch.float32, max_T=4)
    with pytest.raises(H2OError):
        cache.set_policy(7)


@pytest.mark.parametrize("dtype,d,Hq,Hkv,C,T,policy", [
    ("bf16", 128, 8, 2, 300, 1, 0),    # one token per step: classic decode
    ("bf16", 128, 32, 8, 256, 4, 0),   # the bench layer's heads, G = 4
    ("bf16", 64, 8, 1, 200, 4, 0),     # G * T = 32 rows, the most the decode path takes
    ("fp32", 128, 2, 2, 100, 16, 0),   # T = 16, the longest decode chunk (MHA)
    ("fp32", 64, 4, 2, 130, 3, 0),
    ("bf16", 128, 8, 2, 300, 2, 1),    # normalized policy
    ("bf16", 128, 8, 2, 4096, 1, 0),   # a long cache: 65 slices per group
    ("fp32", 64, 4, 2, 2600, 2, 0),    # 42 slices, fp32
])
def test_decode_path_lockstep(dtype, d, Hq, Hkv, C, T, policy):
    """Chunks of T <= 16 tokens take the split-K decode kernels; lockstep
    against the oracle from a full cache with scattered positions, plus a
    cold start (empty cache, a single split)."""
    wl = synth.Workload("decode", dtype, B=2, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * 6, seed=21,
                        recipe="heavy", hh_frac=0.05)
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, TORCH_DTYPE[dtype], max_T=16)
    assert cache.kernel_plan(T)[0] == "decode_split_kernel"
    cache.set_policy(policy)
    for c in range(2):  # cold start
        q, k, v = synth.chunk(wl, c)
        lockstep_full(cache, q, k, v, dtype, wl.C, policy=policy)
    P0 = max(1000, 2 * wl.C)
    K, V, S, pos = synth.random_state(wl, n=wl.C, P=P0, seed=T)
    cache.set_state(to_dev(K, dtype), to_dev(V, dtype), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=P0, n=wl.C)
    for c in range(2, wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        lockstep_full(cache, q, k, v, dtype, wl.C, policy=policy)


def test_decode_path_limits():
    """Chunks with more than 32 query rows per KV group, or T > 16, take the
    chunk path."""
    cache = H2OCache(1, 8, 2, 128, 256, torch.bfloat16, max_T=64)
    assert cache.kernel_plan(8)[0] == "decode_split_kernel"      # 4 heads x 8 = 32 rows
    assert cache.kernel_plan(16)[0] == "sdpa_tc_kernel"          # 64 rows
    cache2 = H2OCache(1, 2, 2, 64, 64, torch.float32, max_T=64)
    assert cache2.kernel_plan(16)[0] == "decode_split_kernel"
    assert cache2.kernel_plan(17)[0] == "sdpa_simt_kernel"


@pytest.mark.slow
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_selection_fallback_for_large_candidate_sets(dtype):
    """Candidate sets whose 64-bit keys do not fit in shared memory (C + T =
    32,832 here) take the selection kernel's other form, which rebuilds each
    key from the candidate arrays on every radix pass. Two evicting steps
    from a full cache, lockstep against the oracle with the selection replayed
    bit-exactly."""
    C, T = 32768, 64
    m = C + T
    smem_limit = 220 * 1024  # the selection kernel's shared-memory budget
    assert m * 8 + m + 4 * C > smem_limit >= m + 4 * C  # keys do not fit; flags and free list do
    wl = synth.Workload("select-fallback", dtype, B=1, Hq=2, Hkv=1, d=64, C=C, T=T, N=2 * T, seed=23,
                        recipe="heavy", hh_frac=0.05)
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, C, TORCH_DTYPE[dtype], max_T=T)
    K, V, S, pos = synth.random_state(wl, n=C, P=100000, seed=5)
    cache.set_state(to_dev(K, dtype), to_dev(V, dtype), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=100000, n=C)
    for c in range(2):
        q, k, v = synth.chunk(wl, c)
        lockstep_full(cache, q, k, v, dtype, C)


def test_cache_of_one_slot():
    wl = synth.Workload("c1slot", "fp32", B=1, Hq=2, Hkv=1, d=64, C=1, T=5, N=20, seed=2)
    run_sequence_lockstep(wl)


def test_planted_score_ties_resolve_to_recent_position():
    """Exact score ties at the eviction boundary: slots 8..15 and the chunk
    tokens receive weights that underflow to exactly 0 in fp32 and start from
    score 0, so 12 candidates tie at 0.0 for 8 places; the most recent
    positions must win."""
    C, T, d = 16, 4, 128
    wl = synth.Workload("ties", "bf16", B=1, Hq=2, Hkv=1, d=d, C=C, T=T, N=T, seed=1)
    cache = H2OCache(1, 2, 1, d, C, torch.bfloat16, max_T=T)
    K, V, S, pos = synth.random_state(wl, n=C, P=1000, seed=4)
    far = -200.0 * np.sqrt(d)           # logit about -200: weight exactly 0 in fp32
    K[0, 0, :8] = 0.0                   # logit 0: these eight share all the weight
    K[0, 0, 8:] = 0.0
    K[0, 0, 8:, 0] = far
    S[0, 0, :8] = 10.0
    S[0, 0, 8:] = 0.0
    K = synth.round_bf16(K)
    cache.set_state(to_dev(K, "bf16"), to_dev(V, "bf16"), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=1000, n=C)
    q = np.zeros((1, 2, T, d), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, T, d), np.float32)
    k[..., 0] = far
    k = synth.round_bf16(k)
    v = np.random.default_rng(0).standard_normal((1, 1, T, d)).astype(np.float32)
    v = synth.round_bf16(v)
    pre = oracle_state_from_device(cache)
    g = gpu_step(cache, q, k, v, "bf16")
    cs = g["cand_score"][0, 0]
    assert (cs[8:] == 0.0).all() and (cs[:8] > 10.0).all()
    tied_pos = np.concatenate([pos[0, 0, 8:], 1000 + np.arange(T)])
    winners = set(np.sort(tied_pos)[-8:].tolist())
    kept_pos = set(g["cand_pos"][0, 0][g["kept"][0, 0] == 1].tolist())
    assert kept_pos == set(pos[0, 0, :8].tolist()) | winners
    check_selection_replay(g, pre, k, v, C, T)


def test_step_host_matches_device_step():
    wl = synth.Workload("host", "bf16", B=1, Hq=8, Hkv=2, d=128, C=256, T=128, N=512, seed=8,
                        recipe="heavy", hh_frac=0.03)
    a = H2OCache(1, 8, 2, 128, 256, torch.bfloat16, max_T=128)
    b = H2OCache(1, 8, 2, 128, 256, torch.bfloat16, max_T=128)
    for c in range(wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
        out_a = a.step(qd, kd, vd)
        out_b = torch.empty_like(qd).cpu().pin_memory()
        b.step_host(qd.cpu().pin_memory(), kd.cpu().pin_memory(), vd.cpu().pin_memory(), out_b)
        torch.cuda.synchronize()
        assert torch.equal(out_a.cpu(), out_b)
    assert torch.equal(a.positions(), b.positions())
    assert torch.equal(a.scores(), b.scores())


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_step_host_async_matches_device_step(dtype):
    """The pipelined host path (two staging slots, upload/download streams)
    gives exactly the device path's outputs, scores and positions, with all
    chunks enqueued before one host_sync; a longer chunk in the middle grows
    the staging slots."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = 128 if dtype == "bf16" else 64
    wl = synth.Workload("host-async", dtype, B=2, Hq=8, Hkv=2, d=d, C=256, T=96, N=96 * 6, seed=11,
                        recipe="heavy", hh_frac=0.03)
    a = H2OCache(2, 8, 2, d, 256, tdt, max_T=160)
    b = H2OCache(2, 8, 2, d, 256, tdt, max_T=160)
    lens = [96, 96, 160, 96, 33, 96]  # chunk lengths: growth, then shorter chunks
    ins, outs_a, outs_b = [], [], []
    for c, T in enumerate(lens):
        q, k, v = (x[:, :, :T].copy() for x in synth.chunk(wl.with_(T=max(lens)), c))
        qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
        outs_a.append(a.step(qd, kd, vd).cpu())
        host = tuple(t.cpu().pin_memory() for t in (qd, kd, vd))
        ins.append(host)  # kept alive until host_sync
        outs_b.append(torch.empty_like(host[0]).pin_memory())
        b.step_host_async(*host, outs_b[-1])
    b.host_sync()
    torch.cuda.synchronize()
    for oa, ob in zip(outs_a, outs_b):
        assert torch.equal(oa, ob)
    assert torch.equal(a.positions(), b.positions())
    assert torch.equal(a.scores(), b.scores())


def test_bounded_wait_reports_timeout():
    """A kernel waiting on a barrier nobody completes gives up and reports
    H2O_ERR_TIMEOUT; the CUDA context stays usable."""
    from h2o_kv_cache_step_b200._lib import H2O_ERR_POISONED, H2O_ERR_TIMEOUT, lib
    cache = H2OCache(1, 2, 1, 64, 8, torch.float32, max_T=4)
    rc = lib().h2o_selftest_wait(cache.handle, 50, None)
    assert rc == H2O_ERR_TIMEOUT
    assert lib().h2o_sync_check(cache.handle, None) == H2O_ERR_POISONED
    x = torch.ones(1000, device="cuda")
    assert float((x * 2).sum()) == 2000.0  # context still fine
    cache.close()


def test_set_state_rejects_holes_and_duplicates():
    from h2o_kv_cache_step_b200._lib import H2OError
    cache = H2OCache(1, 2, 1, 64, 8, torch.float32, max_T=4)
    K = torch.zeros(1, 1, 8, 64, device="cuda")
    S = torch.zeros(1, 1, 8, device="cuda")
    bad = [torch.tensor([[[0, 1, -1, 3, -1, -1, -1, -1]]], dtype=torch.int32),   # hole
           torch.tensor([[[0, 1, 1, 3, -1, -1, -1, -1]]], dtype=torch.int32),    # duplicate
           torch.tensor([[[0, 1, 2, 9, -1, -1, -1, -1]]], dtype=torch.int32)]    # >= P
    for p in bad:
        with pytest.raises(H2OError):
            cache.set_state(K, K, S, p.cuda(), P=8, n=4)


# --------------------------------------------------------------- full size ---
FULL = [w for w in synth.WORKLOAD_ORDER if w != "tiny-fp32"]


@pytest.mark.slow
@pytest.mark.parametrize("name,policy", [(n, oracle.POLICY_SUM) for n in FULL] +
                         [(FULL[0], oracle.POLICY_NORMALIZED)])
def test_full_size_sampled(name, policy):
    """One steady-state step at the workload's full size: a full cache
    (random scores and scattered positions) and one real chunk. Checks
    sampled output rows and LSEs, every candidate score of one whole group,
    and the selection of every group (replayed on the GPU's scores)."""
    wl = synth.WORKLOADS[name]
    P = wl.C + 3 * wl.T  # a mid-sequence position
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, torch.bfloat16, max_T=wl.T)
    cache.set_policy(policy)
    K, V, S, pos = synth.random_state(wl, n=wl.C, P=P, seed=99)
    cache.set_state(to_dev(K, "bf16"), to_dev(V, "bf16"), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=P, n=wl.C)
    c = P // wl.T
    q, k, v = synth.chunk(wl, c)
    pre = oracle_state_from_device(cache)
    g = gpu_step(cache, q, k, v, "bf16")
    rng = np.random.default_rng(5)
    T = wl.T
    rows = np.stack([rng.integers(0, wl.B, 64), rng.integers(0, wl.Hq, 64),
                     np.concatenate([[0, 1, T - 1, T - 2], rng.integers(0, T, 60)])], axis=1)
    o_ref, l_ref = oracle.rows(pre, q, k, v, rows)
    o_gpu = g["out"][rows[:, 0], rows[:, 1], rows[:, 2]]
    l_gpu = g["lse"][rows[:, 0], rows[:, 1], rows[:, 2]]
    record_errors(f"full size {name} sampled rows", o_gpu, o_ref, l_gpu, l_ref)
    assert np.abs(o_gpu - o_ref).max() <= TOL_OUT["bf16"]
    assert np.abs(l_gpu - l_ref).max() <= TOL_LSE["bf16"]
    # one whole group through the full oracle step
    b, gg = wl.B - 1, wl.Hkv // 2
    G = wl.G
    sub = oracle.State(pre.K[b:b + 1, gg:gg + 1].copy(), pre.V[b:b + 1, gg:gg + 1].copy(),
                       pre.phi[b:b + 1, gg:gg + 1].copy(), pre.pos[b:b + 1, gg:gg + 1].copy(), pre.P)
    res = oracle.step(sub, q[b:b + 1, gg * G:(gg + 1) * G], k[b:b + 1, gg:gg + 1], v[b:b + 1, gg:gg + 1],
                      nthreads=8, policy=policy)
    nc = wl.C + T
    compare_scores(g["cand_score"][b, gg], res.cand_score[0, 0, :nc], f"{name} group scores")
    assert np.abs(g["out"][b, gg * G:(gg + 1) * G] - res.out[0]).max() <= TOL_OUT["bf16"]
    check_selection_replay(g, pre, k, v, wl.C, T, policy)
