"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each check here is independent of ``oracle/h2o_oracle.c``: a hand-worked
example with exact rational answers, a structurally different brute-force
simulation (``oracle/brute.py``), dense causal attention when nothing is
evicted, closed forms for constant logits, invariants of softmax and of the
eviction, and a brute-force sort for the selection.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import brute, oracle
from h2o_kv_cache_step_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(s):
    s = str(s)
    if s.startswith("ln(") and s.endswith(")"):
        return math.log(float(Fraction(s[3:-1])))
    return float(Fraction(s))


def run_both(B, Hq, Hkv, d, C, T, n_chunks, gen, normalized=False):
    """Run the oracle and the brute-force simulation over the same chunks and
    yield per-step results of both."""
    st = oracle.State.empty(B, Hkv, C, d)
    br = brute.BruteH2O(B, Hq, Hkv, d, C, normalized=normalized)
    policy = oracle.POLICY_NORMALIZED if normalized else oracle.POLICY_SUM
    for c in range(n_chunks):
        q, k, v = gen(c)
        n_before = st.n_valid.copy()
        res = oracle.step(st, q, k, v, policy=policy)
        bo, bl, bs, bk = br.step(q, k, v)
        yield c, n_before, st, res, (bo, bl, bs, bk)


def iid_gen(B, Hq, Hkv, d, T, seed, kscale=1.0):
    def gen(c):
        r = np.random.default_rng([seed, c])
        q = r.standard_normal((B, Hq, T, d))
        k = kscale * r.standard_normal((B, Hkv, T, d))
        v = r.standard_normal((B, Hkv, T, d))
        return q, k, v
    return gen


# ---------------------------------------------------------------- golden ---
@pytest.mark.parametrize("fname", ["worked_example_c2_t2.json", "worked_example_c2_t2_normalized.json"])
def test_hand_worked_example(oracle_lib, fname):
    g = json.load(open(os.path.join(GOLDEN, fname)))
    policy = oracle.POLICY_NORMALIZED if g.get("policy") == "normalized" else oracle.POLICY_SUM
    s = g["shape"]
    st = oracle.State.empty(s["B"], s["Hkv"], s["C"], s["d"])
    T = s["T"]
    for ch in g["chunks"]:
        q = np.array([_val(x) for x in ch["q"]]).reshape(1, 1, T, 1)
        k = np.array([_val(x) for x in ch["k"]]).reshape(1, 1, T, 1)
        v = np.array([_val(x) for x in ch["v"]]).reshape(1, 1, T, 1)
        r = oracle.step(st, q, k, v, policy=policy)
        n = int(r.n_cand[0, 0])
        np.testing.assert_allclose(r.out.ravel(), [_val(x) for x in ch["out"]], rtol=0, atol=1e-13)
        np.testing.assert_allclose(r.lse.ravel(), [_val(x) for x in ch["lse"]], rtol=0, atol=1e-13)
        assert r.cand_pos[0, 0, :n].tolist() == ch["cand_pos"]
        np.testing.assert_allclose(r.cand_score[0, 0, :n], [_val(x) for x in ch["cand_score"]],
                                   rtol=0, atol=1e-13)
        assert r.cand_kept[0, 0, :n].tolist() == ch["kept"]
        assert r.token_slot[0, 0].tolist() == ch["token_slot"]
        assert st.pos[0, 0].tolist() == ch["slot_pos"]
        np.testing.assert_allclose(st.phi[0, 0], [_val(x) for x in ch["slot_score"]], rtol=0, atol=1e-13)


# ----------------------------------------------------------- brute force ---
@pytest.mark.parametrize("B,Hq,Hkv,d,C,T,n_chunks,kscale", [
    (2, 4, 2, 8, 6, 3, 5, 1.0),     # GQA groups of 2, eviction from step 2 on
    (1, 2, 1, 5, 4, 1, 9, 2.0),     # T = 1: classic per-token H2O
    (1, 3, 3, 4, 3, 5, 3, 1.5),     # chunk longer than the cache (MHA)
    (1, 4, 1, 6, 7, 4, 4, 0.5),     # G = 4
])
@pytest.mark.parametrize("normalized", [False, True])
def test_oracle_matches_brute_force(oracle_lib, B, Hq, Hkv, d, C, T, n_chunks, kscale, normalized):
    gen = iid_gen(B, Hq, Hkv, d, T, seed=C * 100 + T, kscale=kscale)
    for c, n_before, st, res, (bo, bl, bs, bk) in run_both(B, Hq, Hkv, d, C, T, n_chunks, gen,
                                                           normalized=normalized):
        np.testing.assert_allclose(res.out, bo, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res.lse, bl, rtol=0, atol=1e-12)
        for b in range(B):
            for g in range(Hkv):
                n = int(res.n_cand[b, g])
                assert n == n_before[b, g] + T
                pos = res.cand_pos[b, g, :n]
                sc = dict(zip(pos.tolist(), res.cand_score[b, g, :n].tolist()))
                assert set(sc) == set(bs[b][g])
                for p, val in bs[b][g].items():
                    assert abs(sc[p] - val) <= 1e-12
                kept = set(pos[res.cand_kept[b, g, :n] == 1].tolist())
                assert kept == bk[b][g]
                assert set(st.pos[b, g][st.pos[b, g] >= 0].tolist()) == bk[b][g]


def test_heavy_hitter_workload_against_brute(oracle_lib):
    """The synthetic heavy-hitter recipe at a toy size: planted keys must win."""
    wl = synth.Workload("toy-heavy", "fp32", B=1, Hq=4, Hkv=2, d=16, C=8, T=4, N=32, seed=5,
                        recipe="heavy", hh_frac=0.15)
    hh = set(synth.heavy_hitters(wl, 0).tolist())
    gen = lambda c: synth.chunk(wl, c)
    for c, n_before, st, res, (bo, bl, bs, bk) in run_both(1, 4, 2, 16, 8, 4, wl.n_chunks, gen):
        np.testing.assert_allclose(res.out, bo, rtol=0, atol=1e-12)
        for g in range(2):
            assert set(st.pos[0, g][st.pos[0, g] >= 0].tolist()) == bk[0][g]
    kept_final = set(st.pos[0, 0][st.pos[0, 0] >= 0].tolist())
    assert hh <= kept_final  # 4 heavy hitters among 32 tokens all survive in 8 slots


# -------------------------------------------------- dense equivalence -----
@pytest.mark.parametrize("Hq,Hkv,d,T,n_chunks", [(4, 2, 8, 4, 5), (2, 1, 16, 7, 3), (3, 3, 4, 1, 10)])
def test_no_eviction_equals_dense_causal_attention(oracle_lib, Hq, Hkv, d, T, n_chunks):
    B, N = 2, T * n_chunks
    C = N + 3  # the cache never fills: chunked H2O is then exact attention
    r = np.random.default_rng([Hq, d, T])
    qa = r.standard_normal((B, Hq, N, d))
    ka = r.standard_normal((B, Hkv, N, d))
    va = r.standard_normal((B, Hkv, N, d))
    dout, dlse, dcol = brute.dense_causal(qa, ka, va)
    st = oracle.State.empty(B, Hkv, C, d)
    for c in range(n_chunks):
        sl = slice(c * T, c * T + T)
        res = oracle.step(st, qa[:, :, sl], ka[:, :, sl], va[:, :, sl])
        np.testing.assert_allclose(res.out, dout[:, :, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(res.lse, dlse[:, :, sl], rtol=0, atol=1e-12)
        assert (res.token_slot == np.arange(c * T, c * T + T)).all()
    # After the last chunk each slot's score is its key's full causal column sum.
    for b in range(B):
        for g in range(Hkv):
            p = st.pos[b, g]
            assert (p[:N] == np.arange(N)).all() and (p[N:] == -1).all()
            np.testing.assert_allclose(st.phi[b, g, :N], dcol[b, g], rtol=0, atol=1e-11)


# ------------------------------------------------------- closed forms -----
@pytest.mark.parametrize("n0,T,G", [(0, 5, 1), (3, 4, 2), (6, 6, 3)])
def test_zero_keys_closed_form(oracle_lib, n0, T, G):
    """K = 0 makes every visible logit 0: row i of the chunk (seeing n0+i+1
    keys) gives each key weight 1/(n0+i+1)."""
    d, C = 4, n0 + T  # no eviction in this step
    Hkv = 2
    Hq = G * Hkv
    r = np.random.default_rng(7)
    st = oracle.State.empty(1, Hkv, C, d)
    st.pos[:, :, :n0] = np.arange(n0)
    st.V[:, :, :n0] = r.standard_normal((1, Hkv, n0, d))
    st.phi[:, :, :n0] = 0.25
    st.P = n0
    q = r.standard_normal((1, Hq, T, d))
    k = np.zeros((1, Hkv, T, d))
    v = r.standard_normal((1, Hkv, T, d))
    Vc = st.V.copy()
    res = oracle.step(st, q, k, v)
    for g in range(Hkv):
        cache_delta = G * sum(1.0 / (n0 + i + 1) for i in range(T))
        n = int(res.n_cand[0, g])
        assert n == n0 + T
        np.testing.assert_allclose(res.cand_score[0, g, :n0], 0.25 + cache_delta, rtol=0, atol=1e-13)
        for t in range(T):
            want = G * sum(1.0 / (n0 + i + 1) for i in range(t, T))
            assert abs(res.cand_score[0, g, n0 + t] - want) <= 1e-13
        for hh in range(G):
            h = g * G + hh
            for i in range(T):
                vis = np.concatenate([Vc[0, g, :n0], v[0, g, : i + 1]])
                np.testing.assert_allclose(res.out[0, h, i], vis.mean(axis=0), rtol=0, atol=1e-13)
                assert abs(res.lse[0, h, i] - math.log(n0 + i + 1)) <= 1e-13


# --------------------------------------------------------- invariants -----
@pytest.mark.parametrize("C,T", [(5, 3), (8, 8), (3, 7), (16, 1)])
def test_invariants_over_a_sequence(oracle_lib, C, T):
    B, Hq, Hkv, d = 2, 6, 2, 8
    G = Hq // Hkv
    gen = iid_gen(B, Hq, Hkv, d, T, seed=99, kscale=1.3)
    st = oracle.State.empty(B, Hkv, C, d)
    for c in range(6):
        q, k, v = gen(c)
        n_before = st.n_valid.copy()
        phi_before = st.phi.copy()
        pos_before = st.pos.copy()
        # Weights of each row sum to 1: with all-ones values every output is 1.
        probe = st.copy()
        probe.V[:] = 1.0
        ones = oracle.step(probe, q, k, np.ones_like(v))
        np.testing.assert_allclose(ones.out, 1.0, rtol=0, atol=1e-12)
        res = oracle.step(st, q, k, v)
        for b in range(B):
            for g in range(Hkv):
                n = int(res.n_cand[b, g])
                # score mass: this step adds exactly G*T of weight to the group
                old = phi_before[b, g][pos_before[b, g] >= 0].sum()
                assert abs(res.cand_score[b, g, :n].sum() - old - G * T) <= 1e-9
                # exactly min(C, n+T) valid slots, unique positions
                valid = st.pos[b, g] >= 0
                assert valid.sum() == min(C, n_before[b, g] + T)
                assert len(set(st.pos[b, g][valid].tolist())) == valid.sum()
                # kept set = every candidate ranked above the C-th
                key = sorted(zip(res.cand_score[b, g, :n], res.cand_pos[b, g, :n]), reverse=True)
                want = {int(p) for _, p in key[:C]}
                got = set(res.cand_pos[b, g, :n][res.cand_kept[b, g, :n] == 1].tolist())
                assert got == want
                # kept cache entries did not move
                for j in range(C):
                    if pos_before[b, g, j] >= 0 and pos_before[b, g, j] in got:
                        assert st.pos[b, g, j] == pos_before[b, g, j]
                # kept chunk tokens went to the lowest free slots, in order
                ts = res.token_slot[b, g]
                placed = ts[ts >= 0]
                assert (np.diff(placed) > 0).all()
                free = [j for j in range(C) if not (pos_before[b, g, j] >= 0 and
                                                    pos_before[b, g, j] in got)]
                assert placed.tolist() == free[: len(placed)]


def test_permuting_cache_slots(oracle_lib):
    """Permuting the slots permutes per-slot results and leaves O unchanged."""
    B, Hq, Hkv, d, C, T = 1, 4, 2, 8, 6, 3
    gen = iid_gen(B, Hq, Hkv, d, T, seed=3)
    st = oracle.State.empty(B, Hkv, C, d)
    for c in range(3):
        oracle.step(st, *gen(c))
    perm = np.random.default_rng(1).permutation(C)
    st2 = oracle.State(st.K[:, :, perm].copy(), st.V[:, :, perm].copy(), st.phi[:, :, perm].copy(),
                       st.pos[:, :, perm].copy(), st.P)
    q, k, v = gen(3)
    r1 = oracle.step(st, q, k, v)
    r2 = oracle.step(st2, q, k, v)
    np.testing.assert_allclose(r1.out, r2.out, rtol=0, atol=1e-12)
    for b in range(B):
        for g in range(Hkv):
            n = int(r1.n_cand[b, g])
            s1 = dict(zip(r1.cand_pos[b, g, :n].tolist(), r1.cand_score[b, g, :n].tolist()))
            s2 = dict(zip(r2.cand_pos[b, g, :n].tolist(), r2.cand_score[b, g, :n].tolist()))
            assert s1.keys() == s2.keys()
            for p in s1:
                assert abs(s1[p] - s2[p]) <= 1e-12
            assert set(st.pos[b, g].tolist()) == set(st2.pos[b, g].tolist())


# ---------------------------------------------------------- selection -----
@pytest.mark.parametrize("seed", range(6))
def test_select_against_sort_with_planted_ties(oracle_lib, seed):
    r = np.random.default_rng(seed)
    C = int(r.integers(3, 40))
    T = int(r.integers(1, 30))
    n_valid = int(r.integers(0, C + 1))
    n = n_valid + T
    # few distinct score values -> many exact ties, broken by position
    scores = r.choice(np.array([0.0, 0.5, 1.0, 1e-30, 3.25]), size=n)
    pos = r.permutation(10 * n)[:n].astype(np.int64)
    slots = np.full(n, -1, np.int32)
    slots[:n_valid] = r.permutation(C)[:n_valid]
    kept, ts = oracle.select_group(C, T, scores, pos, slots)
    order = sorted(range(n), key=lambda a: (scores[a], pos[a]), reverse=True)
    want = set(order[: min(C, n)])
    assert set(np.nonzero(kept)[0].tolist()) == want
    occupied = {int(slots[a]) for a in range(n_valid) if kept[a]}
    free = [j for j in range(C) if j not in occupied]
    placed = [int(ts[t]) for t in range(T) if kept[n_valid + t]]
    assert placed == free[: len(placed)]
    assert all(ts[t] == -1 for t in range(T) if not kept[n_valid + t])


# ------------------------------------------------------- insert-always ---
def test_insert_always_hand_worked_example(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "worked_example_c3_t2_insert_always.json")))
    s = g["shape"]
    st = oracle.State.empty(s["B"], s["Hkv"], s["C"], s["d"])
    T = s["T"]
    for ch in g["chunks"]:
        q = np.array([_val(x) for x in ch["q"]]).reshape(1, 1, T, 1)
        k = np.array([_val(x) for x in ch["k"]]).reshape(1, 1, T, 1)
        v = np.array([_val(x) for x in ch["v"]]).reshape(1, 1, T, 1)
        out, lse, ts = oracle.step_insert_always(st, q, k, v)
        np.testing.assert_allclose(out.ravel(), [_val(x) for x in ch["out"]], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse.ravel(), [_val(x) for x in ch["lse"]], rtol=0, atol=1e-13)
        assert ts[0, 0].tolist() == ch["token_slot"]
        assert st.pos[0, 0].tolist() == ch["slot_pos"]
        np.testing.assert_allclose(st.phi[0, 0], [_val(x) for x in ch["slot_score"]], rtol=0, atol=1e-13)


@pytest.mark.parametrize("B,Hq,Hkv,d,C,T,n_chunks,kscale", [
    (2, 4, 2, 8, 6, 3, 5, 1.0),     # GQA groups of 2
    (1, 2, 1, 5, 4, 1, 9, 2.0),     # T = 1
    (1, 3, 3, 4, 5, 5, 3, 1.5),     # T = C: the whole cache turns over every step
    (1, 4, 1, 6, 7, 4, 4, 0.5),     # G = 4
])
def test_insert_always_matches_brute_force(oracle_lib, B, Hq, Hkv, d, C, T, n_chunks, kscale):
    gen = iid_gen(B, Hq, Hkv, d, T, seed=C * 7 + T, kscale=kscale)
    st = oracle.State.empty(B, Hkv, C, d)
    br = brute.BruteH2O(B, Hq, Hkv, d, C, insert_always=True)
    for c in range(n_chunks):
        q, k, v = gen(c)
        out, lse, ts = oracle.step_insert_always(st, q, k, v)
        bo, bl, bs, bk = br.step(q, k, v)
        np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)
        for b in range(B):
            for g in range(Hkv):
                valid = st.pos[b, g] >= 0
                assert set(st.pos[b, g][valid].tolist()) == bk[b][g]
                for slot in np.nonzero(valid)[0]:
                    assert abs(st.phi[b, g, slot] - bs[b][g][int(st.pos[b, g, slot])]) <= 1e-12
                # every chunk token entered, at the slot it reports
                P0 = st.P - T
                assert np.array_equal(st.pos[b, g, ts[b, g]], P0 + np.arange(T))


def test_insert_always_equals_the_step_while_nothing_is_evicted(oracle_lib):
    """With room for every chunk (n + T <= C) both orders give the same
    outputs, scores and slots: nothing is evicted before or after."""
    B, Hq, Hkv, d, C, T = 1, 4, 2, 8, 40, 6
    gen = iid_gen(B, Hq, Hkv, d, T, seed=77)
    a, b = oracle.State.empty(B, Hkv, C, d), oracle.State.empty(B, Hkv, C, d)
    for c in range(C // T):
        q, k, v = gen(c)
        out, lse, ts = oracle.step_insert_always(a, q, k, v)
        r = oracle.step(b, q, k, v)
        np.testing.assert_allclose(out, r.out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, r.lse, rtol=0, atol=1e-12)
        assert np.array_equal(ts, r.token_slot)
        assert np.array_equal(a.pos, b.pos)
        np.testing.assert_allclose(a.phi, b.phi, rtol=0, atol=1e-12)


def test_insert_always_score_mass_and_rejects_long_chunks(oracle_lib):
    """Each row's weights sum to one, so a step adds G*T of score per group
    (over the slots that survive it); a chunk longer than the cache is an
    argument error for this variant."""
    B, Hq, Hkv, d, C, T = 1, 6, 2, 4, 5, 3
    gen = iid_gen(B, Hq, Hkv, d, T, seed=5)
    st = oracle.State.empty(B, Hkv, C, d)
    for c in range(4):
        q, k, v = gen(c)
        before = st.phi.copy()
        pos_before = st.pos.copy()
        oracle.step_insert_always(st, q, k, v)
        for g in range(Hkv):
            kept_old = [j for j in range(C) if pos_before[0, g, j] >= 0 and st.pos[0, g, j] == pos_before[0, g, j]]
            mass = st.phi[0, g].sum() - before[0, g, kept_old].sum()
            assert abs(mass - (Hq // Hkv) * T) < 1e-12
    q, k, v = iid_gen(B, Hq, Hkv, d, C + 1, seed=6)(0)
    with pytest.raises(RuntimeError):
        oracle.step_insert_always(oracle.State.empty(B, Hkv, C, d), q, k, v)


# ------------------------------------------------------------- backward ---
def _backward_case(seed, B=1, Hq=4, Hkv=2, d=3, C=5, n=3, T=3, vconst=False):
    r = np.random.default_rng(seed)
    st = oracle.State.empty(B, Hkv, C, d)
    st.K[:, :, :n] = r.standard_normal((B, Hkv, n, d))
    st.V[:, :, :n] = r.standard_normal((B, Hkv, n, d))
    st.pos[:, :, :n] = np.arange(n)
    st.P = n + 2
    q = r.standard_normal((B, Hq, T, d))
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    if vconst:
        st.V[:, :, :n] = 0.7
        v[:] = 0.7
    dout = r.standard_normal((B, Hq, T, d))
    return st, q, k, v, dout


def _loss(st, q, k, v, dout):
    return float((oracle.step(st.copy(), q, k, v).out * dout).sum())


def test_backward_matches_finite_differences(oracle_lib):
    st, q, k, v, dout = _backward_case(1)
    dq, dKc, dVc, dk, dv = oracle.backward(st, q, k, v, dout)
    eps = 1e-6
    n = int(st.n_valid[0, 0])
    checks = [("q", q, dq), ("k", k, dk), ("v", v, dv)]
    for name, arr, grad in checks:
        for idx in np.ndindex(arr.shape):
            a = arr.copy(); a[idx] += eps
            b = arr.copy(); b[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            lp = _loss(st, **{**args, name: a}, dout=dout)
            lm = _loss(st, **{**args, name: b}, dout=dout)
            assert abs((lp - lm) / (2 * eps) - grad[idx]) < 1e-7, (name, idx)
    for name, grad in (("K", dKc), ("V", dVc)):
        for idx in np.ndindex(getattr(st, name).shape):
            if idx[2] >= n:
                assert grad[idx] == 0.0  # empty slot
                continue
            sp, sm = st.copy(), st.copy()
            getattr(sp, name)[idx] += eps
            getattr(sm, name)[idx] -= eps
            fd = (_loss(sp, q, k, v, dout) - _loss(sm, q, k, v, dout)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7, (name, idx)


def test_backward_matches_torch_autograd(oracle_lib):
    import torch
    st, q, k, v, dout = _backward_case(2, B=2, Hq=6, Hkv=3, d=5, C=7, n=6, T=4)
    dq, dKc, dVc, dk, dv = oracle.backward(st, q, k, v, dout)
    B, Hq, T, d = q.shape
    Hkv, C, G = k.shape[1], st.K.shape[2], q.shape[1] // k.shape[1]
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    tK = torch.tensor(st.K, requires_grad=True)
    tV = torch.tensor(st.V, requires_grad=True)
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            valid = [j for j in range(C) if st.pos[b, g, j] >= 0]
            for i in range(T):
                keys = torch.cat([tK[b, g, valid], tk[b, g, : i + 1]])
                vals = torch.cat([tV[b, g, valid], tv[b, g, : i + 1]])
                w = torch.softmax(keys @ tq[b, h, i] / np.sqrt(d), dim=0)
                loss = loss + (w @ vals * torch.tensor(dout[b, h, i])).sum()
    loss.backward()
    for ours, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (dKc, tK.grad), (dVc, tV.grad)):
        np.testing.assert_allclose(ours, ref.numpy(), rtol=0, atol=1e-12)


def test_backward_equal_values_give_no_query_or_key_gradient(oracle_lib):
    """With every visible value row equal, O does not depend on the weights:
    dq, dk and the cache's dK vanish; dV still receives the weights times dO."""
    st, q, k, v, dout = _backward_case(3, vconst=True)
    dq, dKc, dVc, dk, dv = oracle.backward(st, q, k, v, dout)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14 and np.abs(dKc).max() < 1e-14
    # every row's weights sum to one, so the value gradients add up to sum of dO per KV head
    G = q.shape[1] // k.shape[1]
    for g in range(k.shape[1]):
        total = dVc[0, g].sum(axis=0) + dv[0, g].sum(axis=0)
        np.testing.assert_allclose(total, dout[0, g * G:(g + 1) * G].sum(axis=(0, 1)), rtol=0, atol=1e-12)


# ------------------------------------------------------ selected rows -----
def _all_rows(B, Hq, T):
    return np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(T)], np.int32)


@pytest.mark.parametrize("B,Hq,Hkv,d,C,T,n_chunks", [
    (2, 4, 2, 8, 9, 4, 5),     # GQA; cache partly empty (n < C) in the first steps, then evicting
    (1, 6, 2, 5, 7, 5, 4),     # G = 3, T = 5 (ragged against any tile)
    (1, 2, 2, 4, 3, 7, 3),     # chunk longer than the cache
    (1, 4, 1, 6, 5, 1, 8),     # T = 1: only row 0, which is also row T - 1
])
def test_rows_match_brute_force(oracle_lib, B, Hq, Hkv, d, C, T, n_chunks):
    """The per-row checker (O and LSE of chosen rows against the pre-step
    cache) agrees with the structurally different brute force on every row of
    every step: a cold cache, a partly filled one and a full one."""
    gen = iid_gen(B, Hq, Hkv, d, T, seed=C * 31 + T)
    st = oracle.State.empty(B, Hkv, C, d)
    br = brute.BruteH2O(B, Hq, Hkv, d, C)
    rows = _all_rows(B, Hq, T)
    saw_partial = saw_full = False
    for c in range(n_chunks):
        q, k, v = gen(c)
        n_before = st.n_valid
        saw_partial |= bool(((n_before > 0) & (n_before < C)).any())
        saw_full |= bool((n_before == C).all())
        o_rows, l_rows = oracle.rows(st, q, k, v, rows)
        bo, bl, _, _ = br.step(q, k, v)
        oracle.step(st, q, k, v)
        for r, (b, h, i) in enumerate(rows):
            np.testing.assert_allclose(o_rows[r], bo[b, h, i], rtol=0, atol=1e-12)
            assert abs(l_rows[r] - bl[b, h, i]) <= 1e-12
    assert saw_full and (saw_partial or C <= T)


def test_rows_match_dense_causal_attention(oracle_lib):
    """With no eviction, row i of chunk c is row c*T + i of full causal
    attention (textbook softmax attention over the whole prefix)."""
    B, Hq, Hkv, d, T, n_chunks = 1, 4, 2, 8, 6, 4
    N = T * n_chunks
    r = np.random.default_rng(12)
    qa = r.standard_normal((B, Hq, N, d))
    ka = r.standard_normal((B, Hkv, N, d))
    va = r.standard_normal((B, Hkv, N, d))
    dout, dlse, _ = brute.dense_causal(qa, ka, va)
    st = oracle.State.empty(B, Hkv, N + 2, d)
    # rows 0 and T - 1 of every head, plus one interior row
    rows = np.array([(0, h, i) for h in range(Hq) for i in (0, 2, T - 1)], np.int32)
    for c in range(n_chunks):
        sl = slice(c * T, c * T + T)
        o_rows, l_rows = oracle.rows(st, qa[:, :, sl], ka[:, :, sl], va[:, :, sl], rows)
        for j, (b, h, i) in enumerate(rows):
            np.testing.assert_allclose(o_rows[j], dout[b, h, c * T + i], rtol=0, atol=1e-12)
            assert abs(l_rows[j] - dlse[b, h, c * T + i]) <= 1e-12
        oracle.step(st, qa[:, :, sl], ka[:, :, sl], va[:, :, sl])


def test_rows_rejects_out_of_range_rows(oracle_lib):
    st = oracle.State.empty(1, 1, 4, 2)
    q, k, v = iid_gen(1, 2, 1, 2, 3, seed=1)(0)
    for bad in ((1, 0, 0), (0, 2, 0), (0, 0, 3), (0, -1, 0)):
        with pytest.raises(RuntimeError):
            oracle.rows(st, q, k, v, np.array([bad], np.int32))
