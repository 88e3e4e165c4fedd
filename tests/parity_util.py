"""Lockstep parity between the CUDA step (through the C ABI) and the oracle.

The same pre-step state goes to both: it is read back from the device with
``h2o_get_state`` and widened to fp64 for the oracle. One step then runs on
each side and the results are compared element by element.

Tolerances (from the acceptance criteria of the step):
* attention output: 2e-2 max abs for bf16, 1e-4 for fp32;
* updated scores: |gpu - ref| <= 1e-3 * |ref| + 1e-7 (relative, with a floor
  for scores that are ~0);
* LSE: 2e-3 abs (bf16) / 1e-4 (fp32) -- the logits are fp32 dot products of
  the exact inputs, so LSE is far tighter than the output, which carries
  bf16 rounding of P and of O itself;
* selection: bit-exact. The oracle's selection is replayed on the GPU's own
  candidate scores, so a rounding-level difference in a score cannot flip
  a decision on one side only.
"""
from __future__ import annotations

import os

import numpy as np
import torch

from oracle import oracle

TOL_OUT = {"bf16": 2e-2, "fp32": 1e-4}
TOL_LSE = {"bf16": 2e-3, "fp32": 1e-4}
SCORE_RTOL = 1e-3
SCORE_ATOL = 1e-7
TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}


# Achieved errors of every parity comparison in this session, printed in the
# terminal summary (tests/conftest.py): the output bound of 2e-2 (bf16) is
# loose next to the size of O at long contexts, so the summary shows the
# error also relative to the largest |O| of the reference.
ERROR_LOG: list = []


def record_errors(label, out_gpu, out_ref, lse_gpu=None, lse_ref=None, score_rel=None):
    diff = np.abs(np.asarray(out_gpu, np.float64) - out_ref)
    out_err = float(diff.max())
    out_scale = float(np.abs(out_ref).max())
    # per output row: its largest error over its own largest |O| (a diffuse
    # row at a long context has |O| far below 1)
    d = diff.shape[-1]
    row_err = diff.reshape(-1, d).max(axis=1)
    row_ref = np.abs(np.asarray(out_ref)).reshape(-1, d).max(axis=1)
    row_rel = float((row_err / np.maximum(row_ref, 1e-30)).max())
    rec = dict(case=label or os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
               out_max_abs=out_err, out_max_ref=out_scale,
               out_rel=out_err / out_scale if out_scale > 0 else 0.0, row_rel=row_rel,
               lse_max_abs=float(np.abs(lse_gpu - lse_ref).max()) if lse_gpu is not None else None,
               score_rel=score_rel)
    ERROR_LOG.append(rec)
    return rec


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to("cuda").to(TORCH_DTYPE[dtype])


def oracle_state_from_device(cache) -> oracle.State:
    K, V, S, Pos, P, n = cache.get_state()
    torch.cuda.synchronize()
    return oracle.State(K.double().cpu().numpy(), V.double().cpu().numpy(),
                        S.double().cpu().numpy(), Pos.long().cpu().numpy(), P)


def gpu_step(cache, q, k, v, dtype):
    """Run one step on the device; return everything needed for comparison."""
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    out = cache.step(qd, kd, vd)
    cache.sync_check()
    cs, cp, kept = cache.candidates()
    r = dict(out=out.float().cpu().numpy(), lse=cache.lse().cpu().numpy(),
             cand_score=cs.cpu().numpy(), cand_pos=cp.cpu().numpy(), kept=kept.cpu().numpy(),
             token_slot=cache.token_slots().cpu().numpy())
    K, V, S, Pos, P, n = cache.get_state()
    torch.cuda.synchronize()
    r.update(K=K.float().cpu().numpy(), V=V.float().cpu().numpy(), S=S.cpu().numpy(),
             Pos=Pos.cpu().numpy(), P=P, n=n)
    return r


def ranking_keys(cand_score, cand_pos, t_after, policy):
    """The eviction ranking key the device uses, in the device's precision:
    the fp32 score, or (normalized policy) the fp32 score divided by the fp32
    age t_after - pos, rounded to nearest. Returned as float64 (exact)."""
    s = np.asarray(cand_score, np.float32)
    if policy == oracle.POLICY_NORMALIZED:
        age = (np.int64(t_after) - np.asarray(cand_pos, np.int64)).astype(np.float32)
        s = (s / age).astype(np.float32)
    return s.astype(np.float64)


def check_selection_replay(g, pre: oracle.State, k, v, C, T, policy=oracle.POLICY_SUM):
    """Replay the oracle's selection on the GPU's candidate scores; kept flags,
    token slots and the new slot contents must match bit for bit."""
    B, Hkv = g["cand_score"].shape[:2]
    n_prev = g["cand_score"].shape[2] - T
    t_after = int(pre.P) + T
    for b in range(B):
        for gg in range(Hkv):
            cs = ranking_keys(g["cand_score"][b, gg], g["cand_pos"][b, gg], t_after, policy)
            cp = g["cand_pos"][b, gg].astype(np.int64)
            slot = np.concatenate([np.arange(n_prev, dtype=np.int32), np.full(T, -1, np.int32)])
            kept, ts = oracle.select_group(C, T, cs, cp, slot)
            assert np.array_equal(kept, g["kept"][b, gg]), f"kept differs in group ({b},{gg})"
            assert np.array_equal(ts, g["token_slot"][b, gg]), f"token slots differ in group ({b},{gg})"
            # new slot contents implied by the replay
            pos = pre.pos[b, gg].copy()
            sc = pre.phi[b, gg].astype(np.float32).copy()
            for c in range(n_prev):
                if kept[c]:
                    sc[c] = g["cand_score"][b, gg, c]
                else:
                    pos[c], sc[c] = -1, 0.0
            for t in range(T):
                if ts[t] >= 0:
                    pos[ts[t]] = cp[n_prev + t]
                    sc[ts[t]] = g["cand_score"][b, gg, n_prev + t]
            assert np.array_equal(pos, g["Pos"][b, gg]), f"positions differ in group ({b},{gg})"
            assert np.array_equal(sc.view(np.uint32), g["S"][b, gg].view(np.uint32)), \
                f"scores differ in group ({b},{gg})"
            placed = np.nonzero(ts >= 0)[0]
            assert np.array_equal(g["K"][b, gg, ts[placed]], np.asarray(k, np.float32)[b, gg, placed])
            assert np.array_equal(g["V"][b, gg, ts[placed]], np.asarray(v, np.float32)[b, gg, placed])
            kept_cache = [c for c in range(n_prev) if kept[c]]
            assert np.array_equal(g["K"][b, gg, kept_cache], pre.K[b, gg, kept_cache].astype(np.float32))


def compare_scores(gpu_scores, ref_scores, what=""):
    err = np.abs(gpu_scores.astype(np.float64) - ref_scores)
    bound = SCORE_RTOL * np.abs(ref_scores) + SCORE_ATOL
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} scores out of tolerance, worst "
                           f"|d|={err.max():.3e} at ref={ref_scores.ravel()[np.argmax(err)]:.4e}")
    return float((err / (np.abs(ref_scores) + SCORE_ATOL)).max())


def lockstep_full(cache, q, k, v, dtype, C, policy=oracle.POLICY_SUM):
    """One lockstep step with the full oracle step; returns stats."""
    pre = oracle_state_from_device(cache)
    ref_state = pre.copy()
    res = oracle.step(ref_state, q, k, v, policy=policy)
    g = gpu_step(cache, q, k, v, dtype)
    T = q.shape[2]
    out_err = float(np.abs(g["out"] - res.out).max())
    assert out_err <= TOL_OUT[dtype], f"output max abs err {out_err:.3e} > {TOL_OUT[dtype]}"
    lse_err = float(np.abs(g["lse"] - res.lse).max())
    assert lse_err <= TOL_LSE[dtype], f"lse max abs err {lse_err:.3e}"
    B, Hkv = g["cand_score"].shape[:2]
    nc = g["cand_score"].shape[2]
    assert (res.n_cand == nc).all()
    assert np.array_equal(g["cand_pos"], res.cand_pos[:, :, :nc].astype(np.int32))
    score_rel = compare_scores(g["cand_score"], res.cand_score[:, :, :nc], "candidate scores")
    check_selection_replay(g, pre, k, v, C, T, policy)
    same_sel = bool(np.array_equal(g["kept"], res.cand_kept[:, :, :nc]))
    record_errors(None, g["out"], res.out, g["lse"], res.lse, score_rel)
    return dict(out_err=out_err, lse_err=lse_err, score_rel=score_rel, same_selection=same_sel)
