"""Python side of the fp64 H2O oracle (ctypes over ``h2o_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the smoke check and by the
CPU-baseline leg of ``bench.py``; never by the product package. It shares no
code with the CUDA path.

The step it evaluates is the chunked H2O step of "Learning how to Forget:
Fine-tuning for Long-Context Sparse Attention" (paper page, sections
"Improvements to Heavy-Hitter Oracle (H2O)" and "Kernel Support Needs"); the
readings taken where the pages are silent are listed in ``h2o_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "h2o_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libh2o_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE fp64)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _SO)
    return _SO


def bind(L):
    """Declare the oracle's C signatures on a loaded library; returns it."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.h2o_oracle_step.argtypes = [I, I, I, I, I, I, ctypes.c_int64] + [P] * 15 + [I]
    L.h2o_oracle_step.restype = I
    L.h2o_oracle_step_policy.argtypes = [I, I, I, I, I, I, ctypes.c_int64, I] + [P] * 15 + [I]
    L.h2o_oracle_step_policy.restype = I
    L.h2o_oracle_step_insert.argtypes = [I, I, I, I, I, I, ctypes.c_int64] + [P] * 10 + [I]
    L.h2o_oracle_step_insert.restype = I
    L.h2o_oracle_backward.argtypes = [I, I, I, I, I, I, ctypes.c_int64] + [P] * 12 + [I]
    L.h2o_oracle_backward.restype = I
    L.h2o_oracle_select_group.argtypes = [I, I, I, P, P, P, P, P]
    L.h2o_oracle_select_group.restype = I
    L.h2o_oracle_rows.argtypes = [I, I, I, I, I, I, ctypes.c_int64] + [P] * 6 + [I, P, P, P, I]
    L.h2o_oracle_rows.restype = I
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(build()))
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class State:
    """Cache state of the oracle: per (batch, KV head) C slots.

    K, V float64 [B,Hkv,C,d]; phi float64 [B,Hkv,C] (0 where empty);
    pos int64 [B,Hkv,C] (-1 = empty); P = tokens already processed.
    """
    K: np.ndarray
    V: np.ndarray
    phi: np.ndarray
    pos: np.ndarray
    P: int = 0

    @staticmethod
    def empty(B: int, Hkv: int, C: int, d: int) -> "State":
        return State(K=np.zeros((B, Hkv, C, d)), V=np.zeros((B, Hkv, C, d)),
                     phi=np.zeros((B, Hkv, C)), pos=np.full((B, Hkv, C), -1, np.int64), P=0)

    def copy(self) -> "State":
        return State(self.K.copy(), self.V.copy(), self.phi.copy(), self.pos.copy(), self.P)

    @property
    def n_valid(self) -> np.ndarray:
        return (self.pos >= 0).sum(axis=-1)


@dataclass
class StepResult:
    out: np.ndarray          # [B,Hq,T,d]
    lse: np.ndarray          # [B,Hq,T]
    cand_score: np.ndarray   # [B,Hkv,C+T] (first n_cand entries used)
    cand_pos: np.ndarray     # [B,Hkv,C+T]
    cand_slot: np.ndarray    # [B,Hkv,C+T] (-1 for chunk tokens)
    cand_kept: np.ndarray    # [B,Hkv,C+T] uint8
    n_cand: np.ndarray       # [B,Hkv]
    token_slot: np.ndarray   # [B,Hkv,T] (-1 = dropped)
    extra: dict = field(default_factory=dict)


POLICY_SUM = 0         # rank candidates by the H2O score
POLICY_NORMALIZED = 1  # rank by the score over the candidate's age, t = P + T


def step(state: State, q: np.ndarray, k: np.ndarray, v: np.ndarray, nthreads: int = 0,
         policy: int = POLICY_SUM) -> StepResult:
    """One H2O step; mutates ``state`` in place and returns the step's outputs.
    ``policy`` picks the eviction ranking key (the stored scores are the sums
    under both)."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    B, Hq, T, d = q.shape
    _, Hkv, C, _ = state.K.shape
    assert k.shape == (B, Hkv, T, d) and v.shape == (B, Hkv, T, d)
    out = np.zeros((B, Hq, T, d))
    lse = np.zeros((B, Hq, T))
    cs = np.zeros((B, Hkv, C + T))
    cp = np.full((B, Hkv, C + T), -1, np.int64)
    cslot = np.full((B, Hkv, C + T), -1, np.int32)
    ck = np.zeros((B, Hkv, C + T), np.uint8)
    nc = np.zeros((B, Hkv), np.int32)
    ts = np.full((B, Hkv, T), -1, np.int32)
    rc = lib().h2o_oracle_step_policy(B, Hq, Hkv, d, C, T, int(state.P), int(policy),
                               _p(state.K), _p(state.V), _p(state.phi), _p(state.pos),
                               _p(q), _p(k), _p(v), _p(out), _p(lse),
                               _p(cs), _p(cp), _p(cslot), _p(ck), _p(nc), _p(ts), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"h2o_oracle_step failed: {rc}")
    state.P += T
    return StepResult(out, lse, cs, cp, cslot, ck, nc, ts)


def step_insert_always(state: State, q: np.ndarray, k: np.ndarray, v: np.ndarray, nthreads: int = 0):
    """The insert-always variant of the step (T <= C): evict the lowest-scoring
    valid slots first if the chunk does not fit, write the chunk into the
    free slots, then attend over the buffer under the position mask and add
    the weights to the scores. Mutates ``state``; returns (out, lse,
    token_slot)."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    B, Hq, T, d = q.shape
    _, Hkv, C, _ = state.K.shape
    assert k.shape == (B, Hkv, T, d) and v.shape == (B, Hkv, T, d)
    out = np.zeros((B, Hq, T, d))
    lse = np.zeros((B, Hq, T))
    ts = np.full((B, Hkv, T), -1, np.int32)
    rc = lib().h2o_oracle_step_insert(B, Hq, Hkv, d, C, T, int(state.P),
                                      _p(state.K), _p(state.V), _p(state.phi), _p(state.pos),
                                      _p(q), _p(k), _p(v), _p(out), _p(lse), _p(ts), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"h2o_oracle_step_insert failed: {rc}")
    state.P += T
    return out, lse, ts


def backward(state: State, q, k, v, dout, nthreads: int = 0):
    """Gradients of sum(dout * O) for one step's SDPA with the kept set fixed:
    returns dq [B,Hq,T,d], dKc, dVc [B,Hkv,C,d] (zero for empty slots) and
    dk, dv [B,Hkv,T,d]. ``state`` is the cache before the step (unchanged)."""
    q, k, v, dout = (np.ascontiguousarray(x, np.float64) for x in (q, k, v, dout))
    B, Hq, T, d = q.shape
    _, Hkv, C, _ = state.K.shape
    dq = np.zeros_like(q)
    dKc = np.zeros_like(state.K)
    dVc = np.zeros_like(state.V)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rc = lib().h2o_oracle_backward(B, Hq, Hkv, d, C, T, int(state.P), _p(state.K), _p(state.V), _p(state.pos),
                                   _p(q), _p(k), _p(v), _p(dout), _p(dq), _p(dKc), _p(dVc), _p(dk), _p(dv),
                                   int(nthreads))
    if rc != 0:
        raise RuntimeError(f"h2o_oracle_backward failed: {rc}")
    return dq, dKc, dVc, dk, dv


def select_group(C: int, T: int, cand_score, cand_pos, cand_slot):
    """Eviction and slot placement of one group on given candidate scores.

    Returns (kept uint8 [n_cand], token_slot int32 [T]). Used to replay the
    oracle's selection on scores produced elsewhere.
    """
    cs = np.ascontiguousarray(cand_score, np.float64)
    cp = np.ascontiguousarray(cand_pos, np.int64)
    cslot = np.ascontiguousarray(cand_slot, np.int32)
    n = cs.shape[0]
    kept = np.zeros(n, np.uint8)
    ts = np.full(T, -1, np.int32)
    rc = lib().h2o_oracle_select_group(C, T, n, _p(cs), _p(cp), _p(cslot), _p(kept), _p(ts))
    if rc != 0:
        raise RuntimeError(f"h2o_oracle_select_group failed: {rc}")
    return kept, ts


def rows(state: State, q, k, v, rows_bhi, nthreads: int = 0):
    """O and LSE of selected rows (b, h, i) against the pre-step state."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    B, Hq, T, d = q.shape
    _, Hkv, C, _ = state.K.shape
    r = np.ascontiguousarray(rows_bhi, np.int32).reshape(-1, 3)
    o = np.zeros((r.shape[0], d))
    l = np.zeros(r.shape[0])
    rc = lib().h2o_oracle_rows(B, Hq, Hkv, d, C, T, int(state.P), _p(state.K), _p(state.V),
                               _p(state.pos), _p(q), _p(k), _p(v), r.shape[0], _p(r),
                               _p(o), _p(l), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"h2o_oracle_rows failed: {rc}")
    return o, l
