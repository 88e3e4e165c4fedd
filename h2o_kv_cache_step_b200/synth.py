"""Seeded synthetic inputs for the chunked H2O step.

This module only draws random numbers; it holds none of the step's arithmetic.
Both the CUDA path and the oracle consume what it produces. Every tensor is
drawn on the host from a numpy PCG64 stream keyed by (seed, sequence, chunk,
tensor), so any chunk can be regenerated on its own, and is rounded
round-to-nearest-even to bf16 for bf16 workloads, so the device and the oracle
see identical values.

Shapes follow a Qwen3-4B attention layer (32 query heads, 8 KV heads, head
dimension 128), the model the paper fine-tunes ("Learning how to Forget",
metallab page, Table 2 caption); the long-context benchmark sequences the
paper evaluates on are not available, so these recipes stand in for them:

* ``iid``      Q, K, V i.i.d. N(0, 1).
* ``heavy``    K, V ~ N(0, 1). Per (sequence, KV head g) a direction
               m_g = sqrt(d) * u, u uniform on the unit sphere. Query head h
               draws N(0, I) + 0.5 * m_{g(h)}. A set of floor(frac * N)
               positions (without replacement, shared by all KV heads) are
               heavy hitters, whose key is 3 * m_g.
* ``student``  K i.i.d. Student-t(3) clipped to [-8, 8]; Q, V ~ N(0, 1).
"""
from __future__ import annotations

import functools
from dataclasses import dataclass, replace

import numpy as np

_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "fp32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    d: int
    C: int
    T: int
    N: int                # tokens per sequence
    seed: int
    recipe: str = "iid"   # "iid" | "heavy" | "student"
    hh_frac: float = 0.0  # heavy-hitter fraction (recipe "heavy")
    per_seq_seed_base: int = -1  # >= 0: sequence b uses seed base+b and draws its own hh_frac
    hh_frac_range: tuple = (0.0, 0.0)

    @property
    def n_chunks(self) -> int:
        return self.N // self.T

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny-fp32": Workload("tiny-fp32", "fp32", B=1, Hq=4, Hkv=2, d=64, C=256, T=64, N=768,
                          seed=0, recipe="iid"),
    "qwen3-4b-c2048-t1024-n64k": Workload("qwen3-4b-c2048-t1024-n64k", "bf16", B=1, Hq=32, Hkv=8,
                                          d=128, C=2048, T=1024, N=65536, seed=1,
                                          recipe="heavy", hh_frac=0.02),
    "qwen3-4b-c1024-t1024-n128k": Workload("qwen3-4b-c1024-t1024-n128k", "bf16", B=1, Hq=32,
                                           Hkv=8, d=128, C=1024, T=1024, N=131072, seed=2,
                                           recipe="heavy", hh_frac=0.01),
    "qwen3-4b-b4-c4096-t2048-n32k": Workload("qwen3-4b-b4-c4096-t2048-n32k", "bf16", B=4, Hq=32,
                                             Hkv=8, d=128, C=4096, T=2048, N=32768, seed=3,
                                             recipe="heavy", per_seq_seed_base=30,
                                             hh_frac_range=(0.005, 0.05)),
    "qwen3-4b-c16384-t512-n128k": Workload("qwen3-4b-c16384-t512-n128k", "bf16", B=1, Hq=32,
                                           Hkv=8, d=128, C=16384, T=512, N=131072, seed=4,
                                           recipe="student"),
}
# The five workloads in the order they are usually listed.
WORKLOAD_ORDER = ["tiny-fp32", "qwen3-4b-c2048-t1024-n64k", "qwen3-4b-c1024-t1024-n128k",
                  "qwen3-4b-b4-c4096-t2048-n32k", "qwen3-4b-c16384-t512-n128k"]


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def _seq_seed(wl: Workload, b: int) -> int:
    return wl.per_seq_seed_base + b if wl.per_seq_seed_base >= 0 else wl.seed


@functools.lru_cache(maxsize=64)
def _sequence_params(wl: Workload, b: int):
    """Per-sequence draws: KV-head directions, heavy-hitter fraction and set."""
    seed = _seq_seed(wl, b)
    rng = _rng(seed, b, 1_000_001)
    u = rng.standard_normal((wl.Hkv, wl.d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    m = (np.sqrt(wl.d) * u).astype(np.float32)
    frac = wl.hh_frac
    if wl.per_seq_seed_base >= 0:
        lo, hi = wl.hh_frac_range
        frac = float(_rng(seed, b, 1_000_002).uniform(lo, hi))
    n_hh = int(np.floor(frac * wl.N)) if wl.recipe == "heavy" else 0
    hh = np.sort(_rng(seed, b, 1_000_003).choice(wl.N, size=n_hh, replace=False)) if n_hh else \
        np.zeros(0, np.int64)
    return m, frac, hh


def heavy_hitters(wl: Workload, b: int) -> np.ndarray:
    """Sorted heavy-hitter positions of sequence b (empty unless recipe 'heavy')."""
    return _sequence_params(wl, b)[2]


def chunk(wl: Workload, c: int):
    """Inputs of chunk c (positions c*T .. c*T+T-1) as float32 arrays:
    q [B,Hq,T,d], k [B,Hkv,T,d], v [B,Hkv,T,d]; bf16-representable values
    when ``wl.dtype == 'bf16'``."""
    B, Hq, Hkv, d, T = wl.B, wl.Hq, wl.Hkv, wl.d, wl.T
    q = np.empty((B, Hq, T, d), np.float32)
    k = np.empty((B, Hkv, T, d), np.float32)
    v = np.empty((B, Hkv, T, d), np.float32)
    for b in range(B):
        seed = _seq_seed(wl, b)
        rq = _rng(seed, b, c, _TENSOR_ID["q"])
        rk = _rng(seed, b, c, _TENSOR_ID["k"])
        rv = _rng(seed, b, c, _TENSOR_ID["v"])
        q[b] = rq.standard_normal((Hq, T, d), dtype=np.float32)
        v[b] = rv.standard_normal((Hkv, T, d), dtype=np.float32)
        if wl.recipe == "student":
            k[b] = np.clip(rk.standard_t(3, size=(Hkv, T, d)), -8.0, 8.0).astype(np.float32)
        else:
            k[b] = rk.standard_normal((Hkv, T, d), dtype=np.float32)
        if wl.recipe == "heavy":
            m, _, hh = _sequence_params(wl, b)
            G = Hq // Hkv
            q[b] += 0.5 * np.repeat(m, G, axis=0)[:, None, :]
            lo, hi = np.searchsorted(hh, [c * T, c * T + T])
            t_hh = hh[lo:hi] - c * T
            if t_hh.size:
                k[b][:, t_hh, :] = 3.0 * m[:, None, :]
    if wl.dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return q, k, v


def random_state(wl: Workload, n: int, P: int, seed: int = 12345, score_scale: float = 4.0):
    """A synthetic pre-step cache with n valid slots (slots 0..n-1), for
    lockstep checks: K, V drawn like chunk keys/values, positions a random
    increasing subset of 0..P-1, scores uniform in [0, score_scale).
    Returns float32 K, V [B,Hkv,C,d], float32 scores and int32 positions
    [B,Hkv,C] (0 / -1 in the empty slots)."""
    B, Hkv, C, d = wl.B, wl.Hkv, wl.C, wl.d
    assert 0 <= n <= C and n <= P
    rng = _rng(seed, n, P, 7)
    K = np.zeros((B, Hkv, C, d), np.float32)
    V = np.zeros((B, Hkv, C, d), np.float32)
    S = np.zeros((B, Hkv, C), np.float32)
    pos = np.full((B, Hkv, C), -1, np.int32)
    if n:
        if wl.recipe == "student":
            K[:, :, :n] = np.clip(rng.standard_t(3, size=(B, Hkv, n, d)), -8, 8)
        else:
            K[:, :, :n] = rng.standard_normal((B, Hkv, n, d))
        V[:, :, :n] = rng.standard_normal((B, Hkv, n, d))
        S[:, :, :n] = rng.uniform(0, score_scale, size=(B, Hkv, n))
        for b in range(B):
            for g in range(Hkv):
                p = np.sort(rng.choice(P, size=n, replace=False))
                pos[b, g, :n] = rng.permutation(p)
    if wl.dtype == "bf16":
        K, V = round_bf16(K), round_bf16(V)
    return K, V, S, pos
