"""Brute-force reference for pinning the fp64 oracle on tiny inputs.

TEST INFRASTRUCTURE ONLY. A second, structurally different restatement of the
chunked H2O step ("Learning how to Forget", paper page, sections
"Improvements to Heavy-Hitter Oracle (H2O)" and "Kernel Support Needs"): the
cache is a dictionary from token position to (key, value, score); there are
no slots. Attention is a dense numpy softmax over an explicit key list; the
eviction is a full Python sort. It shares no code with ``h2o_oracle.c``.
"""
from __future__ import annotations

import numpy as np


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


class BruteH2O:
    """Set-based H2O over chunks for one batch of sequences (fp64).

    cache[b][g] maps position -> [key (d,), value (d,), score].
    """

    def __init__(self, B: int, Hq: int, Hkv: int, d: int, C: int, normalized: bool = False,
                 insert_always: bool = False):
        """normalized: rank eviction candidates by score / age (age = token
        count after the step minus the position, the same section's improved
        score) instead of by the score."""
        self.B, self.Hq, self.Hkv, self.d, self.C = B, Hq, Hkv, d, C
        self.normalized = normalized
        # insert_always: evict the lowest-scoring entries before the chunk
        # attends (by the scores so far), so every chunk token enters
        self.insert_always = insert_always
        self.G = Hq // Hkv
        self.P = 0
        self.cache = [[dict() for _ in range(Hkv)] for _ in range(B)]

    def step(self, q, k, v):
        """q [B,Hq,T,d], k/v [B,Hkv,T,d]. Returns out, lse, per-group dict
        position -> updated score (all candidates), per-group kept position set."""
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        B, Hq, T, d = q.shape
        scale = 1.0 / np.sqrt(d)
        out = np.zeros((B, Hq, T, d))
        lse = np.zeros((B, Hq, T))
        scores, kept_sets = [], []
        for b in range(B):
            scores.append([])
            kept_sets.append([])
            for g in range(self.Hkv):
                old = self.cache[b][g]
                if self.insert_always:
                    extra = len(old) + T - self.C
                    if extra > 0:
                        lowest = sorted(old, key=lambda p: (old[p][2], p))[:extra]
                        old = {p: e for p, e in old.items() if p not in lowest}
                cand = {p: [e[0], e[1], e[2]] for p, e in old.items()}
                for t in range(T):
                    cand[self.P + t] = [k[b, g, t], v[b, g, t], 0.0]
                positions = sorted(cand)
                Kmat = np.stack([cand[p][0] for p in positions])
                Vmat = np.stack([cand[p][1] for p in positions])
                posv = np.array(positions)
                add = np.zeros(len(positions))
                for hh in range(self.G):
                    h = g * self.G + hh
                    for i in range(T):
                        vis = posv <= self.P + i
                        l = scale * (Kmat[vis] @ q[b, h, i])
                        w = softmax_rows(l[None, :])[0]
                        out[b, h, i] = w @ Vmat[vis]
                        m = l.max()
                        lse[b, h, i] = m + np.log(np.exp(l - m).sum())
                        add[vis] += w
                for idx, p in enumerate(positions):
                    cand[p][2] = cand[p][2] + add[idx]
                scores[b].append({p: cand[p][2] for p in positions})
                t_now = self.P + T
                rank = (lambda p: cand[p][2] / (t_now - p)) if self.normalized else (lambda p: cand[p][2])
                order = sorted(positions, key=lambda p: (rank(p), p), reverse=True)
                keep = set(order[: self.C]) if not self.insert_always else set(positions)
                kept_sets[b].append(keep)
                self.cache[b][g] = {p: cand[p] for p in keep}
        self.P += T
        return out, lse, scores, kept_sets


def dense_causal(q_all, k_all, v_all):
    """Full causal softmax attention over whole sequences (no cache limit).

    q_all [B,Hq,N,d], k_all/v_all [B,Hkv,N,d] -> out [B,Hq,N,d], lse [B,Hq,N],
    colsum [B,Hkv,N]: for each key j the sum over the group's heads and all
    rows i >= j of the attention weight of (i, j).
    """
    q_all = np.asarray(q_all, np.float64)
    k_all = np.asarray(k_all, np.float64)
    v_all = np.asarray(v_all, np.float64)
    B, Hq, N, d = q_all.shape
    Hkv = k_all.shape[1]
    G = Hq // Hkv
    out = np.zeros_like(q_all)
    lse = np.zeros((B, Hq, N))
    colsum = np.zeros((B, Hkv, N))
    mask = np.tril(np.ones((N, N), bool))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            l = (q_all[b, h] @ k_all[b, g].T) / np.sqrt(d)
            l = np.where(mask, l, -np.inf)
            m = l.max(axis=1, keepdims=True)
            e = np.exp(l - m)
            s = e.sum(axis=1, keepdims=True)
            w = e / s
            out[b, h] = w @ v_all[b, g]
            lse[b, h] = (m + np.log(s))[:, 0]
            colsum[b, g] += w.sum(axis=0)
    return out, lse, colsum
