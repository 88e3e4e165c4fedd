"""``H2OCache``: one C-ABI context driven with torch tensors.

Thin marshalling over ``libh2o.so``: torch provides device memory and the
current CUDA stream; every computation happens in the library's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import H2O_BF16, H2O_FP32, check, lib

_DTYPES = {torch.bfloat16: H2O_BF16, torch.float32: H2O_FP32}


def _stream_ptr(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


class H2OCache:
    """H2O KV cache of C slots per (sequence, KV head) on the current device.

    ``step(q, k, v)`` takes q [B,Hq,T,d] and k, v [B,Hkv,T,d] (contiguous CUDA
    tensors of the cache's dtype) and returns the attention output
    [B,Hq,T,d]; the cache, scores and positions update in place.
    """

    def __init__(self, B: int, Hq: int, Hkv: int, d: int, C: int,
                 dtype: torch.dtype = torch.bfloat16, max_T: int | None = None):
        self.B, self.Hq, self.Hkv, self.d, self.C = B, Hq, Hkv, d, C
        self.dtype = dtype
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        rc = lib().h2o_create_ex(B, Hq, Hkv, d, C, _DTYPES[dtype], int(max_T or C), ctypes.byref(h))
        check(rc, None)
        self._h = h

    # -- lifetime -----------------------------------------------------------
    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().h2o_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc: int) -> None:
        check(rc, self._h)

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    # -- the step -----------------------------------------------------------
    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        T = q.shape[2]
        for name, t, heads in (("q", q, self.Hq), ("k", k, self.Hkv), ("v", v, self.Hkv)):
            if (t.dtype != self.dtype or not t.is_cuda or not t.is_contiguous()
                    or tuple(t.shape) != (self.B, heads, T, self.d)):
                raise ValueError(f"{name}: need contiguous CUDA {self.dtype} of shape "
                                 f"{(self.B, heads, T, self.d)}, got {t.dtype} {tuple(t.shape)}")
        if out is None:
            out = torch.empty_like(q)
        self._check(lib().h2o_step(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), T,
                                   _stream_ptr(stream)))
        return out

    def prefill(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """nchunks steps in one call: q [nchunks, B, Hq, T, d], k and v
        [nchunks, B, Hkv, T, d] (contiguous, on the device); returns the
        outputs [nchunks, B, Hq, T, d]. Same results as step() per chunk."""
        if q.dim() != 5:
            raise ValueError("q: need [nchunks, B, Hq, T, d]")
        nch, T = q.shape[0], q.shape[3]
        for name, t, heads in (("q", q, self.Hq), ("k", k, self.Hkv), ("v", v, self.Hkv)):
            if (t.dtype != self.dtype or not t.is_cuda or not t.is_contiguous()
                    or tuple(t.shape) != (nch, self.B, heads, T, self.d)):
                raise ValueError(f"{name}: need contiguous CUDA {self.dtype} of shape "
                                 f"{(nch, self.B, heads, T, self.d)}, got {t.dtype} {tuple(t.shape)}")
        if out is None:
            out = torch.empty_like(q)
        elif out.dtype != q.dtype or tuple(out.shape) != tuple(q.shape) or not out.is_contiguous():
            raise ValueError("out: need a contiguous tensor like q")
        self._check(lib().h2o_prefill(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), T, nch,
                                      _stream_ptr(stream)))
        return out

    def backward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lse: torch.Tensor,
                 dout: torch.Tensor, stream=None):
        """Gradients of one step's attention for the key set it used, taking the
        cache as it stands now as that step's pre-step cache (restore it with
        set_state first when replaying). lse is the step's log-sum-exp.
        Returns fp32 (dq, dK, dV, dk, dv): dK, dV over the cache slots
        [B,Hkv,C,d], dk, dv over the chunk [B,Hkv,T,d]."""
        T = q.shape[2]
        for name, t, heads in (("q", q, self.Hq), ("k", k, self.Hkv), ("v", v, self.Hkv),
                               ("dout", dout, self.Hq)):
            if (t.dtype != self.dtype or not t.is_cuda or not t.is_contiguous()
                    or tuple(t.shape) != (self.B, heads, T, self.d)):
                raise ValueError(f"{name}: need contiguous CUDA {self.dtype} of shape "
                                 f"{(self.B, heads, T, self.d)}, got {t.dtype} {tuple(t.shape)}")
        if lse.dtype != torch.float32 or tuple(lse.shape) != (self.B, self.Hq, T) or not lse.is_contiguous():
            raise ValueError("lse: need contiguous float32 [B, Hq, T]")
        f32 = dict(dtype=torch.float32, device=self.device)
        dq = torch.empty((self.B, self.Hq, T, self.d), **f32)
        dK = torch.empty((self.B, self.Hkv, self.C, self.d), **f32)
        dV = torch.empty_like(dK)
        dk = torch.empty((self.B, self.Hkv, T, self.d), **f32)
        dv = torch.empty_like(dk)
        self._check(lib().h2o_backward(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(lse), _ptr(dout), T,
                                       _ptr(dq), _ptr(dK), _ptr(dV), _ptr(dk), _ptr(dv), _stream_ptr(stream)))
        return dq, dK, dV, dk, dv

    def set_policy(self, policy: int) -> None:
        """Eviction ranking for the following steps: _lib.H2O_POLICY_SUM (the
        H2O score, default) or _lib.H2O_POLICY_NORMALIZED (score / age)."""
        self._check(lib().h2o_set_policy(self._h, int(policy)))

    def _check_host(self, q, k, v, out) -> int:
        T = q.shape[2]
        for name, t, heads in (("q", q, self.Hq), ("k", k, self.Hkv), ("v", v, self.Hkv), ("out", out, self.Hq)):
            if (t.is_cuda or not t.is_contiguous() or t.dtype != self.dtype
                    or tuple(t.shape) != (self.B, heads, T, self.d)):
                raise ValueError(f"{name}: need a contiguous host {self.dtype} tensor of shape "
                                 f"{(self.B, heads, T, self.d)}, got {t.dtype} {tuple(t.shape)}")
        return T

    def step_host(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  out: torch.Tensor, stream=None) -> torch.Tensor:
        """Same step on host (CPU) tensors; pinned memory gives async copies.
        Returns once the output is in `out`."""
        T = self._check_host(q, k, v, out)
        self._check(lib().h2o_step_host(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), T,
                                        _stream_ptr(stream)))
        return out

    def step_host_async(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        out: torch.Tensor, stream=None) -> torch.Tensor:
        """Pipelined step on host tensors (use pinned memory): returns at once;
        the inputs must stay unchanged and `out` is valid only after
        host_sync(). Successive chunks overlap copies with the steps."""
        T = self._check_host(q, k, v, out)
        self._check(lib().h2o_step_host_async(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), T,
                                              _stream_ptr(stream)))
        return out

    def host_sync(self) -> None:
        """Wait for every step_host_async copy (outputs are then in host memory)."""
        self._check(lib().h2o_host_sync(self._h))

    # -- inspection ---------------------------------------------------------
    def counters(self) -> tuple[int, int]:
        P, n = ctypes.c_int64(), ctypes.c_int64()
        self._check(lib().h2o_counters(self._h, ctypes.byref(P), ctypes.byref(n)))
        return P.value, n.value

    def scores(self, stream=None) -> torch.Tensor:
        dst = torch.empty((self.B, self.Hkv, self.C), dtype=torch.float32, device=self.device)
        self._check(lib().h2o_scores(self._h, _ptr(dst), _stream_ptr(stream)))
        return dst

    def positions(self, stream=None) -> torch.Tensor:
        dst = torch.empty((self.B, self.Hkv, self.C), dtype=torch.int32, device=self.device)
        self._check(lib().h2o_positions(self._h, _ptr(dst), _stream_ptr(stream)))
        return dst

    def last_step_info(self) -> tuple[int, int]:
        T, n = ctypes.c_int(), ctypes.c_int()
        self._check(lib().h2o_last_step_info(self._h, ctypes.byref(T), ctypes.byref(n)))
        return T.value, n.value

    def candidates(self, stream=None):
        """(scores float, positions int32, kept uint8), each [B,Hkv,n_prev+T]."""
        T, n = self.last_step_info()
        shape = (self.B, self.Hkv, n + T)
        s = torch.empty(shape, dtype=torch.float32, device=self.device)
        p = torch.empty(shape, dtype=torch.int32, device=self.device)
        kp = torch.empty(shape, dtype=torch.uint8, device=self.device)
        self._check(lib().h2o_candidates(self._h, _ptr(s), _ptr(p), _ptr(kp), _stream_ptr(stream)))
        return s, p, kp

    def token_slots(self, stream=None) -> torch.Tensor:
        T, _ = self.last_step_info()
        dst = torch.empty((self.B, self.Hkv, T), dtype=torch.int32, device=self.device)
        self._check(lib().h2o_token_slots(self._h, _ptr(dst), _stream_ptr(stream)))
        return dst

    def lse(self, stream=None) -> torch.Tensor:
        T, _ = self.last_step_info()
        dst = torch.empty((self.B, self.Hq, T), dtype=torch.float32, device=self.device)
        self._check(lib().h2o_lse(self._h, _ptr(dst), _stream_ptr(stream)))
        return dst

    def get_state(self, stream=None):
        """(K, V, scores, positions, P, n) copies of the current cache."""
        shape = (self.B, self.Hkv, self.C, self.d)
        K = torch.empty(shape, dtype=self.dtype, device=self.device)
        V = torch.empty(shape, dtype=self.dtype, device=self.device)
        S = torch.empty(shape[:3], dtype=torch.float32, device=self.device)
        Pos = torch.empty(shape[:3], dtype=torch.int32, device=self.device)
        P, n = ctypes.c_int64(), ctypes.c_int64()
        self._check(lib().h2o_get_state(self._h, _ptr(K), _ptr(V), _ptr(S), _ptr(Pos),
                                        ctypes.byref(P), ctypes.byref(n), _stream_ptr(stream)))
        return K, V, S, Pos, P.value, n.value

    def set_state(self, K, V, scores, positions, P: int, n: int, stream=None) -> None:
        K, V = K.contiguous(), V.contiguous()
        scores, positions = scores.contiguous(), positions.contiguous()
        self._check(lib().h2o_set_state(self._h, _ptr(K), _ptr(V), _ptr(scores), _ptr(positions),
                                        int(P), int(n), _stream_ptr(stream)))

    def reset(self, stream=None) -> None:
        self._check(lib().h2o_reset(self._h, _stream_ptr(stream)))

    def sync_check(self, stream=None) -> None:
        self._check(lib().h2o_sync_check(self._h, _stream_ptr(stream)))

    def profile_begin(self, max_steps: int) -> None:
        self._check(lib().h2o_profile_begin(self._h, int(max_steps)))

    def profile_end(self) -> dict:
        """{kernel name: (total device ms, launches)} since profile_begin."""
        K = 8
        names = (ctypes.c_char_p * K)()
        ms = (ctypes.c_double * K)()
        cnt = (ctypes.c_int * K)()
        k = lib().h2o_profile_end(self._h, K, names, ms, cnt)
        if k < 0:
            self._check(k)
        return {names[i].decode(): (ms[i], cnt[i]) for i in range(min(k, K))}

    def kernel_plan(self, T: int) -> list[str]:
        names = (ctypes.c_char_p * 8)()
        k = lib().h2o_kernel_plan(self._h, int(T), names, 8)
        if k < 0:
            self._check(k)
        return [names[i].decode() for i in range(k)]


__all__ = ["H2OCache", "_lib"]
