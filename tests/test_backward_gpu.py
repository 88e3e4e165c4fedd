"""GPU parity of the step's backward (h2o_backward through the C ABI) against
the fp64 oracle's backward.

The backward differentiates one step's attention for the key set the step
used ("Learning how to Forget", paper page, section "Gradient Computation
Strategy for Sparse Attention": the logged eviction decisions are replayed,
not differentiated). Each case sets a pre-step cache, runs the forward step
on the device for its output and LSE, restores the pre-step cache (the
replay) and compares all five gradients element by element with
``oracle.backward`` on the same values.

Tolerance: max |gpu - ref| <= tol * max(1, max |ref|) per gradient, tol = 1e-4
for fp32 inputs and 2e-2 for bf16 inputs (the acceptance bounds of the
forward output); the achieved errors go to the parity summary."""
import numpy as np
import pytest
import torch

from h2o_kv_cache_step_b200 import H2OCache, synth
from oracle import oracle
from parity_util import ERROR_LOG, TORCH_DTYPE, oracle_state_from_device, to_dev

pytestmark = pytest.mark.gpu

TOL_GRAD = {"fp32": 1e-4, "bf16": 2e-2}


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _compare(name, got, ref, dtype, label):
    got = got.double().cpu().numpy()
    scale = max(1.0, float(np.abs(ref).max()))
    err = float(np.abs(got - ref).max())
    ERROR_LOG.append(dict(case=f"{label} {name}", out_max_abs=err, out_max_ref=float(np.abs(ref).max()),
                          out_rel=err / scale, row_rel=None, lse_max_abs=None, score_rel=None))
    assert err <= TOL_GRAD[dtype] * scale, f"{name}: max abs err {err:.3e} (max |ref| {scale:.3e})"


def run_backward_case(wl, n, P, seed, label, sub=None):
    """Forward on the device from a random pre-step cache with n valid slots,
    then the backward against the restored cache; compare with the oracle.
    sub = (b, g): compare only that (sequence, KV head) group (large sizes)."""
    dtype = wl.dtype
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, TORCH_DTYPE[dtype], max_T=wl.T)
    K, V, S, pos = synth.random_state(wl, n=n, P=P, seed=seed)
    state = (to_dev(K, dtype), to_dev(V, dtype), torch.from_numpy(S).cuda(), torch.from_numpy(pos).cuda())
    cache.set_state(*state, P=P, n=n)
    pre = oracle_state_from_device(cache)
    q, k, v = synth.chunk(wl, 0)
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    cache.step(qd, kd, vd)
    lse = cache.lse()
    cache.sync_check()
    rng = np.random.default_rng(seed + 1)
    dout_np = rng.standard_normal(q.shape).astype(np.float32)
    dout = to_dev(dout_np, dtype)
    # replay: the cache the step saw
    cache.set_state(*state, P=P, n=n)
    dq, dK, dV, dk, dv = cache.backward(qd, kd, vd, lse, dout)
    cache.sync_check()
    # the oracle on the device's exact input values
    qx, kx, vx = (t.double().cpu().numpy() for t in (qd, kd, vd))
    dox = dout.double().cpu().numpy()
    if sub is None:
        ref = oracle.backward(pre, qx, kx, vx, dox, nthreads=8)
        got = (dq, dK, dV, dk, dv)
    else:
        b, g = sub
        G = wl.G
        hs = slice(g * G, (g + 1) * G)
        st = oracle.State(pre.K[b:b + 1, g:g + 1].copy(), pre.V[b:b + 1, g:g + 1].copy(),
                          pre.phi[b:b + 1, g:g + 1].copy(), pre.pos[b:b + 1, g:g + 1].copy(), pre.P)
        ref = oracle.backward(st, qx[b:b + 1, hs], kx[b:b + 1, g:g + 1], vx[b:b + 1, g:g + 1],
                              dox[b:b + 1, hs], nthreads=8)
        got = (dq[b:b + 1, hs], dK[b:b + 1, g:g + 1], dV[b:b + 1, g:g + 1], dk[b:b + 1, g:g + 1],
               dv[b:b + 1, g:g + 1])
    for name, gt, rf in zip(("dq", "dK", "dV", "dk", "dv"), got, ref):
        _compare(name, gt, rf, dtype, label)
    # empty slots get no gradient
    if n < wl.C:
        assert float(dK[:, :, n:].abs().max()) == 0.0 and float(dV[:, :, n:].abs().max()) == 0.0
    cache.close()


@pytest.mark.parametrize("dtype,d,B,Hq,Hkv,C,n,T", [
    ("fp32", 64, 1, 4, 2, 256, 256, 64),      # the tiny workload's shape, full cache
    ("fp32", 128, 2, 4, 2, 100, 37, 33),      # partly filled cache, ragged T
    ("fp32", 64, 1, 2, 2, 40, 0, 17),         # cold start: the chunk alone (MHA)
    ("bf16", 128, 2, 8, 2, 300, 250, 130),    # ragged, GQA 4
    ("bf16", 64, 1, 8, 1, 200, 200, 64),      # d = 64, G = 8
    ("bf16", 128, 1, 4, 4, 128, 128, 256),    # chunk longer than the cache
    ("bf16", 128, 1, 4, 2, 64, 10, 1),        # one token
])
def test_backward_lockstep(dtype, d, B, Hq, Hkv, C, n, T):
    wl = synth.Workload("bwd", dtype, B=B, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * 4, seed=31,
                        recipe="heavy", hh_frac=0.05)
    run_backward_case(wl, n=n, P=max(n, 3 * T) if n else 0, seed=7, label=f"backward {dtype} d{d} C{C} n{n} T{T}")


@pytest.mark.slow
def test_backward_full_size_group():
    """The bench layer's shape (C = 2048 full, T = 1024, 32 / 8 heads): one
    whole KV group through the oracle, all five gradients."""
    wl = synth.WORKLOADS["qwen3-4b-c2048-t1024-n64k"]
    run_backward_case(wl, n=wl.C, P=3 * wl.T, seed=11, label="backward full size c2048 t1024",
                      sub=(0, wl.Hkv // 2))


def test_backward_leaves_the_cache_unchanged():
    wl = synth.Workload("bwd-state", "bf16", B=1, Hq=4, Hkv=2, d=128, C=64, T=32, N=128, seed=3)
    cache = H2OCache(1, 4, 2, 128, 64, torch.bfloat16, max_T=32)
    K, V, S, pos = synth.random_state(wl, n=50, P=100, seed=2)
    cache.set_state(to_dev(K, "bf16"), to_dev(V, "bf16"), torch.from_numpy(S).cuda(),
                    torch.from_numpy(pos).cuda(), P=100, n=50)
    before = cache.get_state()
    q, k, v = (to_dev(x, "bf16") for x in synth.chunk(wl, 0))
    lse = torch.zeros((1, 4, 32), dtype=torch.float32, device="cuda")
    cache.backward(q, k, v, lse, torch.ones_like(q))
    after = cache.get_state()
    for a, b in zip(before[:4], after[:4]):
        assert torch.equal(a, b)
    assert before[4:] == after[4:]
