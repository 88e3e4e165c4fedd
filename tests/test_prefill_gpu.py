"""h2o_prefill (several steps in one call) against the same steps made one
h2o_step call at a time, through the C ABI.

Both run the same kernels on the same values; h2o_prefill only lets a step's
attention to its own chunk start while the previous step's eviction still
runs, so every result must be bit-identical: the outputs of every chunk, the
cache (keys, values, scores, positions, valid count, P) and the last chunk's
LSE. The per-step results themselves are checked against the oracle by the
lockstep parity tests."""
import pytest
import torch

from h2o_kv_cache_step_b200 import H2OCache, synth
from h2o_kv_cache_step_b200._lib import H2O_POLICY_INSERT_ALWAYS, H2O_POLICY_NORMALIZED, H2OError
from parity_util import TORCH_DTYPE, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _stacked(wl):
    qs, ks, vs = [], [], []
    for c in range(wl.n_chunks):
        q, k, v = synth.chunk(wl, c)
        qs.append(to_dev(q, wl.dtype))
        ks.append(to_dev(k, wl.dtype))
        vs.append(to_dev(v, wl.dtype))
    return torch.stack(qs), torch.stack(ks), torch.stack(vs)


def _run_both(wl, policy=None):
    qs, ks, vs = _stacked(wl)
    caches = []
    for _ in range(2):
        c = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, TORCH_DTYPE[wl.dtype], max_T=wl.T)
        if policy is not None:
            c.set_policy(policy)
        caches.append(c)
    stepwise, fused = caches
    outs_step = torch.stack([stepwise.step(qs[i], ks[i], vs[i]) for i in range(wl.n_chunks)])
    outs_fused = fused.prefill(qs, ks, vs)
    torch.cuda.synchronize()
    stepwise.sync_check()
    fused.sync_check()
    assert torch.equal(outs_step, outs_fused)
    a, b = stepwise.get_state(), fused.get_state()
    for x, y in zip(a[:4], b[:4]):
        assert torch.equal(x, y)
    assert a[4:] == b[4:]
    assert torch.equal(stepwise.lse(), fused.lse())
    for c in caches:
        c.close()


@pytest.mark.parametrize("dtype,d,B,Hq,Hkv,C,T,chunks", [
    ("bf16", 128, 1, 8, 2, 384, 128, 8),     # fills, then evicts every step (tensor cores)
    ("bf16", 128, 2, 8, 2, 300, 200, 5),     # ragged T and C
    ("bf16", 64, 1, 8, 1, 1100, 130, 10),    # d = 64; the SDPA splits its units once the cache is long
    ("bf16", 128, 1, 4, 2, 100, 300, 3),     # chunk longer than the cache
    ("fp32", 64, 1, 4, 2, 256, 64, 6),       # CUDA-core path (steps in sequence)
    ("bf16", 128, 1, 8, 2, 64, 4, 8),        # short chunks: decode path
])
def test_prefill_matches_steps(dtype, d, B, Hq, Hkv, C, T, chunks):
    wl = synth.Workload("prefill", dtype, B=B, Hq=Hq, Hkv=Hkv, d=d, C=C, T=T, N=T * chunks, seed=41,
                        recipe="heavy", hh_frac=0.05)
    _run_both(wl)


@pytest.mark.parametrize("policy", [H2O_POLICY_NORMALIZED, H2O_POLICY_INSERT_ALWAYS])
def test_prefill_matches_steps_other_policies(policy):
    wl = synth.Workload("prefill-pol", "bf16", B=1, Hq=8, Hkv=2, d=128, C=256, T=96, N=96 * 6, seed=43,
                        recipe="heavy", hh_frac=0.05)
    _run_both(wl, policy)


@pytest.mark.slow
def test_prefill_matches_steps_full_size():
    """The bench layer's shape for 12 chunks: the cache fills in two steps,
    then every step evicts (C = 2048, T = 1024, 32 / 8 heads)."""
    wl = synth.WORKLOADS["qwen3-4b-c2048-t1024-n64k"].with_(N=12 * 1024)
    _run_both(wl)


def test_prefill_rejects_bad_arguments():
    cache = H2OCache(1, 4, 2, 64, 32, torch.bfloat16, max_T=8)
    q = torch.zeros((2, 1, 4, 8, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((2, 1, 2, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        cache.prefill(q[0], k[0], k[0])  # not [nchunks, B, H, T, d]
    with pytest.raises(ValueError):
        cache.prefill(q, k[:, :, :1], k)  # wrong KV head count
    from h2o_kv_cache_step_b200._lib import lib
    assert lib().h2o_prefill(cache._h, q.data_ptr(), k.data_ptr(), k.data_ptr(), q.data_ptr(), 8, 0, None) != 0
    with pytest.raises(H2OError):
        cache._check(lib().h2o_prefill(cache._h, q.data_ptr(), k.data_ptr(), k.data_ptr(), None, 8, 2, None))
    cache.close()
