"""The allocation-free eviction entry point (h2o_select_noalloc) against the
eviction inside h2o_step.

h2o_select_noalloc serves callers that cannot call cudaMalloc (plugin hosts
and serving runtimes that only hand out pre-allocated buffers, and paths
where an allocation would synchronise the device): it keeps its scratch in a
static device array instead of a context-owned buffer. Fed the candidate
scores and positions a real step produced, it must reproduce that step's
kept flags, token slots, slot scores and slot positions exactly (selection
is integer/bit-exact work), on two steps in a row; the oracle's selection on
the same candidates must agree, and a call must leave the device's free
memory unchanged. This file is collected
last so that a failure here cannot hide any other test."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_select_noalloc_matches_step_eviction():
    from h2o_kv_cache_step_b200 import H2OCache, synth
    from h2o_kv_cache_step_b200._lib import H2O_ERR_UNSUPPORTED, H2O_OK, lib
    from oracle import oracle

    wl = synth.Workload("noalloc", "bf16", B=2, Hq=8, Hkv=2, d=128, C=192, T=128, N=128 * 4,
                        seed=21, recipe="heavy", hh_frac=0.04)
    cache = H2OCache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.C, torch.bfloat16, max_T=wl.T)
    groups = wl.B * wl.Hkv
    calls = 0
    for c in range(wl.n_chunks):
        _, _, _, pos_before, P, n = cache.get_state()
        scores_before = cache.scores()
        q, k, v = (torch.from_numpy(x).cuda().to(torch.bfloat16) for x in synth.chunk(wl, c))
        cache.step(q, k, v)
        cache.sync_check()
        cand_s, cand_p, kept_step = cache.candidates()
        if n + wl.T <= wl.C:
            continue  # nothing to evict yet; compare on the evicting steps
        # the step's own results
        slots_step = cache.token_slots()
        scores_step = cache.scores()
        pos_step = cache.positions()
        # the allocation-free entry point on the same candidates and pre-step slots
        sc = scores_before.clone()
        ps = pos_before.clone()
        kept = torch.full_like(kept_step, 7)
        ts = torch.full_like(slots_step, -9)
        # outputs of a second call, allocated before it
        sc2, ps2 = scores_before.clone(), pos_before.clone()
        kept2, ts2 = torch.full_like(kept_step, 5), torch.full_like(slots_step, -5)
        stream = torch.cuda.current_stream()
        calls += 1
        rc = lib().h2o_select_noalloc(groups, wl.C, n, wl.T, P, _p(cand_s), _p(cand_p), _p(sc), _p(ps),
                                      _p(kept), _p(ts), ctypes.c_void_p(stream.cuda_stream))
        assert rc == H2O_OK, lib().h2o_last_error(None)
        torch.cuda.synchronize()
        if calls == 1:
            # after the first call on the device, a call leaves the device's
            # free memory exactly as it was: it allocates nothing
            free_before = torch.cuda.mem_get_info()[0]
            rc = lib().h2o_select_noalloc(groups, wl.C, n, wl.T, P, _p(cand_s), _p(cand_p), _p(sc2), _p(ps2),
                                          _p(kept2), _p(ts2), ctypes.c_void_p(stream.cuda_stream))
            assert rc == H2O_OK, lib().h2o_last_error(None)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free_before
            # the replayed call computed the same result
            assert torch.equal(kept2, kept) and torch.equal(ts2, ts)
            # and the oracle's selection on the same candidates agrees
            for grp in range(groups):
                slot = np.concatenate([np.arange(n, dtype=np.int32), np.full(wl.T, -1, np.int32)])
                kept_ref, ts_ref = oracle.select_group(
                    wl.C, wl.T, cand_s.reshape(groups, -1)[grp].double().cpu().numpy(),
                    cand_p.reshape(groups, -1)[grp].long().cpu().numpy(), slot)
                assert np.array_equal(kept_ref, kept.reshape(groups, -1)[grp].cpu().numpy())
                assert np.array_equal(ts_ref, ts.reshape(groups, -1)[grp].cpu().numpy())
        assert torch.equal(kept, kept_step)
        assert torch.equal(ts, slots_step)
        assert torch.equal(ps, pos_step)
        assert torch.equal(sc.view(torch.int32), scores_step.view(torch.int32))
    assert calls >= 2  # two evicting steps in a row

    # sizes beyond the built-in scratch are refused, with a message
    dummy = torch.zeros(16, device="cuda")
    rc = lib().h2o_select_noalloc(64, 8192, 8192, 1, 9000, _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                  _p(dummy), _p(dummy), None)
    assert rc == H2O_ERR_UNSUPPORTED
    assert b"scratch" in lib().h2o_last_error(None)
    cache.close()
