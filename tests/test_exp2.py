"""The FMA-pipe 2^x the tensor-core kernels use for part of their softmax
exponentials (range reduction to [-1/2, 1/2] + fitted polynomial, see
csrc/gen_exp2_poly.py), checked against float64 exp2 and against the
hardware ex2.approx on the device."""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _gen():
    p = os.path.join(ROOT, "h2o_kv_cache_step_b200", "csrc", "gen_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", p)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_fit_error_bounds_cpu():
    g = _gen()
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    for deg, bound in ((3, 8e-5), (4, 3e-6)):
        c = g.fit(deg)
        err = np.abs(g.horner32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
        assert err < bound, (deg, err)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_device_exp2_variants():
    from h2o_kv_cache_step_b200._lib import H2O_OK, lib
    x = np.concatenate([np.linspace(-140, 9, 400001), [-126.0, -125.0, -124.999, -0.5, 0.0, 0.5, 1e-8, -1e-8]])
    xd = torch.tensor(x, dtype=torch.float32, device="cuda")
    y3, y4, ym = (torch.empty_like(xd) for _ in range(3))
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib().h2o_selftest_exp2(p(xd), p(y3), p(y4), p(ym), xd.numel(), None) == H2O_OK
    torch.cuda.synchronize()
    xf = xd.cpu().numpy().astype(np.float64)
    ref = np.exp2(xf)
    ok = xf >= -125.0
    for y, bound in ((y3, 8e-5), (y4, 3e-6), (ym, 2e-6)):
        yy = y.cpu().numpy().astype(np.float64)
        rel = np.abs(yy[ok] / ref[ok] - 1)
        assert rel.max() < bound, (bound, rel.max(), xf[ok][np.argmax(rel)])
    # below 2^-125 the polynomial versions flush to zero (ex2.approx.ftz
    # below 2^-126)
    assert (y3.cpu().numpy()[xf < -125.0] == 0).all()
    assert (y4.cpu().numpy()[xf < -125.0] == 0).all()
    assert (ym.cpu().numpy()[xf < -126.0] == 0).all()
