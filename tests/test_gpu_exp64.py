"""The sampler's float64 exponential (table-driven, with its range fix-up)
against CUDA's exp() on the same device and against the host's exp: a dense
sweep of (-750, 0] (the draw weights' arguments are at most 0), arguments up
to the overflow threshold, the subnormal band and the special values."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200 import s3r                      # noqa: E402

TINY = np.nextafter(0.0, 1.0)                                      # 2^-1074


def _ulps(a, b):
    """Distance of a from b in units of b's last place (0 where equal)."""
    a, b = np.asarray(a), np.asarray(b)
    sp = np.spacing(np.abs(b))
    with np.errstate(invalid="ignore", divide="ignore"):
        d = np.abs(a - b) / sp
    return np.where(a == b, 0.0, d)


def _run(x):
    xd = torch.from_numpy(x).cuda()
    yt = torch.empty_like(xd)
    yr = torch.empty_like(xd)
    s3r.s3r_debug_exp64(xd, yt, yr)
    torch.cuda.synchronize()
    return yt.cpu().numpy(), yr.cpu().numpy()


def test_dense_sweep_of_nonpositive_arguments():
    rng = np.random.default_rng(0)
    x = np.concatenate([-np.linspace(0.0, 745.0, 2_000_001), -rng.uniform(0, 745, 1_000_000),
                        -rng.exponential(1.0, 500_000), -np.logspace(-300, 2.8, 10_000)])
    yt, yr = _run(x)
    normal = yr >= np.finfo(np.float64).tiny
    # normal results: within 2 ulp of CUDA's exp and of the host's
    assert np.max(_ulps(yt[normal], yr[normal])) <= 2.0
    assert np.max(_ulps(yt[normal], np.exp(x[normal]))) <= 2.0
    # subnormal results (about -745 < x < -708.4): one rounding of the scaled value
    sub = ~normal & (yr > 0)
    assert sub.any()
    assert np.max(np.abs(yt[sub] - yr[sub])) <= 2 * TINY


def test_large_and_special_arguments():
    x = np.array([0.0, -0.0, 1e-300, 1.0, 10.0, 100.0, 700.0, 707.5, 708.0, 709.0, 709.78, 710.0, 800.0,
                  -707.0, -707.5, -708.3, -708.5, -740.0, -745.0, -745.2, -746.0, -750.0, -1e10,
                  np.inf, -np.inf, np.nan])
    yt, yr = _run(x)
    host = np.exp(x)
    for xi, a, b, h in zip(x, yt, yr, host):
        if np.isnan(xi):
            assert np.isnan(a)
        elif np.isinf(b) or b == 0.0 or np.isinf(h) or h == 0.0:
            assert a == b or (a == h), (xi, a, b, h)
        elif b >= np.finfo(np.float64).tiny:
            assert _ulps(a, b) <= 2.0 and _ulps(a, h) <= 2.0, (xi, a, b, h)
        else:
            assert abs(a - b) <= 2 * TINY, (xi, a, b)
