"""Decode GEMV edge cases against the float64 oracle, through the C ABI.

The contraction quantizes each column of u once per call to 32-bit fixed point
with a power-of-two scale, so its error is bounded relative to the column's
largest |u|. These tests hold it to the decode tolerance (1e-5 relative,
Frobenius) where that matters most: a few activations 10^3..10^5 times the
rest, heavy-tailed columns, columns of very different magnitude in one call,
extreme exponents. Non-finite activations must come out as an exact IEEE sum
would give them (the oracle's float64 loop): NaN anywhere in a column makes
the column NaN; +-Inf gives +-Inf or NaN per row by the signs of its Inf terms.
Every batch size takes its own path (one or two columns on mma.sync, three or
more on tcgen05), and K = 20480 with two columns is split into two launches.
"""

import ctypes

import numpy as np
import pytest

import oracle
from datagen import make_packed_random, make_u_f32, rng_for
from tests.gpu_common import dev, host, rel_err

pytestmark = pytest.mark.gpu

NTHREADS = min(32, oracle.threads_available())


@pytest.fixture(scope="module")
def lq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_lifted_gemm_b200 as lq
    yield lq
    assert lq.get_device_status() == lq.LQ_OK


def _layer(out, K, seed):
    packed = make_packed_random(out, K, 60, extra=seed)
    s = rng_for(60, 1, seed).uniform(0.01, 0.03, out).astype(np.float32)
    return packed, s


def _check_finite(lq, packed, s, u, tol=1e-5):
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u), NTHREADS)
    assert np.all(np.isfinite(o))
    err = rel_err(o, want)
    assert err <= tol, err
    # every column on its own, too (a small column must not drown in a large one)
    for c in range(u.shape[0]):
        if np.any(want[c] != 0):
            assert rel_err(o[c], want[c]) <= tol, (c, rel_err(o[c], want[c]))
    return o


@pytest.mark.parametrize("K", [12288, 20480])
@pytest.mark.parametrize("scale", [1e3, 1e4, 1e5])
@pytest.mark.parametrize("batch", [1, 2, 4])
def test_outlier_activation(lq, K, scale, batch):
    """One element of each column is `scale` times the typical size."""
    out = 1536
    packed, s = _layer(out, K, K + batch)
    u = make_u_f32(batch, K, 61, extra=K)
    g = rng_for(61, 2, K * 100 + batch)
    for c in range(batch):
        k = int(g.integers(0, K))
        u[c, k] = np.float32(scale * (1 if g.integers(0, 2) else -1))
        if c % 2:  # columns of very different magnitude in one call
            u[c] *= np.float32(1e-3)
    _check_finite(lq, packed, s, u)


@pytest.mark.parametrize("batch", [1, 2, 5])
def test_several_outliers_and_heavy_tails(lq, batch):
    """Log-normal scales (max/rms in the hundreds) plus clustered outliers."""
    out, K = 2048, 12288
    packed, s = _layer(out, K, 7 + batch)
    g = rng_for(62, 1, batch)
    u = (g.standard_normal((batch, K)) * np.exp(2.0 * g.standard_normal((batch, K)))).astype(np.float32)
    u[:, 100:108] = np.float32(3e4)
    _check_finite(lq, packed, s, u)


@pytest.mark.parametrize("magnitude", [1e-30, 1e-40, 1e30])
def test_extreme_exponents(lq, magnitude):
    """Columns of tiny (including subnormal) and huge values scale exactly."""
    out, K, batch = 700, 4096, 2
    packed, s = _layer(out, K, 11)
    u = (make_u_f32(batch, K, 63) * np.float32(magnitude)).astype(np.float32)
    if magnitude < 1e-38:
        assert np.any(u != 0)
    _check_finite(lq, packed, s, u)


@pytest.mark.parametrize("batch", [1, 2, 3])
def test_zero_column(lq, batch):
    out, K = 999, 6144
    packed, s = _layer(out, K, 12)
    u = make_u_f32(batch, K, 64)
    u[batch - 1] = 0.0
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    assert np.all(o[batch - 1] == 0.0)
    want = oracle.contract(packed, s, oracle.to_f64(u))
    assert rel_err(o, want) <= 1e-5


def _assert_ieee_match(o, want):
    """NaN, +Inf and -Inf in the same places; finite entries within 1e-5."""
    assert np.array_equal(np.isnan(o), np.isnan(want))
    assert np.array_equal(np.isposinf(o), np.isposinf(want))
    assert np.array_equal(np.isneginf(o), np.isneginf(want))
    fin = np.isfinite(want)
    if np.any(fin):
        assert rel_err(o[fin], want[fin]) <= 1e-5


@pytest.mark.parametrize("batch,K", [(1, 6144), (2, 6144), (2, 20480), (4, 6144), (6, 20480)])
def test_nonfinite_activations(lq, batch, K):
    """Columns with a NaN, with +Inf, with -Inf, with +Inf and -Inf (which
    gives NaN on rows where their terms oppose, +-Inf where they agree), and
    finite columns beside them."""
    out = 1200
    packed, s = _layer(out, K, 13 + batch)
    s[::97] = 0.0  # 0 * Inf = NaN
    u = make_u_f32(batch, K, 65, extra=batch)
    kinds = ["pinf", "mixed", "nan", "ninf", "finite", "mixed_far"]
    for c in range(batch):
        kind = kinds[c % len(kinds)]
        if kind == "pinf":
            u[c, 5] = np.inf
        elif kind == "ninf":
            u[c, K - 3] = -np.inf
        elif kind == "nan":
            u[c, K // 2] = np.nan
        elif kind == "mixed":
            u[c, 40] = np.inf
            u[c, 41] = -np.inf
        elif kind == "mixed_far":  # +Inf in the first, -Inf in the last part of K
            u[c, 1] = np.inf
            u[c, K - 1] = -np.inf
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u), NTHREADS)
    _assert_ieee_match(o, want)
    if batch >= 2:  # the mixed column really has both outcomes
        assert np.any(np.isnan(o[1])) and np.any(np.isinf(o[1]))


def test_inf_in_second_k_chunk_only(lq):
    """Two columns over K = 20480 (two launches per column pair): an Inf only in
    the second half of K, and Infs of both signs split across the halves."""
    out, K = 1500, 20480
    packed, s = _layer(out, K, 17)
    u = make_u_f32(2, K, 66)
    u[0, K - 10] = -np.inf
    u[1, 3] = np.inf
    u[1, K - 5] = np.inf
    u[1, K - 6] = -np.inf
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u), NTHREADS)
    _assert_ieee_match(o, want)


def test_workspace_reused_without_initialization(lq):
    """One workspace serves calls of different shapes in a row; garbage in it
    before a call changes nothing (every call rewrites what it reads)."""
    import torch
    shapes = [(1000, 4096, 2), (3000, 12288, 1), (1000, 4096, 5), (513, 20480, 2)]
    nbytes = max(lq.gemv_workspace_size(o, K, b) for o, K, b in shapes)
    ws = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    for i, (out, K, batch) in enumerate(shapes):
        packed, s = _layer(out, K, 30 + i)
        u = make_u_f32(batch, K, 67, extra=i)
        o = host(lq.gemv(dev(packed), dev(s), dev(u), workspace=ws))
        want = oracle.contract(packed, s, oracle.to_f64(u), NTHREADS)
        assert rel_err(o, want) <= 1e-5, (out, K, batch)
        ws.fill_(0xFF)


def test_host_pointers_refused(lq):
    """Host memory (pageable or page-locked) where device memory is required is
    refused before any launch; the binding refuses CPU tensors itself."""
    import torch
    out, K, batch = 256, 1024, 1
    packed, s = _layer(out, K, 40)
    u = make_u_f32(batch, K, 68)
    pk, sd, ud = dev(packed), dev(s), dev(u)
    o = torch.empty((batch, out), device="cuda")
    ws = lq.gemv_workspace(out, K, batch)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    s_host = np.ascontiguousarray(s)
    s_pinned = torch.from_numpy(s).pin_memory()
    for bad in (ctypes.c_void_p(s_host.ctypes.data), vp(s_pinned)):
        rc = lq.lib.lq_gemv(vp(pk), bad, out, K, vp(ud), batch, vp(o), vp(ws), ws.numel(), None)
        assert rc == lq.LQ_ERR_INVALID_ARG
    ws_pinned = torch.empty(ws.numel(), dtype=torch.uint8).pin_memory()
    rc = lq.lib.lq_gemv(vp(pk), vp(sd), out, K, vp(ud), batch, vp(o), vp(ws_pinned), ws.numel(), None)
    assert rc == lq.LQ_ERR_INVALID_ARG
    ub = ud.to(torch.bfloat16)
    rc = lq.lib.lq_gemm(vp(pk), ctypes.c_void_p(s_host.ctypes.data), out, K, vp(ub), batch, vp(o), None)
    assert rc == lq.LQ_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        lq.gemv(pk, torch.from_numpy(s), ud)
    with pytest.raises(ValueError):
        lq.gemm(pk, torch.from_numpy(s), ub)
    torch.cuda.synchronize()
    # nothing was launched: the device still computes and reports no error
    got = host(lq.gemv(pk, sd, ud))
    assert rel_err(got, oracle.contract(packed, s, oracle.to_f64(u))) <= 1e-5
