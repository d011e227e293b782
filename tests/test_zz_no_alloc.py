"""lq_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory (code running under CUDA graph capture, serving loops with a fixed
memory pool, plug-ins that only receive tensors), whose scratch is a fixed
array inside the library instead of a caller workspace.

Called through the C ABI (ctypes) twice in a row on fresh inputs, it must give
the results of lq_gemv with a caller workspace, within the decode tolerance of
the other tests (1e-5 relative, Frobenius): both on the mma.sync plan (one and
four columns) and on the tensor-core plan (twelve columns). A shape whose
scratch exceeds the array is refused before any launch. Kept in a file of its
own that pytest collects last; it passes alone in a fresh process and after the
other tests (nothing in it depends on earlier calls).
"""

import ctypes

import numpy as np
import pytest

from datagen import make_packed_random, make_u_f32, rng_for
from tests.gpu_common import dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_lifted_gemm_b200 as lq
    yield lq
    assert lq.get_device_status() == lq.LQ_OK


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("out,K,batch", [(13824, 12288, 1), (3000, 6144, 4), (2048, 4096, 12)])
def test_noalloc_matches_workspace_gemv_twice(lq, out, K, batch):
    import torch
    assert lq.gemv_workspace_size(out, K, batch) <= lq.GEMV_NOALLOC_SCRATCH_BYTES
    packed = make_packed_random(out, K, 80, extra=K + batch)
    s = rng_for(80, 1, out).uniform(0.01, 0.03, out).astype(np.float32)
    pk, sd = dev(packed), dev(s)
    for call in range(2):  # two calls in a row: the array keeps the previous call's contents
        u = dev(make_u_f32(batch, K, 81, extra=call * 100 + batch))
        o = torch.empty((batch, out), dtype=torch.float32, device="cuda")
        rc = lq.lib.lq_gemv_noalloc(_vp(pk), _vp(sd), out, K, _vp(u), batch, _vp(o), None)
        assert rc == lq.LQ_OK, lq.status_str(rc)
        want = lq.gemv(pk, sd, u)
        torch.cuda.synchronize()
        assert rel_err(host(o), host(want)) <= 1e-5, call
    assert lq.get_device_status() == lq.LQ_OK


def test_noalloc_refuses_shapes_beyond_its_array(lq):
    import torch
    out, K, batch = 28672, 20480, 16
    assert lq.gemv_workspace_size(out, K, batch) > lq.GEMV_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(16, dtype=torch.float32, device="cuda")  # never read: refused before any launch
    rc = lq.lib.lq_gemv_noalloc(_vp(x), _vp(x), out, K, _vp(x), batch, _vp(x), None)
    assert rc == lq.LQ_ERR_TOO_LARGE
    assert lq.status_str(rc) == "LQ_ERR_TOO_LARGE"
