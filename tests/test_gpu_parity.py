"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Tolerances: sign packing is bit-exact; the fp32 lift within 1e-6 relative; the
decode GEMV within 1e-5 relative (Frobenius over [batch][out]); the prefill
GEMM within 1e-5 of the oracle fed the same bf16 u (fp32 accumulation only)
and within 5e-3 of the full-precision layer (bf16 rounding of u). Integer
valued inputs make every sum exact, so the GPU must then match bit for bit.
Full-size layers are checked on sampled rows that the oracle computes one by
one, plus properties that hold at any size.
"""

import os

import numpy as np
import pytest

import oracle
from datagen import CONFIGS, make_layer, make_packed_random, make_signs_pm1, make_u_bf16, make_u_f32, rng_for
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


def _sample_rows(out, n, seed):
    g = rng_for(77, 9, seed)
    rows = np.unique(np.concatenate([g.choice(out, size=min(n, out), replace=False), [0, out - 1]]))
    return rows.astype(np.int64)


# ------------------------------------------------------------------ pack / unpack

@pytest.mark.parametrize("rows,K", [(1, 32), (37, 288), (512, 1536), (1000, 12288)])
def test_pack_unpack_bit_exact(lq, rows, K):
    signs = make_signs_pm1(rows, K, cfg_index=50, extra=K)
    packed = lq.pack_signs(dev(signs))
    assert np.array_equal(host(packed), oracle.pack_signs(signs))
    back = lq.unpack_signs(packed, K)
    assert np.array_equal(host(back), signs)


def test_pack_adversarial_patterns(lq):
    K = 96
    pats = np.stack([-np.ones(K), np.ones(K), np.tile([1, -1], K // 2), np.tile([-1, 1], K // 2),
                     np.where(np.arange(K) % 32 == 31, 1, -1), np.where(np.arange(K) % 32 == 0, 1, -1)])
    signs = pats.astype(np.int8)
    assert np.array_equal(host(lq.pack_signs(dev(signs))), oracle.pack_signs(signs))
    words = make_packed_random(8, 1024, cfg_index=51)
    assert np.array_equal(host(lq.unpack_signs(dev(words), 1024)), oracle.unpack_signs(words, 1024))


# ------------------------------------------------------------------ lift

def _oracle_u(L):
    a = oracle.to_f64(L.a, L.a_dtype)
    t = None if L.tinv is None else oracle.to_f64(L.tinv)
    return oracle.lift(oracle.whiten(a, t), oracle.to_f64(L.M), L.cfg.K)


def _gpu_u(lq, L, u_dtype="f32"):
    t = None if L.tinv is None else dev(L.tinv)
    return lq.lift_activations(dev(L.a), dev(L.M), L.cfg.K, tinv=t, u_dtype=u_dtype)


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("tiny", 4), ("decode_lq24_10", 1), ("decode_lq20_8", 16),
                                        ("decode_lq20_8", 3), ("sweep_lq19_8", 1)])
def test_lift_fp32(lq, name, batch):
    L = make_layer(CONFIGS[name], batch, packed=False)
    u = host(_gpu_u(lq, L))
    want = _oracle_u(L)
    assert rel_err(u, want) <= 1e-6
    assert np.max(np.abs(u - want)) <= 1e-5 * np.max(np.abs(want))


def _bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("batch", [40, 100])
def test_lift_bf16_prefill_tiles(lq, batch):
    """Prefill variant (32-token tiles, ragged last tile), bf16 output."""
    L = make_layer(CONFIGS["decode_lq24_10"], batch, packed=False)
    u = oracle.to_f64(host(_gpu_u(lq, L, "bf16")), "bf16")
    want = _oracle_u(L)
    assert np.all(np.abs(u - want) <= _bf16_ulp(want) + 1e-6 * np.max(np.abs(want)))
    assert rel_err(u, want) <= 3e-3


def test_lift_padding_and_small_blocks(lq):
    """in=9, d=3, D=5: K = 32 with 17 padded zeros; 3x3 whitening blocks."""
    g = rng_for(60, 0)
    a = g.standard_normal((2, 9)).astype(np.float32)
    M = g.standard_normal((3, 5)).astype(np.float32)
    tinv = g.standard_normal((3, 3, 3)).astype(np.float32)
    for t in (None, tinv):
        u = host(lq.lift_activations(dev(a), dev(M), 32, tinv=None if t is None else dev(t)))
        want = oracle.lift(oracle.whiten(oracle.to_f64(a), None if t is None else oracle.to_f64(t)),
                           oracle.to_f64(M), 32)
        assert np.all(u[:, 15:] == 0.0)
        assert rel_err(u, want) <= 1e-6


@pytest.mark.parametrize("in_dim,d,D,batch,u_dtype", [
    (5120, 10, 24, 200, "bf16"),  # LQ-24/10 channels: runs of 120 straddling 128-wide blocks, ragged tokens
    (1024, 8, 20, 130, "f32"),    # runs aligned to the whitening blocks, fp32 output, 2-token last tile
    (2048, 16, 40, 64, "bf16"),   # smallest batch of the tensor-core path
    (1280, 20, 40, 300, "bf16"),  # d = 20: runs of 6 lift blocks
    (384, 8, 9, 70, "bf16"),      # odd D (scalar stores), zero tail of 16 lifted entries
    (384, 8, 9, 100, "f32"),      # same with fp32 output
    (640, 5, 9, 128, "bf16"),     # d = 5: runs of 25 lift blocks (125 channels)
])
def test_lift_tensor_core_prefill(lq, in_dim, d, D, batch, u_dtype):
    """Prefill lift with the whitening on tcgen05 (bf16 activations, 128-wide blocks)."""
    from datagen.inputs import bf16_bits_from_f32
    g = rng_for(62, in_dim, d * 1000 + batch)
    a = bf16_bits_from_f32(g.standard_normal((batch, in_dim)).astype(np.float32))
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    tinv = (g.standard_normal((in_dim // 128, 128, 128)) / np.sqrt(128)).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    u = host(lq.lift_activations(dev(a), dev(M), K, tinv=dev(tinv), u_dtype=u_dtype))
    want = oracle.lift(oracle.whiten(oracle.to_f64(a, "bf16"), oracle.to_f64(tinv)), oracle.to_f64(M), K)
    kreal = (in_dim // d) * D
    if u_dtype == "bf16":
        u = oracle.to_f64(u, "bf16")
        assert np.all(np.abs(u - want) <= _bf16_ulp(want) + 1e-6 * np.max(np.abs(want)))
    else:
        assert rel_err(u, want) <= 1e-6
        assert np.max(np.abs(u - want)) <= 1e-5 * np.max(np.abs(want))
    assert np.all(u[:, kreal:] == 0.0)


@pytest.mark.parametrize("in_dim,d,D,tblk,batch,a_bf16,u_dtype", [
    (1024, 16, 48, 256, 3, True, "f32"),   # two float4 per lane of a T row, second M column per lane
    (960, 10, 40, 96, 2, False, "f32"),    # d-blocks straddling whitening blocks
    (600, 5, 9, 20, 16, True, "f32"),      # narrow blocks, full decode batch, padded lifted tail
    (600, 5, 9, 20, 2, True, "bf16"),      # bf16 lifted output from the decode path
    (512, 16, 64, 0, 4, False, "f32"),     # T = identity
    (1280, 20, 40, 128, 2, True, "f32"),   # d > 16: the shared-memory decode kernel
    (960, 10, 24, 96, 70, True, "bf16"),   # prefill tiles: blocks straddling 96-wide whitening blocks, ragged tokens
    (1024, 8, 20, 64, 130, False, "bf16"), # prefill tiles, 64-wide whitening blocks
    (1024, 8, 20, 128, 33, True, "f32"),   # prefill tiles with fp32 output
    (768, 6, 14, 256, 40, True, "bf16"),   # 256-wide whitening blocks: the shared-memory prefill kernel
])
def test_lift_decode_shapes(lq, in_dim, d, D, tblk, batch, a_bf16, u_dtype):
    from datagen.inputs import bf16_bits_from_f32
    g = rng_for(61, in_dim, d * 1000 + batch)
    a32 = g.standard_normal((batch, in_dim)).astype(np.float32)
    a = bf16_bits_from_f32(a32) if a_bf16 else a32
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    tinv = (g.standard_normal((in_dim // tblk, tblk, tblk)) / np.sqrt(tblk)).astype(np.float32) if tblk else None
    K = oracle.lifted_dim(in_dim, d, D)
    u = host(lq.lift_activations(dev(a), dev(M), K, tinv=None if tinv is None else dev(tinv), u_dtype=u_dtype))
    want = oracle.lift(oracle.whiten(oracle.to_f64(a, "bf16" if a_bf16 else "f32"),
                                     None if tinv is None else oracle.to_f64(tinv)), oracle.to_f64(M), K)
    kreal = (in_dim // d) * D
    if u_dtype == "bf16":
        u = oracle.to_f64(u, "bf16")
        assert np.all(np.abs(u - want) <= _bf16_ulp(want) + 1e-6 * np.max(np.abs(want)))
    else:
        assert rel_err(u, want) <= 1e-6
    assert np.all(u[:, kreal:] == 0.0)


# ------------------------------------------------------------------ decode GEMV

@pytest.mark.parametrize("batch", [1, 4])
def test_tiny_layer_full_path(lq, batch):
    L = make_layer(CONFIGS["tiny"], batch)
    u = _gpu_u(lq, L)
    o = host(lq.gemv(dev(L.packed), dev(L.s), u))
    _, want = oracle.forward(L.packed, L.s, oracle.to_f64(L.a), None, oracle.to_f64(L.M), L.cfg.K)
    assert rel_err(o, want) <= 1e-5


@pytest.mark.parametrize("out,K,batch", [(1000, 1536, 1), (1000, 1536, 3), (33, 1632, 16), (1, 32, 1),
                                         (4097, 20480, 2), (700, 16384 + 1024, 1),
                                         # many two-column passes, K chunks, ragged rows
                                         (1000, 3072, 5), (777, 4096, 6), (513, 2048, 8), (2000, 8192, 9),
                                         (300, 20480, 11), (1500, 12288, 16)])
def test_gemv_ragged_vs_oracle(lq, out, K, batch):
    packed = make_packed_random(out, K, 52, extra=K + out)
    s = rng_for(52, 1, out).uniform(0.01, 0.03, out).astype(np.float32)
    u = make_u_f32(batch, K, 52, extra=K)
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u), NTHREADS)
    assert rel_err(o, want) <= 1e-5


def test_gemv_integer_inputs_exact(lq):
    g = rng_for(53, 5)
    out, K, batch = 777, 3072, 5
    packed = make_packed_random(out, K, 53)
    s = np.ones(out, dtype=np.float32)
    u = g.integers(-8, 9, size=(batch, K)).astype(np.float32)
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u))
    assert np.array_equal(o.astype(np.float64), want)


@pytest.mark.parametrize("out,K,batch", [(513, 4096, 8), (1001, 6144, 16)])
def test_gemv_integer_inputs_exact_wide(lq, out, K, batch):
    """Integer-valued u through several two-column passes: every sum is exact."""
    g = rng_for(53, 6, batch)
    packed = make_packed_random(out, K, 53, extra=batch)
    s = np.ones(out, dtype=np.float32)
    u = g.integers(-100, 101, size=(batch, K)).astype(np.float32)
    o = host(lq.gemv(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u))
    assert np.array_equal(o.astype(np.float64), want)


@pytest.mark.parametrize("D", [12, 16])
def test_gemv_exhaustive_codebook(lq, D):
    """One block, one row per sign pattern y in {+-1}^D: every codeword's output."""
    d = 8
    rows = 1 << D
    packed = np.arange(rows, dtype=np.uint32).reshape(rows, 1)   # row r = pattern r, K = 32
    g = rng_for(54, 2, D)
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    a = g.standard_normal((1, d)).astype(np.float32)
    s = np.ones(rows, dtype=np.float32)
    u = lq.lift_activations(dev(a), dev(M), 32)
    o = host(lq.gemv(dev(packed), dev(s), u))
    _, want = oracle.forward(packed, s, oracle.to_f64(a), None, oracle.to_f64(M), 32)
    assert rel_err(o, want) <= 1e-5
    # codeword identity: o[r] = (M y_r) . a for every pattern (dense reconstruction route)
    want2 = oracle.dense_route(packed, s, oracle.to_f64(M), oracle.to_f64(a), 32)
    assert rel_err(o, want2) <= 1e-5


def test_decode_lq24_10_full_size(lq):
    L = make_layer(CONFIGS["decode_lq24_10"], 1)
    u = _gpu_u(lq, L)
    o = host(lq.gemv(dev(L.packed), dev(L.s), u))
    _, want = oracle.forward(L.packed, L.s, oracle.to_f64(L.a, "bf16"), oracle.to_f64(L.tinv),
                             oracle.to_f64(L.M), L.cfg.K, NTHREADS)
    assert rel_err(o, want) <= 1e-5


@pytest.mark.parametrize("batch", [1, 2, 3, 4, 8, 16])  # three columns: the tensor-core path at this size
def test_decode_lq20_8_sampled_rows(lq, batch):
    L = make_layer(CONFIGS["decode_lq20_8"], batch)
    u = _gpu_u(lq, L)
    o = host(lq.gemv(dev(L.packed), dev(L.s), u))
    uref = _oracle_u(L)
    rows = _sample_rows(L.cfg.out, 384, batch)
    want = oracle.contract_rows(L.packed, L.s, uref, rows)
    assert rel_err(o[:, rows], want) <= 1e-5
    # whole-output property: E[o_r^2] = s_r^2 |u|^2 for iid signs
    ratio = np.mean((o / L.s[None, :]) ** 2, axis=1) / np.sum(uref ** 2, axis=1)
    assert np.all(np.abs(ratio - 1) < 0.05)


@pytest.mark.parametrize("D", [16, 19, 20, 22, 24])
def test_sweep_decode_sampled_rows(lq, D):
    L = make_layer(CONFIGS[f"sweep_lq{D}_8"], 1)
    u = _gpu_u(lq, L)
    o = host(lq.gemv(dev(L.packed), dev(L.s), u))
    rows = _sample_rows(L.cfg.out, 512, D)
    want = oracle.contract_rows(L.packed, L.s, _oracle_u(L), rows)
    assert rel_err(o[:, rows], want) <= 1e-5


# ------------------------------------------------------------------ Kronecker-factored whitening

def _kron_case(in_dim, n1, d, D, batch, a_dtype, seed):
    from datagen import make_kron_factors
    from datagen.inputs import bf16_bits_from_f32
    g = rng_for(61, seed, batch)
    a32 = g.standard_normal((batch, in_dim)).astype(np.float32)
    a = bf16_bits_from_f32(a32) if a_dtype == "bf16" else a32
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    kf = make_kron_factors(in_dim, n1, d, 61, seed)
    return a, M, kf


def _kron_oracle_u(a, a_dtype, M, kf, d, K, with_r=True):
    ap = oracle.whiten_kron(oracle.to_f64(a, a_dtype), oracle.to_f64(kf.r1) if with_r else None,
                            oracle.to_f64(kf.q1), oracle.to_f64(kf.q2), oracle.to_f64(kf.r2) if with_r else None, d)
    return oracle.lift(ap, oracle.to_f64(M), K)


@pytest.mark.parametrize("in_dim,n1,d,D,batch,a_dtype,u_dtype,with_r", [
    (640, 8, 10, 24, 1, "f32", "f32", True),      # clusters of 8 CTAs, one row of X each (padded to two)
    (640, 8, 10, 24, 3, "f32", "f32", False),     # no diagonal factors
    (5120, 64, 10, 24, 1, "bf16", "f32", True),   # LQ-24/10 decode layer, 64 x 80 factors
    (5120, 64, 10, 24, 16, "bf16", "f32", True),
    (8192, 64, 8, 20, 2, "bf16", "f32", True),    # LQ-20/8 layer, 64 x 128 factors
    (70, 7, 5, 18, 2, "f32", "f32", True),        # odd n1: one CTA per token; n2 = 10 padded; K tail of 4
    (70, 7, 5, 18, 40, "f32", "f32", True),       # odd n1, 4 tokens per CTA: the narrow multi-token tiles
    (48, 8, 4, 8, 3, "f32", "f32", True),         # d-blocks straddle rows of X; clusters of 4
    (640, 8, 10, 24, 70, "bf16", "bf16", True),   # 4 tokens per cluster, ragged last cluster, bf16 output
    (5120, 64, 10, 24, 40, "bf16", "bf16", True), # prefill-sized batch on the LQ-24/10 layer
    # prefill on the tensor cores (bf16 in and out, 64 tokens or more)
    (5120, 64, 10, 24, 300, "bf16", "bf16", True),  # 64 x 80 factors, ragged last 128-token tile
    (8192, 64, 8, 20, 130, "bf16", "bf16", True),   # 64 x 128 factors, d = 8 blocks
    (5120, 64, 10, 24, 200, "bf16", "bf16", False), # no diagonal factors
    (4096, 64, 8, 16, 70, "bf16", "bf16", True),    # 64 x 64 factors, D = 2 d: K = 2 in exactly
])
def test_lift_kron(lq, in_dim, n1, d, D, batch, a_dtype, u_dtype, with_r):
    """Lift with T^{-1} = diag(r2) (Q1 kron Q2) diag(r1) against the oracle."""
    K = oracle.lifted_dim(in_dim, d, D)
    a, M, kf = _kron_case(in_dim, n1, d, D, batch, a_dtype, 1)
    u = host(lq.lift_activations_kron(dev(a), dev(kf.q1), dev(kf.q2), dev(M), K,
                                      r1=dev(kf.r1) if with_r else None, r2=dev(kf.r2) if with_r else None,
                                      u_dtype=u_dtype))
    want = _kron_oracle_u(a, a_dtype, M, kf, d, K, with_r)
    if u_dtype == "bf16":
        u = oracle.to_f64(u, "bf16")
        assert np.all(np.abs(u - want) <= _bf16_ulp(want) + 1e-6 * np.max(np.abs(want)))
    else:
        assert rel_err(u, want) <= 1e-6
        assert np.max(np.abs(u - want)) <= 1e-5 * np.max(np.abs(want))
    k0 = in_dim // d * D
    assert np.all(u[:, k0:] == 0.0)


def test_lift_kron_persistent_groups(lq):
    """1200 tokens in groups of 4: more groups than resident CTAs, so each
    persistent CTA loops over several groups with its factors kept."""
    in_dim, n1, d, D, batch = 640, 8, 10, 24, 1200
    K = oracle.lifted_dim(in_dim, d, D)
    a, M, kf = _kron_case(in_dim, n1, d, D, batch, "f32", 3)
    u = host(lq.lift_activations_kron(dev(a), dev(kf.q1), dev(kf.q2), dev(M), K, r1=dev(kf.r1), r2=dev(kf.r2)))
    want = _kron_oracle_u(a, "f32", M, kf, d, K)
    assert rel_err(u, want) <= 1e-6
    assert np.max(np.abs(u - want)) <= 1e-5 * np.max(np.abs(want))


def test_lift_kron_then_gemv_vs_oracle(lq):
    """LQ-24/10 decode step with the Kronecker whitening: lift, then the GEMV."""
    L = make_layer(CONFIGS["decode_lq24_10"], 1)
    K = L.cfg.K
    a, M, kf = _kron_case(L.cfg.in_dim, 64, L.cfg.d, L.cfg.D, 1, "bf16", 2)
    u = lq.lift_activations_kron(dev(a), dev(kf.q1), dev(kf.q2), dev(M), K, r1=dev(kf.r1), r2=dev(kf.r2))
    o = host(lq.gemv(dev(L.packed), dev(L.s), u))
    rows = _sample_rows(L.cfg.out, 512, 11)
    want = oracle.contract_rows(L.packed, L.s, _kron_oracle_u(a, "bf16", M, kf, L.cfg.d, K), rows)
    assert rel_err(o[:, rows], want) <= 1e-5


# ------------------------------------------------------------------ one-call decode step

def _fused(lq, L):
    t = None if L.tinv is None else dev(L.tinv)
    return lq.lift_gemv(dev(L.a), dev(L.M), dev(L.packed), dev(L.s), L.cfg.K, tinv=t)


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("tiny", 2), ("tiny", 3), ("decode_lq24_10", 1),
                                        ("decode_lq24_10", 2), ("decode_lq20_8", 1), ("sweep_lq19_8", 1),
                                        ("decode_lq20_8", 4)])
def test_fused_step_equals_two_calls(lq, name, batch):
    """lq_lift_gemv gives exactly the results of lq_lift_activations followed by lq_gemv."""
    L = make_layer(CONFIGS[name], batch)
    u_f, o_f = _fused(lq, L)
    u = _gpu_u(lq, L)
    o = lq.gemv(dev(L.packed), dev(L.s), u)
    assert np.array_equal(host(u_f), host(u))
    assert np.array_equal(host(o_f), host(o))


def _pinned(x):
    import torch
    t = dev(x).cpu()
    return t.pin_memory()


@pytest.mark.parametrize("name,batch", [("tiny", 3), ("decode_lq24_10", 1), ("decode_lq20_8", 4),
                                        ("decode_lq20_8", 16)])
def test_fused_step_zero_copy(lq, name, batch):
    """Activations read from, and outputs written to, pinned host memory by the
    kernels themselves: identical to the all-device call (batch 16 also splits K
    over launches, so the GEMV accumulates into host memory)."""
    import torch
    L = make_layer(CONFIGS[name], batch)
    u_d, o_d = _fused(lq, L)
    a_h = _pinned(L.a)
    o_h = torch.full((batch, L.cfg.out), float("nan"), dtype=torch.float32).pin_memory()
    t = None if L.tinv is None else dev(L.tinv)
    u_z, o_z = lq.lift_gemv(a_h, dev(L.M), dev(L.packed), dev(L.s), L.cfg.K, tinv=t, out=o_h)
    torch.cuda.synchronize()
    assert o_z.data_ptr() == o_h.data_ptr()
    assert np.array_equal(host(u_z), host(u_d))
    assert np.array_equal(o_h.numpy(), host(o_d))


def test_fused_step_rejects_pageable_host(lq):
    """Pageable host memory is refused before any launch (binding and C ABI)."""
    import ctypes
    import torch
    L = make_layer(CONFIGS["tiny"], 1)
    a_p = torch.from_numpy(np.ascontiguousarray(L.a))
    with pytest.raises(ValueError):
        lq.lift_gemv(a_p, dev(L.M), dev(L.packed), dev(L.s), L.cfg.K)
    u = torch.empty((1, L.cfg.K), dtype=torch.float32, device="cuda")
    o = torch.empty((1, L.cfg.out), dtype=torch.float32, device="cuda")
    M, pk, s = dev(L.M), dev(L.packed), dev(L.s)
    d, D = L.M.shape
    ws = lq.gemv_workspace(L.cfg.out, L.cfg.K, 1)
    rc = lq.lib.lq_lift_gemv(ctypes.c_void_p(a_p.data_ptr()), lq.LQ_F32, 1, L.cfg.in_dim, None, 0,
                             ctypes.c_void_p(M.data_ptr()), d, D, ctypes.c_void_p(pk.data_ptr()),
                             ctypes.c_void_p(s.data_ptr()), L.cfg.out, L.cfg.K, ctypes.c_void_p(u.data_ptr()),
                             ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert rc == lq.LQ_ERR_INVALID_ARG


def test_fused_step_vs_oracle_alternating_layers(lq):
    """One-call decode step against the oracle, alternating a small and a large
    layer (32 and 148 CTAs)."""
    small = make_layer(CONFIGS["tiny"], 2)
    big = make_layer(CONFIGS["decode_lq24_10"], 1)
    _, want_small = oracle.forward(small.packed, small.s, oracle.to_f64(small.a), None, oracle.to_f64(small.M),
                                   small.cfg.K)
    rows = _sample_rows(big.cfg.out, 512, 5)
    want_big = oracle.contract_rows(big.packed, big.s, _oracle_u(big), rows)
    for _ in range(3):
        _, o = _fused(lq, small)
        assert rel_err(host(o), want_small) <= 1e-5
        _, o = _fused(lq, big)
        assert rel_err(host(o)[:, rows], want_big) <= 1e-5


# ------------------------------------------------------------------ prefill GEMM

@pytest.mark.parametrize("out,K,tokens", [(300, 1536, 300), (128, 64, 256), (129, 1568, 7), (1, 32, 1),
                                          (517, 4096 + 32, 513),
                                          # 64-token tiles (A stages in TMEM): aligned and ragged rows, K split
                                          (1000, 12288, 64), (77, 4096, 50)])
def test_gemm_isolated_vs_oracle(lq, out, K, tokens):
    packed = make_packed_random(out, K, 55, extra=K + out)
    s = rng_for(55, 1, out).uniform(0.01, 0.03, out).astype(np.float32)
    u = make_u_bf16(tokens, K, 55, extra=K + tokens)
    o = host(lq.gemm(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u, "bf16"), NTHREADS)
    assert rel_err(o, want) <= 1e-5


@pytest.mark.parametrize("tokens", [300, 64, 33])
def test_gemm_integer_inputs_exact(lq, tokens):
    """Integer-valued u: bit-exact for 256-token tiles (A in shared memory) and
    64-token tiles (A in TMEM, K split in two)."""
    g = rng_for(56, 5, tokens)
    out, K = 260, 2048
    packed = make_packed_random(out, K, 56)
    s = np.ones(out, dtype=np.float32)
    from datagen import bf16_bits_from_f32
    u = bf16_bits_from_f32(g.integers(-8, 9, size=(tokens, K)).astype(np.float32))
    o = host(lq.gemm(dev(packed), dev(s), dev(u)))
    want = oracle.contract(packed, s, oracle.to_f64(u, "bf16"), NTHREADS)
    assert np.array_equal(o.astype(np.float64), want)


def test_prefill_lq24_10_full_size_sampled(lq):
    L = make_layer(CONFIGS["prefill_lq24_10"], 2048)
    u = _gpu_u(lq, L, "bf16")
    o = host(lq.gemm(dev(L.packed), dev(L.s), u))
    rows = _sample_rows(L.cfg.out, 96, 3)
    toks = np.sort(rng_for(77, 8).choice(2048, size=192, replace=False))
    # contraction alone: oracle fed the same bf16 u
    u_host = oracle.to_f64(host(u), "bf16")
    want_c = oracle.contract_rows(L.packed, L.s, u_host[toks], rows)
    assert rel_err(o[np.ix_(toks, rows)], want_c) <= 1e-5
    # whole layer against full-precision u
    a = oracle.to_f64(L.a, "bf16")[toks]
    uref = oracle.lift(oracle.whiten(a, oracle.to_f64(L.tinv)), oracle.to_f64(L.M), L.cfg.K)
    want = oracle.contract_rows(L.packed, L.s, uref, rows)
    assert rel_err(o[np.ix_(toks, rows)], want) <= 5e-3


@pytest.mark.parametrize("D", [16, 19, 20, 22, 24])
def test_sweep_prefill_b64(lq, D):
    """Every configured bit-width at 64 tokens (the shapes the benchmark times)."""
    L = make_layer(CONFIGS[f"sweep_lq{D}_8"], 64)
    u = _gpu_u(lq, L, "bf16")
    o = host(lq.gemm(dev(L.packed), dev(L.s), u))
    rows = _sample_rows(L.cfg.out, 256, D)
    want = oracle.contract_rows(L.packed, L.s, _oracle_u(L), rows)
    assert rel_err(o[:, rows], want) <= 5e-3


# ------------------------------------------------------------------ encoder

def _patterns_from_words(words, rows, nblk, D):
    """Per-block sign patterns (bit j <=> +1) read back from packed rows: block b
    of a row occupies bits [b D, (b + 1) D), 32 per word, least significant first."""
    bits = np.unpackbits(np.ascontiguousarray(words).view(np.uint8).reshape(rows, -1), axis=1, bitorder="little")
    blk = bits[:, :nblk * D].reshape(rows, nblk, D).astype(np.uint64)
    return (blk << np.arange(D, dtype=np.uint64)[None, None, :]).sum(axis=2).astype(np.uint64).reshape(-1)


def _block_errors(M, wblocks, y, D):
    s = oracle.patterns_to_signs(y, D).astype(np.float64)
    return np.sum((wblocks - s @ M.T) ** 2, axis=1)


@pytest.mark.parametrize("rows,in_dim,d,D", [
    (5, 40, 4, 12),    # 256 auxiliary patterns, 8 per lane
    (3, 640, 10, 24),  # LQ-24/10: 16384 patterns per block
    (4, 256, 8, 16),   # LQ-16/8
    (2, 30, 6, 14),    # 70 code bits per row: K = 96 with 26 padding bits
    (3, 60, 6, 6),     # D = d: no auxiliary coordinates
    (2, 96, 16, 20),   # d = 16, 16 patterns: half the lanes idle
    (2, 160, 20, 32),  # LQ-32/20 (d = 20, the widest variant): 4096 patterns per block
    (1, 72, 24, 30),   # d = 24, the largest accepted
])
def test_encode_vs_oracle(lq, rows, in_dim, d, D):
    g = rng_for(62, d * 100 + D, rows)
    M = g.standard_normal((d, D)) / np.sqrt(D)
    if D == d:
        M += 2.0 * np.eye(d)
    M = M.astype(np.float32)
    w = g.standard_normal((rows, in_dim)).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    nblk = in_dim // d
    packed, err = lq.encode(dev(w), dev(M), K, err=True)
    words, err = host(packed), host(err)
    y_gpu = _patterns_from_words(words, rows, nblk, D)
    Md, wb = oracle.to_f64(M), oracle.to_f64(w).reshape(-1, d)
    yo, eo = oracle.encode_blocks(Md, wb, nthreads=NTHREADS)
    # the code is an argmin: identical patterns, or (rarely) a different pattern of equal error
    same = y_gpu == yo
    e_gpu = _block_errors(Md, wb, y_gpu, D)
    assert np.all(same | (np.abs(e_gpu - eo) <= 1e-9 * np.maximum(eo, 1e-300)))
    assert np.mean(same) >= 0.99
    assert np.allclose(err.reshape(-1), eo, rtol=1e-6, atol=1e-7)
    # the words are the library's packing of those patterns (padding bits zero)
    signs = np.full((rows, K), -1, dtype=np.int8)
    signs[:, :nblk * D] = oracle.patterns_to_signs(y_gpu, D).reshape(rows, nblk * D)
    assert np.array_equal(words, oracle.pack_signs(signs))


def test_encode_exact_codewords_recovered(lq):
    """Blocks that are codewords M y* (up to fp32 rounding of w) encode to y*."""
    g = rng_for(62, 7, 0)
    d, D, rows, in_dim = 8, 16, 6, 256
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    nblk = in_dim // d
    ystar = g.integers(0, 1 << D, size=rows * nblk, dtype=np.uint64)
    w = (oracle.patterns_to_signs(ystar, D).astype(np.float64) @ oracle.to_f64(M).T).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    packed, err = lq.encode(dev(w.reshape(rows, in_dim)), dev(M), K, err=True)
    assert np.array_equal(_patterns_from_words(host(packed), rows, nblk, D), ystar)
    assert np.all(host(err) < 1e-9)


def test_encode_singular_projection(lq):
    """A zero row makes M M^T singular: every pattern 0, every error NaN."""
    d, D, rows, in_dim = 4, 12, 2, 40
    M = rng_for(62, 8, 0).standard_normal((d, D)).astype(np.float32)
    M[0, :] = 0.0
    w = rng_for(62, 9, 0).standard_normal((rows, in_dim)).astype(np.float32)
    packed, err = lq.encode(dev(w), dev(M), oracle.lifted_dim(in_dim, d, D), err=True)
    assert np.all(host(packed) == 0)
    assert np.all(np.isnan(host(err)))


def test_encode_many_rows(lq):
    """More rows than CTAs (the grid strides over rows), on a cheap shape."""
    g = rng_for(62, 10, 0)
    d, D, rows, in_dim = 4, 8, 700, 16
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    w = g.standard_normal((rows, in_dim)).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    words = host(lq.encode(dev(w), dev(M), K))
    y_gpu = _patterns_from_words(words, rows, in_dim // d, D)
    yo, eo = oracle.encode_blocks(oracle.to_f64(M), oracle.to_f64(w).reshape(-1, d), nthreads=NTHREADS)
    e_gpu = _block_errors(oracle.to_f64(M), oracle.to_f64(w).reshape(-1, d), y_gpu, D)
    assert np.all((y_gpu == yo) | (np.abs(e_gpu - eo) <= 1e-9 * np.maximum(eo, 1e-300)))
    assert np.mean(y_gpu == yo) >= 0.99


# ------------------------------------------------------------------ row-sharded decode

def test_sharded_decode_single_gpu(lq):
    """ShardedDecode on one GPU: with no process group, and in a 1-rank NCCL group
    (the all-gather runs), equal to lq_lift_gemv bit for bit."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    from bit_lifted_gemm_b200.sharded import ShardedDecode
    L = make_layer(CONFIGS["decode_lq20_8"], 4)
    K = L.cfg.K
    packed_h = torch.from_numpy(L.packed.view(np.int32))
    s_h = torch.from_numpy(L.s)
    a = dev(L.a)
    _, want = lq.lift_gemv(a, dev(L.M), dev(L.packed), dev(L.s), K, tinv=dev(L.tinv))
    sd = ShardedDecode(packed_h, s_h, dev(L.M), K, tinv=dev(L.tinv))
    assert np.array_equal(host(sd(a)), host(want))
    sdb = ShardedDecode(packed_h, s_h, dev(L.M), K, tinv=dev(L.tinv), batch=4)  # preallocated step
    sdb.step(a)
    assert np.array_equal(host(sdb.assembled()), host(want))
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sd1 = ShardedDecode(packed_h, s_h, dev(L.M), K, tinv=dev(L.tinv))
        got = sd1(a)
        torch.cuda.synchronize()
        assert np.array_equal(host(got), host(want))
        sd2 = ShardedDecode(packed_h, s_h, dev(L.M), K, tinv=dev(L.tinv), batch=4)
        sd2.step(a)  # all_gather_into_tensor into the preallocated buffer
        torch.cuda.synchronize()
        assert np.array_equal(host(sd2.assembled()), host(want))
    finally:
        dist.destroy_process_group()


# ------------------------------------------------------------------ failure reporting

def test_bounded_wait_reports_timeout(lq):
    """A wait that nothing completes gives up after its limit (1 ms here), latches
    LQ_ERR_TIMEOUT for lq_get_device_status, which then clears it, and leaves the
    context usable."""
    assert lq.get_device_status() == lq.LQ_OK
    assert lq.lib.lq_selftest_wait_timeout(1000, None) == lq.LQ_OK
    assert lq.get_device_status() == lq.LQ_ERR_TIMEOUT
    assert lq.get_device_status() == lq.LQ_OK
    L = make_layer(CONFIGS["tiny"], 2)
    o = host(lq.gemv(dev(L.packed), dev(L.s), _gpu_u(lq, L)))
    want = oracle.contract(L.packed, L.s, _oracle_u(L))
    assert rel_err(o, want) <= 1e-5


# ------------------------------------------------------------------ bench-size sampled checks

def test_lift_kron_prefill_bench_size_sampled(lq):
    """The 2048-token LQ-24/10 prefill lift as bench.py runs it (64 x 80 factors,
    bf16 activations and u, persistent CTAs with 8-row tiles), checked on sampled
    tokens that the oracle computes one by one."""
    from datagen import make_kron_factors
    cfg = CONFIGS["decode_lq24_10"]
    kf = make_kron_factors(cfg.in_dim, 64, cfg.d, cfg.index)
    L = make_layer(CONFIGS["prefill_lq24_10"], 2048, packed=False)
    u = host(lq.lift_activations_kron(dev(L.a), dev(kf.q1), dev(kf.q2), dev(L.M), cfg.K, r1=dev(kf.r1),
                                      r2=dev(kf.r2), u_dtype="bf16"))
    toks = np.unique(np.concatenate([rng_for(63, 1, 0).choice(2048, size=6, replace=False), [0, 2047]]))
    want = _kron_oracle_u(L.a[toks], "bf16", L.M, kf, cfg.d, cfg.K)
    got = oracle.to_f64(u[toks], "bf16")
    assert np.all(np.abs(got - want) <= _bf16_ulp(want) + 1e-6 * np.max(np.abs(want)))


def test_encode_bench_size_sampled(lq):
    """The LQ-24/10 encoder input bench.py times (26 x 5120 seeded weights), checked
    on sampled blocks that the oracle searches one by one."""
    d, D, rows, in_dim = 10, 24, 26, 5120
    g = np.random.default_rng(0x4C51 + D)
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    w = g.standard_normal((rows, in_dim)).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    packed, err = lq.encode(dev(w), dev(M), K, err=True)
    nblk = in_dim // d
    y_gpu = _patterns_from_words(host(packed), rows, nblk, D)
    e_gpu = host(err).reshape(-1)
    pick = rng_for(63, 2, 0).choice(rows * nblk, size=200, replace=False)
    wb = oracle.to_f64(w).reshape(-1, d)[pick]
    yo, eo = oracle.encode_blocks(oracle.to_f64(M), wb, nthreads=NTHREADS)
    same = y_gpu[pick] == yo
    e_pick = _block_errors(oracle.to_f64(M), wb, y_gpu[pick], D)
    assert np.all(same | (np.abs(e_pick - eo) <= 1e-9 * np.maximum(eo, 1e-300)))
    assert np.mean(same) >= 0.99
    assert np.allclose(e_gpu[pick], eo, rtol=1e-6, atol=1e-7)
