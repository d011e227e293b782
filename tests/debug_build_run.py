"""Runs the debug build (liblq_debug.so; the caller sets LQ_DEBUG=1 before this
process imports the package) through every entry point on small seeded cases:
each result is compared with the oracle, and after each call
lq_get_device_status must be LQ_OK, i.e. no device-side bounds check failed.
Then the bounds self-test trips one check, with no memory access behind it, and
LQ_ERR_BOUNDS must be reported once and then cleared. Prints "debug build ok".

Run by tests/test_gpu_debug_build.py in a child process (the library is chosen
when the package is imported)."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import oracle  # noqa: E402
from datagen import CONFIGS, make_kron_factors, make_layer, make_packed_random, make_signs_pm1  # noqa: E402
from datagen import make_u_bf16, rng_for  # noqa: E402
from datagen.inputs import bf16_bits_from_f32  # noqa: E402
from gpu_common import dev, host, rel_err  # noqa: E402


def bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


def main():
    import torch

    import bit_lifted_gemm_b200 as lq
    assert lq.lib.lq_is_debug_build() == 1, lq.LIB_PATH
    torch.cuda.set_device(0)

    def clean(step):
        st = lq.get_device_status()
        assert st == lq.LQ_OK, f"{step}: {lq.status_str(st)}"

    # pack / unpack, bit-exact
    signs = make_signs_pm1(64, 1536, cfg_index=0)
    packed = host(lq.pack_signs(dev(signs)))
    assert np.array_equal(packed, oracle.pack_signs(signs))
    assert np.array_equal(host(lq.unpack_signs(dev(packed), 1536)), signs)
    clean("pack/unpack")

    # decode lift (fp32) + GEMV, one and four columns
    for batch in (1, 4):
        L = make_layer(CONFIGS["tiny"], batch)
        u = lq.lift_activations(dev(L.a), dev(L.M), L.cfg.K)
        o = host(lq.gemv(dev(L.packed), dev(L.s), u))
        _, oref = oracle.forward(L.packed, L.s, oracle.to_f64(L.a), None, oracle.to_f64(L.M), L.cfg.K)
        assert rel_err(o, oref) <= 1e-5, ("gemv", batch, rel_err(o, oref))
        clean(f"lift + gemv, batch {batch}")

    # prefill lift with 128-wide whitening blocks on tcgen05, bf16 u, ragged tokens
    g = rng_for(62, 5120, 200)
    in_dim, d, D, batch = 5120, 10, 24, 200
    a = bf16_bits_from_f32(g.standard_normal((batch, in_dim)).astype(np.float32))
    M = (g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    tinv = (g.standard_normal((in_dim // 128, 128, 128)) / np.sqrt(128)).astype(np.float32)
    K = oracle.lifted_dim(in_dim, d, D)
    u = oracle.to_f64(host(lq.lift_activations(dev(a), dev(M), K, tinv=dev(tinv), u_dtype="bf16")), "bf16")
    want = oracle.lift(oracle.whiten(oracle.to_f64(a, "bf16"), oracle.to_f64(tinv)), oracle.to_f64(M), K)
    assert np.all(np.abs(u - want) <= bf16_ulp(want) + 1e-6 * np.max(np.abs(want))), "lift tc"
    clean("prefill lift on tcgen05")

    # Kronecker whitening: CUDA-core kernel (decode, fp32 u) and tensor-core kernels (prefill, bf16)
    for batch, u_dtype in ((3, "f32"), (300, "bf16")):
        kf = make_kron_factors(in_dim, 64, d, 61, batch)
        a32 = rng_for(61, 7, batch).standard_normal((batch, in_dim)).astype(np.float32)
        ab = bf16_bits_from_f32(a32)
        u = host(lq.lift_activations_kron(dev(ab), dev(kf.q1), dev(kf.q2), dev(M), K, r1=dev(kf.r1),
                                          r2=dev(kf.r2), u_dtype=u_dtype))
        ap = oracle.whiten_kron(oracle.to_f64(ab, "bf16"), oracle.to_f64(kf.r1), oracle.to_f64(kf.q1),
                                oracle.to_f64(kf.q2), oracle.to_f64(kf.r2), d)
        want = oracle.lift(ap, oracle.to_f64(M), K)
        if u_dtype == "bf16":
            u = oracle.to_f64(u, "bf16")
            assert np.all(np.abs(u - want) <= bf16_ulp(want) + 1e-6 * np.max(np.abs(want))), "kron tc"
        else:
            assert rel_err(u, want) <= 1e-6, ("kron", rel_err(u, want))
        clean(f"Kronecker lift, {batch} tokens")

    # prefill GEMM: 256-token tiles, 64-token tiles with K split, odd row count (per-thread stores)
    for out, K2, tokens in ((300, 1536, 300), (1000, 4096, 64), (129, 1568, 7)):
        pk = make_packed_random(out, K2, 55, extra=K2 + out)
        s = rng_for(55, 1, out).uniform(0.01, 0.03, out).astype(np.float32)
        ub = make_u_bf16(tokens, K2, 55, extra=K2 + tokens)
        o = host(lq.gemm(dev(pk), dev(s), dev(ub)))
        want = oracle.contract(pk, s, oracle.to_f64(ub, "bf16"), 8)
        assert rel_err(o, want) <= 1e-5, ("gemm", out, K2, tokens, rel_err(o, want))
        clean(f"gemm {out} x {K2}, {tokens} tokens")

    # encoder: LQ-24/10 and LQ-32/20 (the widest variant)
    for rows, in_e, de, De in ((3, 640, 10, 24), (2, 160, 20, 32)):
        ge = rng_for(57, de, De)
        Me = (ge.standard_normal((de, De)) / np.sqrt(De)).astype(np.float32)
        w = ge.standard_normal((rows, in_e)).astype(np.float32)
        Ke = oracle.lifted_dim(in_e, de, De)
        words, err = lq.encode(dev(w), dev(Me), Ke, err=True)
        eo = oracle.encode_blocks(oracle.to_f64(Me), oracle.to_f64(w).reshape(-1, de), nthreads=8)[1]
        assert np.allclose(host(err).reshape(-1), eo, rtol=1e-6, atol=1e-7), ("encode", de, De)
        assert host(words).shape == (rows, Ke // 32)
        clean(f"encode d={de} D={De}")

    # the reporting path: one failed check, reported once, then cleared
    assert lq.lib.lq_selftest_bounds(None) == lq.LQ_OK
    assert lq.get_device_status() == lq.LQ_ERR_BOUNDS
    assert lq.get_device_status() == lq.LQ_OK
    torch.cuda.synchronize()
    print("debug build ok")


if __name__ == "__main__":
    main()
