"""Pins of the float64 oracle against facts fixed outside the oracle itself:
values printed in the LiftQuant paper note, closed forms, special cases that
reduce to a textbook routine, invariants and brute force on tiny inputs.

Each pin is chosen so that a plausible slip in the oracle (a transposed M, a
wrong block offset, a flipped bit order, a dropped scale) fails at least one.
"""

import os

import numpy as np
import pytest

import oracle
from datagen import CONFIGS, make_layer, make_signs_pm1, rng_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_positions(spec, K):
    if spec == "-":
        return []
    out = []
    for part in spec.split(","):
        if "-" in part:
            lo, hi = part.split("-")
            out.extend(range(int(lo), int(hi) + 1))
        else:
            out.append(int(part))
    assert all(0 <= k < K for k in out)
    return out


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- storage

def test_bitwidth_table_from_pages():
    """bits = K/in = D/d when in/d is a multiple of 32 (no padding)."""
    for D, d, printed in _golden_lines("bitwidths.txt"):
        D, d = int(D), int(d)
        in_dim = d * 32
        K = oracle.lifted_dim(in_dim, d, D)
        assert K == 32 * D
        assert f"{K / in_dim:.2f}" == printed


def test_lifted_dim_closed_form():
    assert oracle.lifted_dim(640, 10, 24) == 1536
    assert oracle.lifted_dim(5120, 10, 24) == 12288
    assert oracle.lifted_dim(8192, 8, 20) == 20480
    for D in (16, 19, 20, 22, 24):
        assert oracle.lifted_dim(4096, 8, D) == 512 * D
    # padding: (in/d)*D = 3*5 = 15 -> 32
    assert oracle.lifted_dim(9, 3, 5) == 32
    assert oracle.lifted_dim(10, 3, 5) == -1      # d does not divide in
    assert oracle.lifted_dim(0, 3, 5) == -1
    for name, cfg in CONFIGS.items():
        assert oracle.lifted_dim(cfg.in_dim, cfg.d, cfg.D) == cfg.K, name
        # storage: exactly D bits per d weights
        assert cfg.K * cfg.out / 8 == cfg.out * cfg.in_dim * cfg.D / cfg.d / 8


def test_pack_golden_words():
    for row in _golden_lines("pack_words.txt"):
        K = int(row[1])
        pos = _parse_positions(row[3], K)
        want = [int(w, 16) for w in row[5].split(",")]
        signs = -np.ones((1, K), dtype=np.int8)
        signs[0, pos] = 1
        got = oracle.pack_signs(signs)
        assert got.tolist() == [want]
        back = oracle.unpack_signs(got, K)
        assert np.array_equal(back, signs)


def test_pack_roundtrip_random():
    signs = make_signs_pm1(37, 32 * 9, cfg_index=99)
    assert np.array_equal(oracle.unpack_signs(oracle.pack_signs(signs), 32 * 9), signs)


# ---------------------------------------------------------------- whitening

def test_whiten_identity_and_null():
    a = rng_for(99, 4).standard_normal((3, 256))
    assert np.array_equal(oracle.whiten(a, None), a)
    eye = np.stack([np.eye(128)] * 2)
    assert np.array_equal(oracle.whiten(a, eye), a)


def test_whiten_permutation_bruteforce():
    g = rng_for(99, 3)
    tblk, nblk = 8, 5
    perms = [g.permutation(tblk) for _ in range(nblk)]
    tinv = np.zeros((nblk, tblk, tblk))
    for b, p in enumerate(perms):
        tinv[b, np.arange(tblk), p] = 1.0
    a = g.standard_normal((2, tblk * nblk))
    ap = oracle.whiten(a, tinv)
    for c in range(2):
        for b in range(nblk):
            for i in range(tblk):
                assert ap[c, b * tblk + i] == a[c, b * tblk + perms[b][i]]


def test_whiten_orthogonal_norm():
    L = make_layer(CONFIGS["decode_lq24_10"], 2, packed=False)
    a = oracle.to_f64(L.a, "bf16")
    ap = oracle.whiten(a, L.tinv)
    for blk in range(L.tinv.shape[0]):
        sl = slice(blk * 128, (blk + 1) * 128)
        na, nap = np.linalg.norm(a[:, sl], axis=1), np.linalg.norm(ap[:, sl], axis=1)
        assert np.allclose(na, nap, rtol=2e-6)


# ---------------------------------------------------------------- lift

# ------------------------------------------- Kronecker-factored whitening
# T = diag(s1) (P1 kron P2) diag(s2), s2 constant per d-block (LiftQuant paper
# note, "Key designs" 3); the oracle is handed the factors of T^{-1}.

def test_whiten_kron_sylvester_hadamard():
    """H_4 kron H_8 = H_32 in Sylvester's ordering, so normalised Hadamard
    factors give the 32-point Walsh-Hadamard transform (scipy's matrix)."""
    from scipy.linalg import hadamard
    g = rng_for(90, 1, 0)
    a = g.standard_normal((3, 32))
    q1 = hadamard(4) / 2.0
    q2 = hadamard(8) / np.sqrt(8.0)
    got = oracle.whiten_kron(a, None, q1, q2, None, 4)
    want = a @ (hadamard(32) / np.sqrt(32.0)).T
    assert np.max(np.abs(got - want)) < 1e-13
    assert np.allclose(np.linalg.norm(got, axis=1), np.linalg.norm(a, axis=1), rtol=1e-14)


@pytest.mark.parametrize("n1,n2,d", [(3, 5, 5), (4, 6, 3), (2, 8, 4)])
def test_whiten_kron_inverts_T(n1, n2, d):
    """Round trip: T built densely from its factors with numpy's kron maps the
    oracle's a' = T^{-1} a back to a. Catches swapped s1/s2, a transposed
    factor, and the Kronecker index order (n1 != n2)."""
    g = rng_for(90, 2, n1 * 100 + n2)
    n = n1 * n2
    p1 = g.standard_normal((n1, n1)) + 3 * np.eye(n1)
    p2 = g.standard_normal((n2, n2)) + 3 * np.eye(n2)
    s1 = np.exp(g.uniform(-1, 1, n))
    s2_blk = np.exp(g.uniform(-1, 1, n // d))
    T = np.diag(s1) @ np.kron(p1, p2) @ np.diag(np.repeat(s2_blk, d))
    a = g.standard_normal((2, n))
    ap = oracle.whiten_kron(a, 1.0 / s1, np.linalg.inv(p1), np.linalg.inv(p2), 1.0 / s2_blk, d)
    assert np.max(np.abs(ap @ T.T - a)) < 1e-10


def test_whiten_kron_diagonal_case():
    """Identity factors: a' = r2[i/d] * r1[i] * a[i], element by element."""
    g = rng_for(90, 3, 0)
    n1, n2, d = 4, 10, 5
    a = g.standard_normal((2, n1 * n2))
    r1 = g.uniform(0.5, 2.0, n1 * n2)
    r2 = g.uniform(0.5, 2.0, n1 * n2 // d)
    got = oracle.whiten_kron(a, r1, np.eye(n1), np.eye(n2), r2, d)
    assert np.array_equal(got, a * r1[None, :] * np.repeat(r2, d)[None, :])


def test_whiten_kron_single_factor_is_block_whitening():
    """Q1 = I: Q1 kron Q2 is block-diagonal with n1 copies of Q2, i.e. the
    block whitening with tblk = n2 and every block equal to Q2."""
    g = rng_for(90, 4, 0)
    n1, n2 = 3, 8
    q2 = g.standard_normal((n2, n2))
    a = g.standard_normal((2, n1 * n2))
    got = oracle.whiten_kron(a, None, np.eye(n1), q2, None, 4)
    want = oracle.whiten(a, np.stack([q2] * n1))
    assert np.max(np.abs(got - want)) < 1e-13


def test_lift_one_hot_recovers_rows_of_M():
    g = rng_for(99, 2)
    d, D, nblk = 3, 7, 4
    M = g.standard_normal((d, D))
    K = oracle.lifted_dim(d * nblk, d, D)
    for blk in range(nblk):
        for i in range(d):
            ap = np.zeros((1, d * nblk))
            ap[0, blk * d + i] = 1.0
            u = oracle.lift(ap, M, K)[0]
            want = np.zeros(K)
            want[blk * D:(blk + 1) * D] = M[i]
            assert np.array_equal(u, want)


def test_lift_identity_projection():
    g = rng_for(99, 4)
    d = D = 8
    ap = g.standard_normal((3, 64))
    u = oracle.lift(ap, np.eye(8), 64)
    assert np.array_equal(u, ap)


def test_lift_padding_is_zero():
    g = rng_for(99, 5)
    ap = g.standard_normal((2, 9))
    u = oracle.lift(ap, g.standard_normal((3, 5)), 32)
    assert np.all(u[:, 15:] == 0.0)
    assert np.all(u[:, :15] != 0.0)


# ---------------------------------------------------------------- contraction

def test_contract_textbook_gemv():
    """D = d, M = I, T = I: o = diag(s) . S . a with S the +-1 matrix."""
    g = rng_for(99, 6)
    out, in_dim = 40, 96
    signs = make_signs_pm1(out, in_dim, cfg_index=98)
    packed = oracle.pack_signs(signs)
    s = g.uniform(0.01, 0.03, out)
    a = g.standard_normal((3, in_dim))
    u, o = oracle.forward(packed, s, a, None, np.eye(4), in_dim)
    want = (a @ signs.astype(np.float64).T) * s[None, :]
    assert np.allclose(o, want, rtol=1e-13, atol=1e-13)
    assert np.array_equal(u, a)


def _tiny_integer_layer(seed):
    g = np.random.default_rng(seed)
    in_dim, d, D, tblk, out, batch = 12, 3, 5, 4, 6, 2
    K = 32  # (12/3)*5 = 20 -> 32
    M = g.integers(-2, 3, size=(d, D))
    tinv = g.integers(-1, 2, size=(in_dim // tblk, tblk, tblk))
    a = g.integers(-3, 4, size=(batch, in_dim))
    s = g.integers(1, 4, size=out)
    signs = g.choice([-1, 1], size=(out, K)).astype(np.int8)
    return in_dim, d, D, tblk, out, batch, K, M, tinv, a, s, signs


def test_contract_integer_bruteforce_exact():
    in_dim, d, D, tblk, out, batch, K, M, tinv, a, s, signs = _tiny_integer_layer(7)
    # pure-Python integer arithmetic, straight from the definitions
    want = [[0] * out for _ in range(batch)]
    for c in range(batch):
        ap = [0] * in_dim
        for blk in range(in_dim // tblk):
            for i in range(tblk):
                ap[blk * tblk + i] = sum(int(tinv[blk][i][j]) * int(a[c][blk * tblk + j]) for j in range(tblk))
        u = [0] * K
        for blk in range(in_dim // d):
            for j in range(D):
                u[blk * D + j] = sum(int(M[i][j]) * ap[blk * d + i] for i in range(d))
        for r in range(out):
            want[c][r] = int(s[r]) * sum(int(signs[r][k]) * u[k] for k in range(K))
    packed = oracle.pack_signs(signs)
    _, o = oracle.forward(packed, s.astype(float), a.astype(float), tinv.astype(float),
                          M.astype(float), K)
    assert o.tolist() == [[float(x) for x in row] for row in want]


def test_bit_flip_and_negation():
    in_dim, d, D, tblk, out, batch, K, M, tinv, a, s, signs = _tiny_integer_layer(11)
    packed = oracle.pack_signs(signs)
    u, o = oracle.forward(packed, s.astype(float), a.astype(float), tinv.astype(float), M.astype(float), K)
    # flipping all bits negates o
    _, oneg = oracle.forward(~packed, s.astype(float), a.astype(float), tinv.astype(float), M.astype(float), K)
    assert np.array_equal(oneg, -o)
    # flipping bit k of row r moves o[c][r] by exactly -2 sigma s[r] u[c][k]
    for r, k in [(0, 0), (3, 17), (5, 31), (2, 14)]:
        flipped = packed.copy()
        flipped[r, k // 32] ^= np.uint32(1 << (k % 32))
        o2 = oracle.contract(flipped, s.astype(float), u)
        delta = o2 - o
        for c in range(batch):
            assert delta[c, r] == -2.0 * signs[r, k] * s[r] * u[c, k]
        other = [x for x in range(out) if x != r]
        assert np.all(delta[:, other] == 0.0)


def test_linearity_in_activations():
    L = make_layer(CONFIGS["tiny"], 4)
    a = oracle.to_f64(L.a)
    b = rng_for(99, 8).standard_normal(a.shape)
    M = oracle.to_f64(L.M)
    _, oa = oracle.forward(L.packed, L.s, a, None, M, L.cfg.K)
    _, ob = oracle.forward(L.packed, L.s, b, None, M, L.cfg.K)
    _, oab = oracle.forward(L.packed, L.s, 2.5 * a - 0.75 * b, None, M, L.cfg.K)
    assert np.allclose(oab, 2.5 * oa - 0.75 * ob, rtol=1e-12, atol=1e-14)


def test_dense_reconstruction_route():
    """w = M y per block: the dense route equals the lifted route to 1e-12."""
    L = make_layer(CONFIGS["tiny"], 4)
    rows = 64
    a = oracle.to_f64(L.a)
    M = oracle.to_f64(L.M)
    u, o = oracle.forward(L.packed[:rows], L.s[:rows], a, None, M, L.cfg.K)
    o2 = oracle.dense_route(L.packed[:rows], L.s[:rows], M, a, L.cfg.K)
    assert np.linalg.norm(o - o2) / np.linalg.norm(o) <= 1e-12
    # with a whitening transform too
    Lw = make_layer(CONFIGS["decode_lq24_10"], 1)
    aw = oracle.to_f64(Lw.a, "bf16")[:, :640]
    tw = oracle.to_f64(Lw.tinv[:5])
    ap = oracle.whiten(aw, tw)
    Mw = oracle.to_f64(Lw.M)
    K = oracle.lifted_dim(640, 10, 24)
    pk = Lw.packed[:32, :K // 32]
    _, ow = oracle.forward(pk, Lw.s[:32], aw, tw, Mw, K)
    ow2 = oracle.dense_route(pk, Lw.s[:32], Mw, ap, K)
    assert np.linalg.norm(ow - ow2) / np.linalg.norm(ow) <= 1e-12


@pytest.mark.parametrize("d,D", [(4, 12), (8, 16)])
def test_codebook_moments_closed_form(d, D):
    M = rng_for(99, 9, D).standard_normal((d, D)) / np.sqrt(D)
    mean, second = oracle.codebook_moments(M)
    assert np.max(np.abs(mean)) <= 1e-12
    assert np.allclose(second, M @ M.T, rtol=0, atol=1e-12)


def test_block_identity_all_patterns():
    g = rng_for(99, 10)
    M = g.standard_normal((8, 16)) / 4.0
    ap = g.standard_normal(8)
    assert oracle.block_identity_maxerr(M, ap) <= 1e-12


def test_output_second_moment_statistics():
    """iid signs: E[o_r] = 0, E[o_r^2] = s_r^2 |u|^2."""
    g = rng_for(99, 11)
    out, K = 4096, 256
    packed = g.integers(0, 1 << 32, size=(out, K // 32), dtype=np.uint64).astype(np.uint32)
    u = g.standard_normal((1, K))
    o = oracle.contract(packed, np.ones(out), u)
    ratio = np.mean(o ** 2) / np.sum(u ** 2)
    assert abs(ratio - 1.0) < 0.1
    assert abs(np.mean(o)) / np.sqrt(np.sum(u ** 2)) < 0.1


def test_contract_rows_and_threads_agree():
    L = make_layer(CONFIGS["tiny"], 4)
    a = oracle.to_f64(L.a)
    u, o = oracle.forward(L.packed, L.s, a, None, oracle.to_f64(L.M), L.cfg.K, nthreads=1)
    o4 = oracle.contract(L.packed, L.s, u, nthreads=4)
    assert np.array_equal(o, o4)
    rows = np.array([0, 5, 511, 100])
    assert np.array_equal(oracle.contract_rows(L.packed, L.s, u, rows), o[:, rows])


# ---------------------------------------------------------------- encoder
# Nearest lifted codeword M y, y in {+-1}^D, of a block w of d weights
# (LiftQuant paper note, "Key designs" 2).

def _np_err(M, w, y, D):
    s = oracle.patterns_to_signs(np.asarray([y], dtype=np.uint64), D)[0].astype(np.float64)
    return float(np.sum((w - M @ s) ** 2))


def test_encode_brute_identity_projection():
    """M = I: the nearest point of {+-1}^d to w is sign(w), coordinate by coordinate."""
    g = rng_for(91, 1, 0)
    d = 8
    w = g.standard_normal((20, d))
    y, err = oracle.encode_blocks(np.eye(d), w, brute=True)
    want = ((w >= 0).astype(np.uint64) << np.arange(d, dtype=np.uint64)[None, :]).sum(axis=1)
    assert np.array_equal(y, want.astype(np.uint64))
    assert np.allclose(err, np.sum((np.abs(w) - 1.0) ** 2, axis=1), rtol=1e-12, atol=1e-12)


def test_encode_brute_locally_optimal():
    """The brute-force optimum is at least as good as each of its D one-bit
    neighbours, and its reported error is ||w - M y||^2 recomputed by numpy."""
    g = rng_for(91, 2, 0)
    d, D = 3, 9
    M = g.standard_normal((d, D)) / np.sqrt(D)
    w = g.standard_normal((15, d))
    y, err = oracle.encode_blocks(M, w, brute=True)
    for b in range(w.shape[0]):
        e0 = _np_err(M, w[b], int(y[b]), D)
        assert abs(e0 - err[b]) <= 1e-12 * max(1.0, e0)
        for j in range(D):
            assert _np_err(M, w[b], int(y[b]) ^ (1 << j), D) >= e0 - 1e-12


@pytest.mark.parametrize("d,D", [(4, 10), (6, 14), (10, 16)])
def test_encode_exact_codewords(d, D):
    """w = M y*: both searches return y* with zero error (the auxiliary vector
    z = y*_A makes the solved coordinates exact)."""
    g = rng_for(91, 3, d * 100 + D)
    M = g.standard_normal((d, D)) / np.sqrt(D)
    ystar = g.integers(0, 1 << D, size=12, dtype=np.uint64)
    w = oracle.patterns_to_signs(ystar, D).astype(np.float64) @ M.T
    for brute in (True, False):
        if brute and D > 14:
            continue
        y, err = oracle.encode_blocks(M, w, brute=brute)
        assert np.array_equal(y, ystar)
        assert np.all(err < 1e-20)


@pytest.mark.parametrize("d,D", [(2, 8), (4, 12), (5, 13), (6, 14)])
def test_encode_search_never_beats_brute(d, D):
    g = rng_for(91, 4, d * 100 + D)
    M = g.standard_normal((d, D)) / np.sqrt(D)
    w = g.standard_normal((25, d))
    _, eb = oracle.encode_blocks(M, w, brute=True)
    ys, es = oracle.encode_blocks(M, w)
    assert np.all(es >= eb - 1e-12)
    for b in range(w.shape[0]):
        assert abs(_np_err(M, w[b], int(ys[b]), D) - es[b]) <= 1e-12 * max(1.0, es[b])
    # candidate 0 is the pseudo-inverse start, so no block ends worse than sign(M^+ w)
    y0 = np.where(w @ np.linalg.pinv(M).T >= 0, 1.0, -1.0)
    e0 = np.sum((w - y0 @ M.T) ** 2, axis=1)
    assert np.all(es <= e0 + 1e-12)


def test_encode_search_square_closed_form():
    """D = d: no auxiliary coordinates, so the result is sign(M^{-1} w)."""
    g = rng_for(91, 5, 0)
    d = 6
    M = g.standard_normal((d, d)) + 2 * np.eye(d)
    w = g.standard_normal((10, d))
    y, _ = oracle.encode_blocks(M, w)
    x = np.linalg.solve(M, w.T).T
    want = ((x >= 0).astype(np.uint64) << np.arange(d, dtype=np.uint64)[None, :]).sum(axis=1)
    assert np.array_equal(y, want.astype(np.uint64))


# ---------------------------------------------------------------- Gaussian source

def test_gaussian_table_info_and_rate_distortion():
    """The note's Gaussian-source table: Info is -1/2 log2 MSE on every row (to the
    printed rounding), and no code beats the rate-distortion bound of an i.i.d.
    N(0, 1) source at its D/d bits per weight, MSE >= 2^(-2 D/d)."""
    rows = _golden_lines("gaussian_source.txt")
    assert len(rows) == 5
    for D, d, bits, mse, info in rows:
        D, d, bits, mse, info = int(D), int(d), float(bits), float(mse), float(info)
        assert abs(bits - D / d) <= 0.005
        assert abs(info - (-0.5 * np.log2(mse))) <= 0.015, (D, d)
        assert mse >= 2.0 ** (-2.0 * D / d), (D, d)


@pytest.mark.parametrize("d,D", [(8, 16), (10, 24), (6, 14)])
def test_encode_gaussian_source_above_rate_distortion(d, D):
    """The search on i.i.d. N(0, 1) weights with M ~ N(0, 1/D): its per-weight
    squared error, computed independently here from the returned patterns, equals
    the oracle's and stays above 2^(-2 D/d), which no quantizer at D/d bits per
    weight can beat on this source."""
    g = rng_for(92, d, D)
    M = g.standard_normal((d, D)) / np.sqrt(D)
    w = g.standard_normal((300, d))
    y, e = oracle.encode_blocks(M, w, nthreads=4)
    s = oracle.patterns_to_signs(y, D).astype(np.float64)
    e_np = np.sum((w - s @ M.T) ** 2, axis=1)
    assert np.allclose(e, e_np, rtol=1e-12, atol=1e-14)
    mse = float(np.mean(e_np)) / d
    assert mse >= 2.0 ** (-2.0 * D / d), mse
