"""Float64 CPU oracle for the LiftQuant lift-then-project layer (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package. The CUDA library and its Python
binding never import it, and it never imports them.

All arithmetic lives in lq_oracle.c (plain float64 loops). This wrapper only
reads inputs exactly (fp32 and bf16 widen to float64 without rounding) and
marshals numpy arrays.

Parity status of each routine (what pins it, in tests/test_oracle_pins.py):
  lifted_dim       closed form K = (in/d)*D, bit-width K/in = D/d
  pack/unpack      hand-derived golden words + round trip
  whiten           identity, permutation (brute force), norm invariance
  whiten_kron      Sylvester Hadamard H_n1 kron H_n2 = H_n (scipy), round trip
                   T (T^{-1} a) = a with T built by numpy's kron, diagonal case
  lift             one-hot inputs recover M's rows at the right block; M = I
  contract         textbook +-1 GEMV (numpy matmul) when D = d, M = I, T = I;
                   exact integer brute force; bit-flip and negation identities
  dense_route      equals the lifted route (w.a' = y^T(M^T a'))
  codebook moments closed forms 0 and M M^T over all 2^D patterns
  encode (brute)   M = I gives sign(w); local optimality against every one-bit
                   flip; exact codewords M y* return y* with zero error
  encode (search)  never below the brute-force optimum; exact codewords M y*
                   recovered; D = d reduces to the closed form sign(M^{-1} w)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_p = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.lqo_lifted_dim.restype = _int
        lib.lqo_lifted_dim.argtypes = [_int, _int, _int]
        lib.lqo_pack_signs.argtypes = [_p, _i64, _i64, _p]
        lib.lqo_unpack_signs.argtypes = [_p, _i64, _i64, _p]
        lib.lqo_whiten.argtypes = [_p, _i64, _i64, _p, _i64, _p]
        lib.lqo_whiten_kron.argtypes = [_p, _i64, _i64, _p, _p, _i64, _p, _i64, _p, _i64, _p]
        lib.lqo_lift.argtypes = [_p, _i64, _i64, _p, _int, _int, _i64, _p]
        lib.lqo_contract.argtypes = [_p, _p, _i64, _i64, _p, _i64, _p, _int]
        lib.lqo_contract_rows.argtypes = [_p, _p, _i64, _i64, _p, _i64, _p, _i64, _p]
        lib.lqo_dense_route.argtypes = [_p, _p, _i64, _i64, _p, _int, _int, _p, _i64, _i64, _p]
        lib.lqo_forward.restype = _int
        lib.lqo_forward.argtypes = [_p, _p, _i64, _i64, _p, _i64, _i64, _p, _i64, _p, _int, _int,
                                    _p, _p, _int]
        lib.lqo_codebook_moments.argtypes = [_p, _int, _int, _p, _p]
        lib.lqo_encode_blocks.argtypes = [_p, _int, _int, _p, _i64, _int, _p, _p, _int]
        lib.lqo_block_identity_maxerr.restype = ctypes.c_double
        lib.lqo_block_identity_maxerr.argtypes = [_p, _int, _int, _p]
        _lib = lib
    return _lib


def _ptr(x: Optional[np.ndarray]):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def to_f64(x: np.ndarray, dtype: str = "f32") -> np.ndarray:
    """Exact float64 view of an fp32 array or of bf16 bit patterns (uint16)."""
    if dtype == "bf16":
        bits = np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << 16
        return bits.view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)


def lifted_dim(in_dim: int, d: int, D: int) -> int:
    return int(_load().lqo_lifted_dim(in_dim, d, D))


def pack_signs(signs: np.ndarray) -> np.ndarray:
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    out, K = signs.shape
    assert K % 32 == 0
    packed = np.zeros((out, K // 32), dtype=np.uint32)
    _load().lqo_pack_signs(_ptr(signs), out, K, _ptr(packed))
    return packed


def unpack_signs(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    out = packed.shape[0]
    signs = np.zeros((out, K), dtype=np.int8)
    _load().lqo_unpack_signs(_ptr(packed), out, K, _ptr(signs))
    return signs


def whiten(a: np.ndarray, tinv: Optional[np.ndarray]) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    batch, in_dim = a.shape
    t = None if tinv is None else np.ascontiguousarray(tinv, dtype=np.float64)
    tblk = 0 if t is None else t.shape[-1]
    ap = np.zeros_like(a)
    _load().lqo_whiten(_ptr(a), batch, in_dim, _ptr(t), tblk, _ptr(ap))
    return ap


def whiten_kron(a: np.ndarray, r1: Optional[np.ndarray], q1: np.ndarray, q2: np.ndarray,
                r2: Optional[np.ndarray], d: int) -> np.ndarray:
    """a' = diag(r2) (Q1 kron Q2) diag(r1) a, r2 constant per d-block ([in/d] entries)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    batch, in_dim = a.shape
    q1 = np.ascontiguousarray(q1, dtype=np.float64)
    q2 = np.ascontiguousarray(q2, dtype=np.float64)
    n1, n2 = q1.shape[0], q2.shape[0]
    assert q1.shape == (n1, n1) and q2.shape == (n2, n2) and n1 * n2 == in_dim and in_dim % d == 0
    r1 = None if r1 is None else np.ascontiguousarray(r1, dtype=np.float64)
    r2 = None if r2 is None else np.ascontiguousarray(r2, dtype=np.float64)
    assert r1 is None or r1.shape == (in_dim,)
    assert r2 is None or r2.shape == (in_dim // d,)
    ap = np.zeros_like(a)
    _load().lqo_whiten_kron(_ptr(a), batch, in_dim, _ptr(r1), _ptr(q1), n1, _ptr(q2), n2, _ptr(r2), d,
                            _ptr(ap))
    return ap


def lift(ap: np.ndarray, M: np.ndarray, K: int) -> np.ndarray:
    ap = np.ascontiguousarray(ap, dtype=np.float64)
    M = np.ascontiguousarray(M, dtype=np.float64)
    batch, in_dim = ap.shape
    d, D = M.shape
    u = np.zeros((batch, K), dtype=np.float64)
    _load().lqo_lift(_ptr(ap), batch, in_dim, _ptr(M), d, D, K, _ptr(u))
    return u


def contract(packed: np.ndarray, s: np.ndarray, u: np.ndarray, nthreads: int = 1) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    out = packed.shape[0]
    batch, K = u.shape
    assert packed.shape[1] * 32 == K
    o = np.zeros((batch, out), dtype=np.float64)
    _load().lqo_contract(_ptr(packed), _ptr(s), out, K, _ptr(u), batch, _ptr(o), nthreads)
    return o


def contract_rows(packed: np.ndarray, s: np.ndarray, u: np.ndarray, rows: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float64)
    u = np.ascontiguousarray(u, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    batch, K = u.shape
    o = np.zeros((batch, rows.size), dtype=np.float64)
    _load().lqo_contract_rows(_ptr(packed), _ptr(s), packed.shape[0], K, _ptr(u), batch,
                              _ptr(rows), rows.size, _ptr(o))
    return o


def dense_route(packed: np.ndarray, s: np.ndarray, M: np.ndarray, ap: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float64)
    M = np.ascontiguousarray(M, dtype=np.float64)
    ap = np.ascontiguousarray(ap, dtype=np.float64)
    out = packed.shape[0]
    batch, in_dim = ap.shape
    d, D = M.shape
    o = np.zeros((batch, out), dtype=np.float64)
    _load().lqo_dense_route(_ptr(packed), _ptr(s), out, K, _ptr(M), d, D, _ptr(ap), batch,
                            in_dim, _ptr(o))
    return o


def forward(packed: np.ndarray, s: np.ndarray, a: np.ndarray, tinv: Optional[np.ndarray],
            M: np.ndarray, K: int, nthreads: int = 1) -> Tuple[np.ndarray, np.ndarray]:
    """Whole layer. Inputs already widened to float64. Returns (u, o)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float64)
    a = np.ascontiguousarray(a, dtype=np.float64)
    M = np.ascontiguousarray(M, dtype=np.float64)
    t = None if tinv is None else np.ascontiguousarray(tinv, dtype=np.float64)
    tblk = 0 if t is None else t.shape[-1]
    out = packed.shape[0]
    batch, in_dim = a.shape
    d, D = M.shape
    u = np.zeros((batch, K), dtype=np.float64)
    o = np.zeros((batch, out), dtype=np.float64)
    rc = _load().lqo_forward(_ptr(packed), _ptr(s), out, K, _ptr(a), batch, in_dim, _ptr(t), tblk,
                             _ptr(M), d, D, _ptr(u), _ptr(o), nthreads)
    assert rc == 0
    return u, o


def encode_blocks(M: np.ndarray, w: np.ndarray, brute: bool = False,
                  nthreads: int = 1) -> Tuple[np.ndarray, np.ndarray]:
    """Blocks w [n][d] -> (sign patterns uint64 [n], bit j set <=> y_j = +1; squared
    errors ||w - M y||^2 [n]). brute=True enumerates all 2^D patterns; otherwise the
    pseudo-inverse start plus the 2^{D-d} auxiliary-vector search."""
    M = np.ascontiguousarray(M, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    d, D = M.shape
    assert w.ndim == 2 and w.shape[1] == d and D <= 63 and D >= d
    n = w.shape[0]
    y = np.zeros(n, dtype=np.uint64)
    err = np.zeros(n, dtype=np.float64)
    _load().lqo_encode_blocks(_ptr(M), d, D, _ptr(w), n, int(brute), _ptr(y), _ptr(err), nthreads)
    return y, err


def patterns_to_signs(y: np.ndarray, D: int) -> np.ndarray:
    """Sign patterns uint64 [n] -> +-1 int8 [n][D] (bit j set <=> +1)."""
    y = np.asarray(y, dtype=np.uint64)
    bits = (y[:, None] >> np.arange(D, dtype=np.uint64)[None, :]) & np.uint64(1)
    return (2 * bits.astype(np.int8) - 1).astype(np.int8)


def codebook_moments(M: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    M = np.ascontiguousarray(M, dtype=np.float64)
    d, D = M.shape
    mean = np.zeros(d)
    second = np.zeros((d, d))
    _load().lqo_codebook_moments(_ptr(M), d, D, _ptr(mean), _ptr(second))
    return mean, second


def block_identity_maxerr(M: np.ndarray, ap_blk: np.ndarray) -> float:
    M = np.ascontiguousarray(M, dtype=np.float64)
    ap_blk = np.ascontiguousarray(ap_blk, dtype=np.float64)
    d, D = M.shape
    return float(_load().lqo_block_identity_maxerr(_ptr(M), d, D, _ptr(ap_blk)))


def threads_available() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
