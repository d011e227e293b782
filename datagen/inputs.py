"""Seeded synthetic layer inputs (random draws only).

Every tensor is drawn from its own PCG64 stream, keyed by
(base seed + workload index, tensor id, extra), so any tensor can be
re-drawn alone and the same bytes reach the oracle and the GPU path.

Tensor ids: 0 = weight signs, 1 = row scales s, 2 = projection M,
3 = whitening inverse blocks, 4 = activations a, 5 = lifted activations u
drawn directly (used to isolate the contraction from the lift), 6 = factors
of a Kronecker-factored whitening inverse.

Distributions follow the synthetic workloads of the LiftQuant layer:
signs iid Bernoulli(0.5); s ~ U[0.01, 0.03]; M ~ N(0, 1/D) in fp32;
whitening-inverse blocks are random orthogonal 128x128 matrices (Q of a
Householder QR of a Gaussian matrix, column signs fixed so diag(R) > 0,
rounded to fp32); activations ~ N(0, 1) in fp32 or bf16 (round to nearest
even). Kronecker factors of T^{-1} = diag(r2) (Q1 kron Q2) diag(r1): Q1, Q2 a
random orthogonal matrix plus N(0, 0.05^2 / n) noise (learned factors start
orthogonal and drift), r1 = exp(U[-0.5, 0.5]) per channel, r2 = exp(U[-0.25,
0.25]) per d-block, all fp32.
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

BASE_SEED = 0x4C51

# tensor stream ids
SIGNS, SCALES, PROJ, TINV, ACT, LIFTED, KRON = 0, 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """One synthetic linear layer of LiftQuant type LQ-D/d.

    in_dim/out: dense layer shape; d/D: block and lifted block widths;
    K: lifted width (in_dim/d)*D rounded up to a multiple of 32;
    tblk: whitening-inverse block size (0 = identity);
    batches: decode batch sizes (or prefill token counts);
    a_dtype: "f32" or "bf16".
    """

    name: str
    index: int
    in_dim: int
    out: int
    d: int
    D: int
    K: int
    tblk: int
    batches: Sequence[int]
    a_dtype: str
    kind: str  # "decode" or "prefill"


CONFIGS = {
    # LQ-24/10 tiny layer, T = identity, fp32 activations
    "tiny": LayerConfig("tiny", 0, 640, 512, 10, 24, 1536, 0, (1, 4), "f32", "decode"),
    # LQ-24/10 decode GEMV, 40 orthogonal 128x128 whitening blocks
    "decode_lq24_10": LayerConfig("decode_lq24_10", 1, 5120, 13824, 10, 24, 12288, 128, (1,), "bf16", "decode"),
    # LQ-20/8 decode sweep (2.5 bit)
    "decode_lq20_8": LayerConfig("decode_lq20_8", 2, 8192, 28672, 8, 20, 20480, 128, (1, 2, 4, 8, 16), "bf16", "decode"),
    # LQ-24/10 prefill GEMM, 2048 tokens
    "prefill_lq24_10": LayerConfig("prefill_lq24_10", 3, 5120, 13824, 10, 24, 12288, 128, (2048,), "bf16", "prefill"),
}

# bit-width sweep LQ-D/8, in=4096, out=11008, D in {16,19,20,22,24}
for _D in (16, 19, 20, 22, 24):
    CONFIGS[f"sweep_lq{_D}_8"] = LayerConfig(
        f"sweep_lq{_D}_8", 4, 4096, 11008, 8, _D, 512 * _D, 128, (1, 64), "bf16", "sweep")


def rng_for(cfg_index: int, tensor_id: int, extra: int = 0) -> np.random.Generator:
    """Independent PCG64 stream for one tensor of one workload."""
    ss = np.random.SeedSequence([BASE_SEED + cfg_index, tensor_id, extra])
    return np.random.Generator(np.random.PCG64(ss))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((b >> 16) & 1)
    return ((b + bias) >> 16).astype(np.uint16)


def f32_from_bf16_bits(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_signs_pm1(rows: int, K: int, cfg_index: int = 0, extra: int = 0) -> np.ndarray:
    """iid +-1 signs as int8 [rows][K]."""
    g = rng_for(cfg_index, SIGNS, extra)
    bits = g.integers(0, 2, size=(rows, K), dtype=np.int8)
    return (2 * bits - 1).astype(np.int8)


def make_packed_random(rows: int, K: int, cfg_index: int, extra: int = 0) -> np.ndarray:
    """Random sign words uint32 [rows][K/32]: every bit is an iid fair coin, so
    the words are the packed form of iid Bernoulli(0.5) signs."""
    g = rng_for(cfg_index, SIGNS, extra)
    return g.integers(0, 1 << 32, size=(rows, K // 32), dtype=np.uint64).astype(np.uint32)


def make_u_bf16(tokens: int, K: int, cfg_index: int, extra: int = 0) -> np.ndarray:
    """Lifted activations drawn directly, N(0, 1) rounded to bf16 (uint16 bits)."""
    g = rng_for(cfg_index, LIFTED, extra)
    return bf16_bits_from_f32(g.standard_normal((tokens, K)).astype(np.float32))


def make_u_f32(batch: int, K: int, cfg_index: int, extra: int = 0) -> np.ndarray:
    """Lifted activations drawn directly, N(0, 1) in fp32."""
    return rng_for(cfg_index, LIFTED, extra).standard_normal((batch, K)).astype(np.float32)


def _orthogonal_blocks(nblk: int, tblk: int, g: np.random.Generator) -> np.ndarray:
    out = np.empty((nblk, tblk, tblk), dtype=np.float32)
    for b in range(nblk):
        q, r = np.linalg.qr(g.standard_normal((tblk, tblk)))
        q = q * np.sign(np.diag(r))[None, :]
        out[b] = q.astype(np.float32)
    return out


@dataclasses.dataclass
class KronFactors:
    r1: np.ndarray   # fp32 [in]
    q1: np.ndarray   # fp32 [n1][n1]
    q2: np.ndarray   # fp32 [n2][n2]
    r2: np.ndarray   # fp32 [in/d]


def make_kron_factors(in_dim: int, n1: int, d: int, cfg_index: int, extra: int = 0) -> KronFactors:
    """Seeded factors of a Kronecker-factored whitening inverse for in = n1 * n2."""
    assert in_dim % n1 == 0 and in_dim % d == 0
    n2 = in_dim // n1
    g = rng_for(cfg_index, KRON, extra)

    def factor(n):
        q, r = np.linalg.qr(g.standard_normal((n, n)))
        q = q * np.sign(np.diag(r))[None, :]
        return (q + 0.05 / np.sqrt(n) * g.standard_normal((n, n))).astype(np.float32)

    q1, q2 = factor(n1), factor(n2)
    r1 = np.exp(g.uniform(-0.5, 0.5, in_dim)).astype(np.float32)
    r2 = np.exp(g.uniform(-0.25, 0.25, in_dim // d)).astype(np.float32)
    return KronFactors(r1, q1, q2, r2)


@dataclasses.dataclass
class LayerInputs:
    cfg: LayerConfig
    batch: int
    packed: Optional[np.ndarray]   # uint32 [out][K/32]
    s: np.ndarray                  # fp32 [out]
    M: np.ndarray                  # fp32 [d][D]
    tinv: Optional[np.ndarray]     # fp32 [in/tblk][tblk][tblk] or None (identity)
    a: np.ndarray                  # fp32 [batch][in] or uint16 bf16 bits [batch][in]
    a_dtype: str                   # "f32" | "bf16"


def make_layer(cfg: LayerConfig, batch: int, *, packed: bool = True, extra: int = 0) -> LayerInputs:
    """All inputs of one layer at one batch size (seeded, deterministic)."""
    i = cfg.index
    ex = cfg.D if cfg.kind == "sweep" else extra
    pk = make_packed_random(cfg.out, cfg.K, i, ex) if packed else None
    s = rng_for(i, SCALES, ex).uniform(0.01, 0.03, size=cfg.out).astype(np.float32)
    M = (rng_for(i, PROJ, ex).standard_normal((cfg.d, cfg.D)) / np.sqrt(cfg.D)).astype(np.float32)
    tinv = None
    if cfg.tblk:
        tinv = _orthogonal_blocks(cfg.in_dim // cfg.tblk, cfg.tblk, rng_for(i, TINV, ex))
    ga = rng_for(i, ACT, ex * 100000 + batch)
    a32 = ga.standard_normal((batch, cfg.in_dim)).astype(np.float32)
    a = bf16_bits_from_f32(a32) if cfg.a_dtype == "bf16" else a32
    return LayerInputs(cfg, batch, pk, s, M, tinv, a, cfg.a_dtype)
