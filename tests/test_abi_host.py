"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/lq.h declares, and rejects bad arguments synchronously
(before any CUDA call) with LQ_ERR_INVALID_ARG."""

import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "lq.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"LQ_API\s+[\w\s\*]+?\b(lq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import bit_lifted_gemm_b200 as lq
    declared = _declared_symbols()
    assert len(declared) >= 8
    assert set(declared) == set(lq.SYMBOLS)
    for name in declared:
        assert hasattr(lq.lib, name), name
    with open(os.path.join(ROOT, "bit_lifted_gemm_b200", "liblq.so"), "rb") as f:
        blob = f.read()
    for name in declared:
        assert name.encode() in blob


def test_status_strings():
    import bit_lifted_gemm_b200 as lq
    assert lq.status_str(0) == "LQ_OK"
    assert lq.status_str(1) == "LQ_ERR_INVALID_ARG"
    assert lq.status_str(4) == "LQ_ERR_TIMEOUT"
    assert lq.status_str(lq.LQ_ERR_BOUNDS) == "LQ_ERR_BOUNDS"
    assert lq.status_str(99) == "LQ_ERR_UNKNOWN"


def test_debug_build_exports_and_identifies_itself():
    """liblq_debug.so, the -DLQ_DEBUG build of the same sources (device-side
    bounds checks), is built incrementally here, exports every declared symbol
    and is the library the package loads under LQ_DEBUG=1. The release library
    says it is not the debug build and refuses the bounds self-test without
    launching; the debug library, with no GPU, fails its device check."""
    import importlib.util
    import subprocess
    import sys

    import bit_lifted_gemm_b200 as lq
    spec = importlib.util.spec_from_file_location("lq_build", os.path.join(ROOT, "bit_lifted_gemm_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    path = mod.build(debug=True)
    assert os.path.basename(path) == "liblq_debug.so"
    with open(path, "rb") as f:
        blob = f.read()
    for name in _declared_symbols():
        assert name.encode() in blob, name
    assert lq.lib.lq_is_debug_build() == 0
    assert lq.lib.lq_selftest_bounds(None) == lq.LQ_ERR_UNSUPPORTED
    code = ("import bit_lifted_gemm_b200 as lq, os; "
            "print(lq.lib.lq_is_debug_build(), os.path.basename(lq.LIB_PATH), "
            "lq.lib.lq_selftest_bounds(None) in (lq.LQ_ERR_CUDA, lq.LQ_ERR_UNSUPPORTED))")
    env = dict(os.environ, LQ_DEBUG="1")
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True,
                         check=True, timeout=300).stdout.split()
    assert out == ["1", "liblq_debug.so", "True"]


def test_lifted_dim_matches_oracle_closed_form():
    import bit_lifted_gemm_b200 as lq
    for args in [(640, 10, 24), (5120, 10, 24), (8192, 8, 20), (4096, 8, 19), (9, 3, 5), (10, 3, 5),
                 (0, 1, 1), (7, 7, 1), (1 << 30, 1, 4)]:
        assert lq.lifted_dim(*args) == oracle.lifted_dim(*args), args


P = 0x100000  # a 16-byte-aligned fake address; never dereferenced (validation fails first)
MIS = P + 4   # misaligned
W = 0x200000  # a 256-byte-aligned fake workspace address
BIG = 1 << 40  # workspace bytes: more than any shape needs


def _c(v):
    return ctypes.c_void_p(v)


def _far(i):
    """Distinct fake buffer addresses, 64 GiB apart: never dereferenced (the calls
    that get them return before any launch), far enough apart that no range of
    any tested shape reaches the next."""
    return _c((i + 1) << 36)


@pytest.mark.parametrize("case", [
    ("pack null", "lq_pack_signs", [None, 4, 32, _c(P), None]),
    ("pack K%32", "lq_pack_signs", [_c(P), 4, 48, _c(P), None]),
    ("pack out<1", "lq_pack_signs", [_c(P), 0, 32, _c(P), None]),
    ("pack misaligned", "lq_pack_signs", [_c(MIS), 4, 32, _c(P), None]),
    ("unpack null", "lq_unpack_signs", [_c(P), 4, 32, None, None]),
    ("gemv batch 0", "lq_gemv", [_c(P), _c(P), 8, 64, _c(P), 0, _c(P), _c(W), BIG, None]),
    ("gemv batch 17", "lq_gemv", [_c(P), _c(P), 8, 64, _c(P), 17, _c(P), _c(W), BIG, None]),
    ("gemv K%32", "lq_gemv", [_c(P), _c(P), 8, 40, _c(P), 1, _c(P), _c(W), BIG, None]),
    ("gemv misaligned u", "lq_gemv", [_c(P), _c(P), 8, 64, _c(MIS), 1, _c(P), _c(W), BIG, None]),
    ("gemv null workspace", "lq_gemv", [_c(P), _c(P), 8, 64, _c(P), 1, _c(P), None, BIG, None]),
    ("gemv workspace misaligned", "lq_gemv", [_c(P), _c(P), 8, 64, _c(P), 1, _c(P), _c(W + 16), BIG, None]),
    ("gemv workspace too small", "lq_gemv", [_c(P), _c(P), 8, 64, _c(P), 1, _c(P), _c(W), 16, None]),
    ("gemv null s", "lq_gemv", [_c(P), None, 8, 64, _c(P), 1, _c(P), _c(W), BIG, None]),
    ("lift_gemv batch 17", "lq_lift_gemv", [_c(P), 0, 17, 640, None, 0, _c(P), 10, 24, _c(P), _c(P), 8, 1536,
                                            _c(P), _c(P), _c(W), BIG, None]),
    ("lift_gemv K mismatch", "lq_lift_gemv", [_c(P), 0, 1, 640, None, 0, _c(P), 10, 24, _c(P), _c(P), 8, 1504,
                                              _c(P), _c(P), _c(W), BIG, None]),
    ("lift_gemv null o", "lq_lift_gemv", [_c(P), 0, 1, 640, None, 0, _c(P), 10, 24, _c(P), _c(P), 8, 1536,
                                          _c(P), None, _c(W), BIG, None]),
    ("lift_gemv misaligned u", "lq_lift_gemv", [_c(P), 0, 1, 640, None, 0, _c(P), 10, 24, _c(P), _c(P), 8, 1536,
                                                _c(MIS), _c(P), _c(W), BIG, None]),
    ("lift_gemv out 0", "lq_lift_gemv", [_c(P), 0, 1, 640, None, 0, _c(P), 10, 24, _c(P), _c(P), 0, 1536,
                                         _c(P), _c(P), _c(W), BIG, None]),
    ("gemm tokens 0", "lq_gemm", [_c(P), _c(P), 8, 64, _c(P), 0, _c(P), None]),
    ("gemm K<32", "lq_gemm", [_c(P), _c(P), 8, 0, _c(P), 4, _c(P), None]),
    ("gemm null o", "lq_gemm", [_c(P), _c(P), 8, 64, _c(P), 4, None, None]),
    ("lift K mismatch", "lq_lift_activations", [_c(P), 0, 1, 640, None, 0, _c(P), 10, 24, _c(P), 0, 1504, None]),
    ("lift d does not divide in", "lq_lift_activations", [_c(P), 0, 1, 641, None, 0, _c(P), 10, 24, _c(P), 0, 1536, None]),
    ("lift tblk does not divide in", "lq_lift_activations", [_c(P), 1, 1, 640, _c(P), 96, _c(P), 10, 24, _c(P), 0, 1536, None]),
    ("lift tblk too big", "lq_lift_activations", [_c(P), 1, 1, 1024, _c(P), 512, _c(P), 8, 16, _c(P), 0, 2048, None]),
    ("lift bad dtype", "lq_lift_activations", [_c(P), 7, 1, 640, None, 0, _c(P), 10, 24, _c(P), 0, 1536, None]),
    ("lift d too big", "lq_lift_activations", [_c(P), 0, 1, 130, None, 0, _c(P), 65, 2, _c(P), 0, 32, None]),
    ("lift batch 0", "lq_lift_activations", [_c(P), 0, 0, 640, None, 0, _c(P), 10, 24, _c(P), 0, 1536, None]),
    ("kron n1*n2 != in", "lq_lift_activations_kron", [_c(P), 0, 1, 640, None, _c(P), 8, _c(P), 81, None, _c(P), 10,
                                                      24, _c(P), 0, 1536, None]),
    ("kron null q2", "lq_lift_activations_kron", [_c(P), 0, 1, 640, None, _c(P), 8, None, 80, None, _c(P), 10, 24,
                                                  _c(P), 0, 1536, None]),
    ("kron misaligned r1", "lq_lift_activations_kron", [_c(P), 0, 1, 640, _c(MIS), _c(P), 8, _c(P), 80, None, _c(P),
                                                        10, 24, _c(P), 0, 1536, None]),
    ("kron n2 too big", "lq_lift_activations_kron", [_c(P), 0, 1, 640, None, _c(P), 4, _c(P), 160, None, _c(P), 10,
                                                     24, _c(P), 0, 1536, None]),
    ("kron K mismatch", "lq_lift_activations_kron", [_c(P), 0, 1, 640, None, _c(P), 8, _c(P), 80, None, _c(P), 10,
                                                     24, _c(P), 0, 1504, None]),
    ("kron in too big", "lq_lift_activations_kron", [_c(P), 0, 1, 20480, None, _c(P), 160, _c(P), 128, None, _c(P),
                                                     10, 24, _c(P), 0, 49152, None]),
    ("kron plan too big (odd n1)", "lq_lift_activations_kron", [_c(P), 0, 1, 16320, None, _c(P), 255, _c(P), 64,
                                                                None, _c(P), 10, 24, _c(P), 0, 39168, None]),
    ("encode d > 24", "lq_encode", [_c(P), 4, 500, _c(P), 25, 32, _c(P), 640, None, None]),
    ("encode D - d > 24", "lq_encode", [_c(P), 4, 40, _c(P), 4, 29, _c(P), 320, None, None]),
    ("encode D < d", "lq_encode", [_c(P), 4, 40, _c(P), 8, 4, _c(P), 32, None, None]),
    ("encode d does not divide in", "lq_encode", [_c(P), 4, 42, _c(P), 4, 12, _c(P), 128, None, None]),
    ("encode K mismatch", "lq_encode", [_c(P), 4, 40, _c(P), 4, 12, _c(P), 96, None, None]),
    ("encode null packed", "lq_encode", [_c(P), 4, 40, _c(P), 4, 12, None, 128, None, None]),
    ("encode misaligned err", "lq_encode", [_c(P), 4, 40, _c(P), 4, 12, _c(P), 128, _c(MIS), None]),
    ("selftest limit 0", "lq_selftest_wait_timeout", [0, None]),
    ("selftest limit above 1 s", "lq_selftest_wait_timeout", [2000000, None]),
], ids=lambda c: c[0])
def test_invalid_arguments_rejected_before_launch(case):
    import bit_lifted_gemm_b200 as lq
    _, fn, args = case
    assert getattr(lq.lib, fn)(*args) == lq.LQ_ERR_INVALID_ARG


@pytest.mark.parametrize("lang,compiler", [("c", "gcc"), ("c++", "g++")])
def test_header_compiles_standalone(lang, compiler):
    """include/lq.h is a plain C header (also usable from C++)."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    r = subprocess.run([compiler, "-fsyntax-only", "-Wall", "-Wextra", "-Werror", "-x", lang,
                        os.path.join(ROOT, "include", "lq.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_fault_injection_timeout(monkeypatch):
    """LQ_FAULT=timeout: lq_get_device_status reports a timeout without a device."""
    import bit_lifted_gemm_b200 as lq
    monkeypatch.setenv("LQ_FAULT", "timeout")
    assert lq.lib.lq_get_device_status(None) == lq.LQ_ERR_TIMEOUT
    assert lq.lib.lq_status_str(lq.LQ_ERR_TIMEOUT)


def test_fault_injection_launch(monkeypatch):
    """LQ_FAULT=launch: valid calls return LQ_ERR_CUDA without touching their
    pointers; argument checks still come first."""
    import bit_lifted_gemm_b200 as lq
    monkeypatch.setenv("LQ_FAULT", "launch")
    assert lq.lib.lq_pack_signs(_far(0), 4, 32, _far(1), None) == lq.LQ_ERR_CUDA
    assert lq.lib.lq_gemv(_far(0), _far(1), 8, 64, _far(2), 1, _far(3), _far(4), BIG, None) == lq.LQ_ERR_CUDA
    assert lq.lib.lq_gemm(_far(0), _far(1), 8, 64, _far(2), 4, _far(3), None) == lq.LQ_ERR_CUDA
    assert lq.lib.lq_encode(_far(0), 4, 40, _far(1), 4, 12, _far(2), 128, None, None) == lq.LQ_ERR_CUDA
    assert lq.lib.lq_gemv(_c(P), _c(P), 8, 64, _c(P), 0, _c(P), _c(W), BIG, None) == lq.LQ_ERR_INVALID_ARG


def test_encode_accepts_every_tabulated_code(monkeypatch):
    """The encoder's argument checks accept every LQ-D/d code of the pages' table,
    LQ-32/20 (d = 20) included, and d up to 24; with LQ_FAULT=launch an accepted
    call returns LQ_ERR_CUDA right after its checks, without launching."""
    import bit_lifted_gemm_b200 as lq
    monkeypatch.setenv("LQ_FAULT", "launch")
    for d, D in ((20, 32), (16, 32), (8, 16), (14, 30), (10, 24), (24, 48)):
        in_dim = d * 8
        K = lq.lifted_dim(in_dim, d, D)
        assert lq.lib.lq_encode(_far(0), 2, in_dim, _far(1), d, D, _far(2), K, None, None) == lq.LQ_ERR_CUDA, (d, D)
    assert lq.lib.lq_encode(_c(P), 2, 200, _c(P), 25, 40, _c(P), lq.lifted_dim(200, 25, 40), None,
                            None) == lq.LQ_ERR_INVALID_ARG


def test_gemv_rejects_rows_beyond_the_plan():
    """Row lengths that are not a multiple of four words run on the mma.sync
    kernel, whose CTAs keep 64-bit partial sums for their rows in shared memory;
    row counts beyond that plan are refused before any launch (a 2^24-row
    exhaustive codebook, for instance). The tensor-core plan for K % 128 == 0
    has no such bound."""
    import bit_lifted_gemm_b200 as lq
    assert lq.gemv_workspace_size(1 << 24, 32, 1) == 0
    assert lq.lib.lq_gemv(_c(P), _c(P), 1 << 24, 32, _c(P), 1, _c(P), _c(W), BIG, None) == lq.LQ_ERR_INVALID_ARG
    assert lq.lib.lq_lift_gemv(_c(P), 0, 1, 650, None, 0, _c(P), 10, 24, _c(P), _c(P), 1 << 24, 1568,
                               _c(P), _c(P), _c(W), BIG, None) == lq.LQ_ERR_INVALID_ARG
    assert lq.gemv_workspace_size(1 << 24, 1536, 1) > 0


def test_gemv_plan_fits_every_configured_layer(monkeypatch):
    """The shape check accepts every configured decode layer and batch. The calls
    run with LQ_FAULT=launch, so they return right after their argument checks
    and never launch anything with the fake pointers, on any machine."""
    import bit_lifted_gemm_b200 as lq
    from datagen import CONFIGS
    monkeypatch.setenv("LQ_FAULT", "launch")
    for cfg in CONFIGS.values():
        if cfg.kind == "prefill":
            continue
        for batch in (1, 2, 4, 8, 16):
            ws = lq.gemv_workspace_size(cfg.out, cfg.K, batch)
            assert ws > 0, (cfg.name, batch)
            rc = lq.lib.lq_gemv(_far(0), _far(1), cfg.out, cfg.K, _far(2), batch, _far(3), _far(4), ws, None)
            assert rc == lq.LQ_ERR_CUDA, (cfg.name, batch)
            # one byte short of the workspace the plan needs is refused
            rc = lq.lib.lq_gemv(_c(P), _c(P), cfg.out, cfg.K, _c(P), batch, _c(P), _c(W), ws - 1, None)
            assert rc == lq.LQ_ERR_INVALID_ARG, (cfg.name, batch)


def test_outputs_may_not_overlap_other_buffers(monkeypatch):
    """Every entry point refuses, before any launch, an output range that shares a
    byte with an input or another output of the same call (sizes from the
    arguments); ranges that merely touch are fine, and inputs may share memory.
    LQ_FAULT=launch makes accepted calls return LQ_ERR_CUDA right after the
    checks, so no fake pointer is ever dereferenced."""
    import bit_lifted_gemm_b200 as lq
    monkeypatch.setenv("LQ_FAULT", "launch")
    base = 1 << 36
    INV, OK = lq.LQ_ERR_INVALID_ARG, lq.LQ_ERR_CUDA
    # pack: signs 4 x 32 bytes, packed 4 x 1 words = 16 bytes
    assert lq.lib.lq_pack_signs(_c(base), 4, 32, _c(base + 128), None) == OK       # packed right after signs
    assert lq.lib.lq_pack_signs(_c(base), 4, 32, _c(base + 112), None) == INV      # last 16 bytes of signs
    assert lq.lib.lq_unpack_signs(_c(base), 4, 32, _c(base + 16), None) == OK
    assert lq.lib.lq_unpack_signs(_c(base + 16), 4, 32, _c(base), None) == INV     # signs cover packed
    # lift: a fp32 [2][640] = 5120 B, M 10 x 24 fp32, u fp32 [2][1536] = 12288 B
    lift = lambda a, M, u: lq.lib.lq_lift_activations(_c(a), 0, 2, 640, None, 0, _c(M), 10, 24, _c(u), 0, 1536, None)
    assert lift(base, 2 * base, base + 5120) == OK
    assert lift(base, 2 * base, base) == INV                                      # in place
    assert lift(base, base + 5120, 2 * base) == OK                                # inputs adjacent
    assert lift(base, 2 * base, 2 * base + 944) == INV                            # u covers the end of M (960 B)
    # Kronecker lift: u over q2
    kron = lambda u: lq.lib.lq_lift_activations_kron(_c(base), 0, 1, 640, None, _c(2 * base), 8, _c(3 * base), 80,
                                                      None, _c(4 * base), 10, 24, _c(u), 0, 1536, None)
    assert kron(5 * base) == OK
    assert kron(3 * base + 16) == INV
    # GEMV: o [1][8] fp32 against u [1][64]; the workspace range is what the plan needs
    ws = lq.gemv_workspace_size(8, 64, 1)
    gemv = lambda o, w: lq.lib.lq_gemv(_c(base), _c(2 * base), 8, 64, _c(3 * base), 1, _c(o), _c(w), BIG, None)
    assert gemv(4 * base, 5 * base) == OK
    assert gemv(3 * base + 224, 5 * base) == INV                                  # o over the end of u (256 B)
    assert gemv(4 * base, 4 * base + 16) == INV                                   # workspace over o
    assert gemv(4 * base, 4 * base + 256) == OK                                   # workspace right after o (32 B)
    assert lq.lib.lq_gemv_noalloc(_c(base), _c(2 * base), 8, 64, _c(3 * base), 1, _c(base), None) == INV
    # lift + GEMV: u over a, o over the workspace
    lg = lambda u, o, w: lq.lib.lq_lift_gemv(_c(base), 0, 1, 640, None, 0, _c(2 * base), 10, 24, _c(3 * base),
                                              _c(4 * base), 8, 1536, _c(u), _c(o), _c(w), BIG, None)
    assert lg(5 * base, 6 * base, 7 * base) == OK
    assert lg(base + 1024, 6 * base, 7 * base) == INV
    assert lg(5 * base, 7 * base, 7 * base) == INV
    # GEMM: o over the packed signs; encode: err over packed
    assert lq.lib.lq_gemm(_c(base), _c(2 * base), 8, 64, _c(3 * base), 4, _c(4 * base), None) == OK
    assert lq.lib.lq_gemm(_c(base), _c(2 * base), 8, 64, _c(3 * base), 4, _c(base), None) == INV
    enc = lambda packed, err: lq.lib.lq_encode(_c(base), 4, 40, _c(2 * base), 4, 12, _c(packed), 128, _c(err), None)
    assert enc(3 * base, 4 * base) == OK
    assert enc(3 * base, 3 * base + 48) == INV                                    # packed is 4 x 16 bytes
    assert enc(3 * base, 3 * base + 64) == OK
