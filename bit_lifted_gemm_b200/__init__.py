"""Python binding of liblq.so, the C-ABI LiftQuant layer for B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream. There is
no fallback: if liblq.so is missing or cannot be loaded, import fails loudly.

    o = diag(s) . W_q . (blockdiag(M^T) . T^{-1} . a)

Entry points (same names as include/lq.h, minus the `lq_` prefix):
    lifted_dim, pack_signs, unpack_signs, lift_activations,
    lift_activations_kron, gemv_workspace_size, gemv, lift_gemv, gemm, encode,
    get_device_status (lq_selftest_wait_timeout is reached through `lib`)
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# LQ_DEBUG=1 selects the debug build (device-side bounds checks, LQ_ERR_BOUNDS)
DEBUG = os.environ.get("LQ_DEBUG", "") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "liblq_debug.so" if DEBUG else "liblq.so")

LQ_OK, LQ_ERR_INVALID_ARG, LQ_ERR_UNSUPPORTED, LQ_ERR_CUDA, LQ_ERR_TIMEOUT, LQ_ERR_TOO_LARGE = 0, 1, 2, 3, 4, 5
LQ_ERR_BOUNDS = 6
LQ_F32, LQ_BF16 = 0, 1
GEMV_NOALLOC_SCRATCH_BYTES = 4 << 20  # LQ_GEMV_NOALLOC_SCRATCH_BYTES of include/lq.h

SYMBOLS = ("lq_status_str", "lq_lifted_dim", "lq_pack_signs", "lq_unpack_signs", "lq_lift_activations",
           "lq_lift_activations_kron", "lq_gemv_workspace_size", "lq_gemv", "lq_gemv_noalloc", "lq_lift_gemv",
           "lq_gemm", "lq_encode", "lq_selftest_wait_timeout", "lq_selftest_bounds", "lq_is_debug_build",
           "lq_get_device_status")


class LQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        how = "python bit_lifted_gemm_b200/build.py" + (" --debug" if DEBUG else "")
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run `{how}`")
    lib = ctypes.CDLL(LIB_PATH)
    p, i = ctypes.c_void_p, ctypes.c_int
    lib.lq_status_str.restype = ctypes.c_char_p
    lib.lq_status_str.argtypes = [i]
    lib.lq_lifted_dim.restype = i
    lib.lq_lifted_dim.argtypes = [i, i, i]
    lib.lq_pack_signs.restype = i
    lib.lq_pack_signs.argtypes = [p, i, i, p, p]
    lib.lq_unpack_signs.restype = i
    lib.lq_unpack_signs.argtypes = [p, i, i, p, p]
    lib.lq_lift_activations.restype = i
    lib.lq_lift_activations.argtypes = [p, i, i, i, p, i, p, i, i, p, i, i, p]
    lib.lq_lift_activations_kron.restype = i
    lib.lq_lift_activations_kron.argtypes = [p, i, i, i, p, p, i, p, i, p, p, i, i, p, i, i, p]
    z = ctypes.c_size_t
    lib.lq_gemv_workspace_size.restype = z
    lib.lq_gemv_workspace_size.argtypes = [i, i, i]
    lib.lq_gemv.restype = i
    lib.lq_gemv.argtypes = [p, p, i, i, p, i, p, p, z, p]
    lib.lq_gemv_noalloc.restype = i
    lib.lq_gemv_noalloc.argtypes = [p, p, i, i, p, i, p, p]
    lib.lq_lift_gemv.restype = i
    lib.lq_lift_gemv.argtypes = [p, i, i, i, p, i, p, i, i, p, p, i, i, p, p, p, z, p]
    lib.lq_gemm.restype = i
    lib.lq_encode.restype = i
    lib.lq_selftest_wait_timeout.restype = i
    lib.lq_selftest_wait_timeout.argtypes = [ctypes.c_uint, p]
    lib.lq_selftest_bounds.restype = i
    lib.lq_selftest_bounds.argtypes = [p]
    lib.lq_is_debug_build.restype = i
    lib.lq_is_debug_build.argtypes = []
    lib.lq_encode.argtypes = [p, i, i, p, i, i, p, i, p, p]
    lib.lq_gemm.argtypes = [p, p, i, i, p, i, p, p]
    lib.lq_get_device_status.restype = i
    lib.lq_get_device_status.argtypes = [p]
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.lq_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != LQ_OK:
        raise LQError(status, where)


def lifted_dim(in_dim: int, d: int, D: int) -> int:
    return int(lib.lq_lifted_dim(in_dim, d, D))


# ------------------------------------------------------------------ torch helpers

def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev_tensor(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return t


def pack_signs(signs, out=None, stream=None):
    """int8 +-1 [out][K] (CUDA) -> packed words [out][K/32] (int32 storage of uint32)."""
    import torch
    _dev_tensor(signs, "signs")
    rows, K = signs.shape
    if out is None:
        out = torch.empty((rows, K // 32), dtype=torch.int32, device=signs.device)
    _check(lib.lq_pack_signs(_ptr(signs), rows, K, _ptr(out), _stream(stream)), "lq_pack_signs")
    return out


def unpack_signs(packed, K, out=None, stream=None):
    import torch
    _dev_tensor(packed, "packed")
    rows = packed.shape[0]
    if out is None:
        out = torch.empty((rows, K), dtype=torch.int8, device=packed.device)
    _check(lib.lq_unpack_signs(_ptr(packed), rows, K, _ptr(out), _stream(stream)), "lq_unpack_signs")
    return out


def lift_activations(a, M, K, tinv=None, u_dtype="f32", out=None, stream=None):
    """a [batch][in] (float32 or bfloat16) -> u [batch][K] (float32 or bfloat16)."""
    import torch
    _dev_tensor(a, "a")
    _dev_tensor(M, "M")
    batch, in_dim = a.shape
    d, D = M.shape
    a_t = LQ_BF16 if a.dtype == torch.bfloat16 else LQ_F32
    u_t = LQ_BF16 if u_dtype in ("bf16", torch.bfloat16) else LQ_F32
    if out is None:
        out = torch.empty((batch, K), dtype=torch.bfloat16 if u_t == LQ_BF16 else torch.float32, device=a.device)
    tblk = 0 if tinv is None else int(tinv.shape[-1])
    if tinv is not None:
        _dev_tensor(tinv, "tinv")
    _check(lib.lq_lift_activations(_ptr(a), a_t, batch, in_dim, _ptr(tinv), tblk, _ptr(M), d, D, _ptr(out), u_t,
                                   K, _stream(stream)), "lq_lift_activations")
    return out


def lift_activations_kron(a, q1, q2, M, K, r1=None, r2=None, u_dtype="f32", out=None, stream=None):
    """Lift with the Kronecker-factored whitening a' = diag(r2) (q1 kron q2) diag(r1) a.

    a [batch][in] (float32 or bfloat16), q1 [n1][n1], q2 [n2][n2] with in = n1 * n2,
    r1 [in] or None, r2 [in/d] or None -> u [batch][K] (float32 or bfloat16)."""
    import torch
    for t, name in ((a, "a"), (q1, "q1"), (q2, "q2"), (M, "M")):
        _dev_tensor(t, name)
    for t, name in ((r1, "r1"), (r2, "r2")):
        if t is not None:
            _dev_tensor(t, name)
    batch, in_dim = a.shape
    d, D = M.shape
    a_t = LQ_BF16 if a.dtype == torch.bfloat16 else LQ_F32
    u_t = LQ_BF16 if u_dtype in ("bf16", torch.bfloat16) else LQ_F32
    if out is None:
        out = torch.empty((batch, K), dtype=torch.bfloat16 if u_t == LQ_BF16 else torch.float32, device=a.device)
    _check(lib.lq_lift_activations_kron(_ptr(a), a_t, batch, in_dim, _ptr(r1), _ptr(q1), int(q1.shape[0]), _ptr(q2),
                                        int(q2.shape[0]), _ptr(r2), _ptr(M), d, D, _ptr(out), u_t, K,
                                        _stream(stream)), "lq_lift_activations_kron")
    return out


def gemv_workspace_size(out_rows: int, K: int, batch: int) -> int:
    """Bytes of device scratch lq_gemv / lq_lift_gemv need (0: shape not supported)."""
    return int(lib.lq_gemv_workspace_size(out_rows, K, batch))


def gemv_workspace(out_rows: int, K: int, batch: int, device=None):
    """A device scratch tensor big enough for lq_gemv / lq_lift_gemv on this shape
    (256-byte aligned: the caching allocator hands out 512-byte aligned blocks)."""
    import torch
    n = gemv_workspace_size(out_rows, K, batch)
    if n == 0:
        raise LQError(LQ_ERR_INVALID_ARG, "lq_gemv_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def _workspace(ws, out_rows, K, batch, device):
    if ws is None:
        ws = gemv_workspace(out_rows, K, batch, device)
    _dev_tensor(ws, "workspace")
    return ws


def gemv(packed, s, u, out=None, workspace=None, stream=None):
    """Decode: packed [out][K/32], s [out], u fp32 [batch][K] (batch <= 16) -> o fp32 [batch][out].

    `workspace` (uint8 CUDA tensor of gemv_workspace_size bytes) is allocated
    when not given; calls that share one must run on the same stream."""
    import torch
    _dev_tensor(packed, "packed")
    _dev_tensor(s, "s")
    _dev_tensor(u, "u")
    rows = packed.shape[0]
    batch, K = u.shape
    if out is None:
        out = torch.empty((batch, rows), dtype=torch.float32, device=u.device)
    _dev_tensor(out, "out")
    ws = _workspace(workspace, rows, K, batch, u.device)
    _check(lib.lq_gemv(_ptr(packed), _ptr(s), rows, K, _ptr(u), batch, _ptr(out), _ptr(ws), ws.numel(),
                       _stream(stream)), "lq_gemv")
    return out


def _dev_or_pinned(t, name):
    if not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor or pinned host tensor")
    return t


def lift_gemv(a, M, packed, s, K, tinv=None, u=None, out=None, workspace=None, stream=None):
    """Fused decode step: a [batch][in] (float32 or bfloat16) -> (u fp32 [batch][K], o fp32 [batch][out]).

    `a` and `out` may be pinned host tensors (zero-copy: the kernels read and
    write them across the host link); everything else lives on the device."""
    import torch
    _dev_or_pinned(a, "a")
    _dev_tensor(M, "M")
    _dev_tensor(packed, "packed")
    _dev_tensor(s, "s")
    batch, in_dim = a.shape
    d, D = M.shape
    rows = packed.shape[0]
    a_t = LQ_BF16 if a.dtype == torch.bfloat16 else LQ_F32
    if u is None:
        u = torch.empty((batch, K), dtype=torch.float32, device=M.device)
    if out is None:
        out = torch.empty((batch, rows), dtype=torch.float32, device=M.device)
    _dev_tensor(u, "u")
    _dev_or_pinned(out, "out")
    tblk = 0 if tinv is None else int(tinv.shape[-1])
    if tinv is not None:
        _dev_tensor(tinv, "tinv")
    ws = _workspace(workspace, rows, K, batch, M.device)
    _check(lib.lq_lift_gemv(_ptr(a), a_t, batch, in_dim, _ptr(tinv), tblk, _ptr(M), d, D, _ptr(packed), _ptr(s),
                            rows, K, _ptr(u), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "lq_lift_gemv")
    return u, out


def gemm(packed, s, u, out=None, stream=None):
    """Prefill: packed [out][K/32], s [out], u bf16 [tokens][K] -> o fp32 [tokens][out]."""
    import torch
    _dev_tensor(packed, "packed")
    _dev_tensor(s, "s")
    _dev_tensor(u, "u")
    rows = packed.shape[0]
    tokens, K = u.shape
    if out is None:
        out = torch.empty((tokens, rows), dtype=torch.float32, device=u.device)
    _dev_tensor(out, "out")
    _check(lib.lq_gemm(_ptr(packed), _ptr(s), rows, K, _ptr(u), tokens, _ptr(out), _stream(stream)), "lq_gemm")
    return out


def encode(w, M, K, err=False, out=None, stream=None):
    """Encoder: weights w [rows][in] fp32, M [d][D] -> packed signs [rows][K/32]
    (int32 storage of uint32), and the per-block squared errors [rows][in/d] when
    err=True."""
    import torch
    _dev_tensor(w, "w")
    _dev_tensor(M, "M")
    rows, in_dim = w.shape
    d, D = M.shape
    if out is None:
        out = torch.empty((rows, K // 32), dtype=torch.int32, device=w.device)
    e = torch.empty((rows, in_dim // d), dtype=torch.float32, device=w.device) if err else None
    _check(lib.lq_encode(_ptr(w), rows, in_dim, _ptr(M), d, D, _ptr(out), K, _ptr(e), _stream(stream)), "lq_encode")
    return (out, e) if err else out


def get_device_status(stream=None) -> int:
    return int(lib.lq_get_device_status(_stream(stream)))
