"""Python binding of libcsa -- hybrid compressed attention (CSA / HCA) on B200.

A thin ctypes layer over the C ABI declared in ``include/csa.h``: it checks
dtypes, devices and contiguity of torch tensors, passes their device pointers
and the current CUDA stream, and raises :class:`CsaError` on a non-zero
return code.  Every step of the computation runs in the library's CUDA
kernels; there is no Python or CPU fallback.  If ``libcsa.so`` has not been
built, loading fails with an error that says so.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# the library to load: libcsa.so, or another build (the CSA_CHECK build
# libcsa_check.so) named by the CSA_LIBRARY environment variable
LIB_PATH = os.environ.get("CSA_LIBRARY") or os.path.join(_HERE, "libcsa.so")

CSA_OK = 0
CSA_ERR_INVALID = -1
CSA_ERR_UNSUPPORTED = -2
CSA_ERR_CUDA = -3
CSA_ERR_TIMEOUT = -4
CSA_ERR_WORKSPACE = -5
CSA_ERR_CHECK = -6

# every symbol declared in include/csa.h
SYMBOLS = (
    "csa_compress",
    "csa_compress_ew",
    "csa_index_topk_workspace",
    "csa_index_topk",
    "csa_index_topk_noalloc",
    "csa_index_topk_mx_workspace",
    "csa_index_topk_mx",
    "csa_check_topk",
    "csa_check_build",
    "csa_attend_workspace",
    "csa_attend",
    "hca_attend_workspace",
    "hca_attend",
    "csa_last_error",
    "csa_sync_status",
    "csa_version",
    "csa_launch_count",
    "csa_quantize_mxfp4",
    "csa_selftest_timeout",
    "csa_decode_step_workspace",
    "csa_decode_step",
)


class CsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libcsa error {code}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    """Mirror of ``csa_dims`` in include/csa.h."""

    _fields_ = [
        ("B", ctypes.c_int32), ("Tq", ctypes.c_int32), ("H", ctypes.c_int32),
        ("D", ctypes.c_int32), ("HI", ctypes.c_int32), ("dI", ctypes.c_int32),
        ("K", ctypes.c_int32), ("W", ctypes.c_int32), ("m", ctypes.c_int32),
        ("n_entries", ctypes.c_int32), ("entry_cap", ctypes.c_int64),
        ("win_cap", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
    ]

    def __init__(self, B=1, Tq=1, H=1, D=512, HI=4, dI=64, K=512, W=128, m=4, n_entries=0,
                 entry_cap=None, win_cap=None, softmax_scale=1.0):
        super().__init__(B, Tq, H, D, HI, dI, K, W, m, n_entries,
                         n_entries if entry_cap is None else entry_cap,
                         W if win_cap is None else win_cap, softmax_scale)


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libcsa.so once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libcsa.so not built at {LIB_PATH}: run "
                          "`python -m compressed_sparse_attention_16_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.csa_compress.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _I64, _P, _P, _I64, _I64, _I32, _P, _P]
    L.csa_compress.restype = ctypes.c_int
    L.csa_compress_ew.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _I64, _P, _P, _I64, _I64, _I32, _P, _P, _I64,
                                  _I64, _I32, _P, _P]
    L.csa_compress_ew.restype = ctypes.c_int
    L.csa_index_topk_workspace.argtypes = [ctypes.POINTER(Dims)]
    L.csa_index_topk_workspace.restype = _SZ
    L.csa_index_topk.argtypes = [_P, _P, _P, _P, ctypes.POINTER(Dims), _P, _P, _P, _SZ, _P]
    L.csa_index_topk.restype = ctypes.c_int
    L.csa_index_topk_noalloc.argtypes = [_P, _P, _P, _P, ctypes.POINTER(Dims), _P, _P, _P]
    L.csa_index_topk_noalloc.restype = ctypes.c_int
    L.csa_index_topk_mx_workspace.argtypes = [ctypes.POINTER(Dims)]
    L.csa_index_topk_mx_workspace.restype = _SZ
    L.csa_index_topk_mx.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Dims), _P, _P, _P, _SZ, _P]
    L.csa_index_topk_mx.restype = ctypes.c_int
    L.csa_check_topk.argtypes = [_P, _P, _P, ctypes.POINTER(Dims), _P]
    L.csa_check_topk.restype = ctypes.c_int
    L.csa_check_build.argtypes = []
    L.csa_check_build.restype = ctypes.c_int
    for name in ("csa_attend_workspace", "hca_attend_workspace"):
        getattr(L, name).argtypes = [ctypes.POINTER(Dims)]
        getattr(L, name).restype = _SZ
    L.csa_attend.argtypes = [_P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(Dims), _P, _P, _P, _SZ, _P]
    L.csa_attend.restype = ctypes.c_int
    L.hca_attend.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Dims), _P, _P, _P, _SZ, _P]
    L.hca_attend.restype = ctypes.c_int
    L.csa_last_error.argtypes = []
    L.csa_last_error.restype = ctypes.c_char_p
    L.csa_sync_status.argtypes = [_P]
    L.csa_sync_status.restype = ctypes.c_int
    L.csa_version.argtypes = []
    L.csa_version.restype = ctypes.c_int
    L.csa_launch_count.argtypes = []
    L.csa_launch_count.restype = ctypes.c_uint64
    L.csa_selftest_timeout.argtypes = [ctypes.c_uint64, _P]
    L.csa_selftest_timeout.restype = ctypes.c_int
    L.csa_quantize_mxfp4.argtypes = [_P, _I64, _I32, _P, _P, _P]
    L.csa_quantize_mxfp4.restype = ctypes.c_int
    L.csa_decode_step_workspace.argtypes = [ctypes.POINTER(Dims), _I32]
    L.csa_decode_step_workspace.restype = _SZ
    L.csa_decode_step.argtypes = [_P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(Dims),
                                  _P, _P, _P, _P, _P, _SZ, _P]
    L.csa_decode_step.restype = ctypes.c_int
    _lib = L
    return L


def _check(rc: int):
    if rc != CSA_OK:
        raise CsaError(rc, lib().csa_last_error().decode(errors="replace"))


def _ptr(t: torch.Tensor | None, dtype, name: str, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ---------------------------------------------------------------------------
# operations
# ---------------------------------------------------------------------------


def compress(x: torch.Tensor, z: torch.Tensor, m: int, codes: torch.Tensor, scales: torch.Tensor,
             dst_first: int = 0, ring_cap: int = 0, pooled: torch.Tensor | None = None,
             T: int | None = None, first_token: int = 0, stream=None) -> None:
    """csa_compress: pool full m-token blocks of tokens [first_token, first_token + T)
    of x, z [B, Ttot, D] into codes u8 [B, cap, D] / scales f32 [B, cap] at slots
    dst_first + i (no copy of the token range is made)."""
    if x.dim() != 3 or z.shape != x.shape:
        raise ValueError("x and z must be [B, T, D] of equal shape")
    B, Ttot, D = x.shape
    T = Ttot - first_token if T is None else T
    if first_token < 0 or first_token + T > Ttot:
        raise ValueError("token range outside x")
    if codes.dim() != 3 or codes.shape[0] != B or codes.shape[2] != D or scales.shape != codes.shape[:2]:
        raise ValueError("codes must be [B, cap, D] and scales [B, cap]")
    dev = x.device
    off = first_token * D * 4
    _check(lib().csa_compress(_ptr(x, torch.float32, "x") + off, _ptr(z, torch.float32, "z", dev) + off,
                              B, T, D, m, Ttot * D,
                              _ptr(codes, torch.uint8, "codes", dev), _ptr(scales, torch.float32, "scales", dev),
                              dst_first, codes.shape[1], ring_cap,
                              _ptr(pooled, torch.float32, "pooled", dev), _stream(stream)))


def compress_ew(x: torch.Tensor, z: torch.Tensor, m: int, codes: torch.Tensor, scales: torch.Tensor,
                win_codes: torch.Tensor, win_scales: torch.Tensor, dst_first: int = 0, ring_cap: int = 0,
                win_first: int = 0, win_ring_cap: int = 0, pooled: torch.Tensor | None = None,
                T: int | None = None, first_token: int = 0, stream=None) -> None:
    """csa_compress_ew: the m-token entries of tokens [first_token, first_token + T)
    of x, z [B, Ttot, D] (as compress) and every one of those tokens as a
    window entry (compress with m = 1), in one pass."""
    if x.dim() != 3 or z.shape != x.shape:
        raise ValueError("x and z must be [B, T, D] of equal shape")
    B, Ttot, D = x.shape
    T = Ttot - first_token if T is None else T
    if first_token < 0 or first_token + T > Ttot:
        raise ValueError("token range outside x")
    for c, s_, what in ((codes, scales, "codes"), (win_codes, win_scales, "win_codes")):
        if c.dim() != 3 or c.shape[0] != B or c.shape[2] != D or s_.shape != c.shape[:2]:
            raise ValueError(f"{what} must be [B, cap, D] with scales [B, cap]")
    dev = x.device
    off = first_token * D * 4
    _check(lib().csa_compress_ew(_ptr(x, torch.float32, "x") + off, _ptr(z, torch.float32, "z", dev) + off, B, T, D,
                                 m, Ttot * D,
                                 _ptr(codes, torch.uint8, "codes", dev), _ptr(scales, torch.float32, "scales", dev),
                                 dst_first, codes.shape[1], ring_cap,
                                 _ptr(win_codes, torch.uint8, "win_codes", dev),
                                 _ptr(win_scales, torch.float32, "win_scales", dev), win_first, win_codes.shape[1],
                                 win_ring_cap, _ptr(pooled, torch.float32, "pooled", dev), _stream(stream)))


def quantize_mxfp4(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    """csa_quantize_mxfp4: fp32 x [rows, cols] (cols a multiple of 32) to packed
    E2M1 codes u8 [rows, cols/2] and E8M0 block scales u8 [rows, cols/32]."""
    if x.dim() != 2:
        raise ValueError("x must be [rows, cols]")
    rows, cols = x.shape
    if codes.shape != (rows, cols // 2) or scales.shape != (rows, cols // 32):
        raise ValueError("codes must be [rows, cols/2] and scales [rows, cols/32]")
    dev = x.device
    _check(lib().csa_quantize_mxfp4(_ptr(x, torch.float32, "x"), rows, cols, _ptr(codes, torch.uint8, "codes", dev),
                                    _ptr(scales, torch.uint8, "scales", dev), _stream(stream)))


def index_topk_workspace(dims: Dims) -> int:
    return int(lib().csa_index_topk_workspace(ctypes.byref(dims)))


def index_topk_mx_workspace(dims: Dims) -> int:
    return int(lib().csa_index_topk_mx_workspace(ctypes.byref(dims)))


def check_topk(idx, score, q_pos, dims: Dims, stream=None) -> None:
    """csa_check_topk: device-side check of top-k lists; a violation is
    reported by the next sync_status() (CSA_ERR_CHECK)."""
    dev = idx.device
    _check(lib().csa_check_topk(_ptr(idx, torch.int32, "idx"), _ptr(score, torch.float32, "score", dev),
                                _ptr(q_pos, torch.int32, "q_pos", dev), ctypes.byref(dims), _stream(stream)))


def is_check_build() -> bool:
    """True when the loaded library is the CSA_CHECK build."""
    return bool(lib().csa_check_build())


def attend_workspace(dims: Dims, dense: bool = False) -> int:
    fn = lib().hca_attend_workspace if dense else lib().csa_attend_workspace
    return int(fn(ctypes.byref(dims)))


def _ws(workspace, nbytes, device):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        raise ValueError(f"this call needs a workspace of {nbytes} bytes")
    return _ptr(workspace, torch.uint8, "workspace", device), workspace.numel()


def index_topk(qI, w, kI, q_pos, dims: Dims, idx_out, score_out=None, workspace=None, stream=None):
    """csa_index_topk: indexer scores + top-k; see include/csa.h."""
    dev = qI.device
    need = index_topk_workspace(dims)
    wp, wn = _ws(workspace, need, dev)
    _check(lib().csa_index_topk(_ptr(qI, torch.uint8, "qI"), _ptr(w, torch.float32, "w", dev),
                                _ptr(kI, torch.uint8, "kI", dev), _ptr(q_pos, torch.int32, "q_pos", dev),
                                ctypes.byref(dims), _ptr(idx_out, torch.int32, "idx_out", dev),
                                _ptr(score_out, torch.float32, "score_out", dev), wp, wn, _stream(stream)))


def index_topk_noalloc(qI, w, kI, q_pos, dims: Dims, idx_out, score_out=None, stream=None):
    """csa_index_topk_noalloc: as index_topk, but the library's own fixed 8 MiB
    device scratch replaces the workspace (for callers that cannot allocate).
    Calls that overlap on the GPU share that scratch and must be serialised."""
    dev = qI.device
    _check(lib().csa_index_topk_noalloc(_ptr(qI, torch.uint8, "qI"), _ptr(w, torch.float32, "w", dev),
                                        _ptr(kI, torch.uint8, "kI", dev),
                                        _ptr(q_pos, torch.int32, "q_pos", dev), ctypes.byref(dims),
                                        _ptr(idx_out, torch.int32, "idx_out", dev),
                                        _ptr(score_out, torch.float32, "score_out", dev), _stream(stream)))


def index_topk_mx(qI, qI_scales, w, kI, kI_scales, q_pos, dims: Dims, idx_out, score_out=None, workspace=None,
                  stream=None):
    """csa_index_topk_mx: indexer + top-k on block-scaled FP4 (MXFP4) queries
    and keys; see include/csa.h."""
    dev = qI.device
    wp, wn = _ws(workspace, index_topk_mx_workspace(dims), dev)
    _check(lib().csa_index_topk_mx(_ptr(qI, torch.uint8, "qI"), _ptr(qI_scales, torch.uint8, "qI_scales", dev),
                                   _ptr(w, torch.float32, "w", dev), _ptr(kI, torch.uint8, "kI", dev),
                                   _ptr(kI_scales, torch.uint8, "kI_scales", dev),
                                   _ptr(q_pos, torch.int32, "q_pos", dev), ctypes.byref(dims),
                                   _ptr(idx_out, torch.int32, "idx_out", dev),
                                   _ptr(score_out, torch.float32, "score_out", dev), wp, wn, _stream(stream)))


def attend(q, codes, scales, idx, win_codes, win_scales, q_pos, dims: Dims, out, lse=None,
           workspace=None, stream=None):
    """csa_attend: sparse shared-KV MQA over selected entries + window."""
    dev = q.device
    wp, wn = _ws(workspace, attend_workspace(dims, False), dev)
    _check(lib().csa_attend(_ptr(q, torch.bfloat16, "q"), _ptr(codes, torch.uint8, "codes", dev),
                            _ptr(scales, torch.float32, "scales", dev), _ptr(idx, torch.int32, "idx", dev),
                            _ptr(win_codes, torch.uint8, "win_codes", dev),
                            _ptr(win_scales, torch.float32, "win_scales", dev),
                            _ptr(q_pos, torch.int32, "q_pos", dev), ctypes.byref(dims),
                            _ptr(out, torch.bfloat16, "out", dev), _ptr(lse, torch.float32, "lse", dev),
                            wp, wn, _stream(stream)))


def hca_attend(q, codes, scales, win_codes, win_scales, q_pos, dims: Dims, out, lse=None,
               workspace=None, stream=None):
    """hca_attend: dense attention over every visible entry + window."""
    dev = q.device
    wp, wn = _ws(workspace, attend_workspace(dims, True), dev)
    _check(lib().hca_attend(_ptr(q, torch.bfloat16, "q"), _ptr(codes, torch.uint8, "codes", dev),
                            _ptr(scales, torch.float32, "scales", dev),
                            _ptr(win_codes, torch.uint8, "win_codes", dev),
                            _ptr(win_scales, torch.float32, "win_scales", dev),
                            _ptr(q_pos, torch.int32, "q_pos", dev), ctypes.byref(dims),
                            _ptr(out, torch.bfloat16, "out", dev), _ptr(lse, torch.float32, "lse", dev),
                            wp, wn, _stream(stream)))


def decode_step_workspace(dims: Dims, n_new: int) -> int:
    """Bytes of workspace csa_decode_step needs (0: the shape is outside the
    fused step's set; use the separate calls)."""
    return int(lib().csa_decode_step_workspace(ctypes.byref(dims), int(n_new)))


def decode_step(x_new, z_new, kI_new, q, qI, w, q_pos, codes, scales, kI, win_codes, win_scales,
                dims: Dims, idx_out, score_out, out, lse, workspace, stream=None) -> None:
    """csa_decode_step: append x_new/z_new [B, n, D] (and kI_new [B, n/m, dI/2]
    or None), then index, select and attend for one query per sequence, in one
    launch; see include/csa.h.  `workspace` (u8, >= decode_step_workspace
    bytes) must have been zero-filled before its first use."""
    dev = q.device
    if x_new.dim() != 3 or z_new.shape != x_new.shape:
        raise ValueError("x_new and z_new must be [B, n_new, D] of equal shape")
    _check(lib().csa_decode_step(
        _ptr(x_new, torch.float32, "x_new", dev), _ptr(z_new, torch.float32, "z_new", dev), x_new.shape[1],
        _ptr(kI_new, torch.uint8, "kI_new", dev), _ptr(q, torch.bfloat16, "q", dev),
        _ptr(qI, torch.uint8, "qI", dev), _ptr(w, torch.float32, "w", dev), _ptr(q_pos, torch.int32, "q_pos", dev),
        _ptr(codes, torch.uint8, "codes", dev), _ptr(scales, torch.float32, "scales", dev),
        _ptr(kI, torch.uint8, "kI", dev), _ptr(win_codes, torch.uint8, "win_codes", dev),
        _ptr(win_scales, torch.float32, "win_scales", dev), ctypes.byref(dims),
        _ptr(idx_out, torch.int32, "idx_out", dev), _ptr(score_out, torch.float32, "score_out", dev),
        _ptr(out, torch.bfloat16, "out", dev), _ptr(lse, torch.float32, "lse", dev),
        _ptr(workspace, torch.uint8, "workspace", dev), workspace.numel() if workspace is not None else 0,
        _stream(stream)))


def sync_status(stream=None) -> None:
    """Wait for the stream and raise if a kernel flagged bad data or a timeout."""
    _check(lib().csa_sync_status(_stream(stream)))


def version() -> int:
    return int(lib().csa_version())


def selftest_timeout(limit_ns: int = 1_000_000, stream=None) -> None:
    """Run the bounded-wait diagnostic kernel (its wait always expires); the
    next sync_status() raises CsaError(CSA_ERR_TIMEOUT)."""
    _check(lib().csa_selftest_timeout(int(limit_ns), _stream(stream)))


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().csa_launch_count())
