"""Thin Python binding of libbsattn (include/bsattn.h).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels. torch supplies device memory and the current stream. The functions named
``bsa_*`` mirror the C entry points one to one and take torch tensors; the lower-case
helpers (``build_mask``, ``precompute``, ``route``, ``forward``) allocate the outputs
and workspace with torch and call them.

If the shared library is missing or cannot be loaded, every call raises: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_BAD_CSR, ERR_TIMEOUT, ERR_WORKSPACE, \
    ERR_CAPACITY, ERR_SCRATCH_LIMIT, ERR_BAD_PADDING = range(10)
NOALLOC_SCRATCH_BYTES = 16 << 20
MODE_KEEP_OR_DROP, MODE_PISA, MODE_PISA_BLOCK = 0, 1, 2
CALL_BUILD_MASK, CALL_PRECOMPUTE, CALL_ROUTE, CALL_FORWARD = 0, 1, 2, 3

# Every symbol include/bsattn.h declares, in header order.
EXPORTS = ("bsa_version", "bsa_status_string", "bsa_mask_blocks", "bsa_workspace_bytes",
           "bsa_build_mask", "bsa_precompute", "bsa_route", "bsa_forward",
           "bsa_forward_noalloc", "bsa_selftest_wait_timeout", "bsa_selftest_forward_timeout")


class BsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class MaskDesc(ctypes.Structure):
    _fields_ = [("n_text_blocks", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("radius", ctypes.c_int32),
                ("global_stride", ctypes.c_int32), ("global_rows_full", ctypes.c_int32)]


_lib = None
_vp, _i32, _i64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                              ctypes.c_float, ctypes.c_size_t)
_SIGS = {
    "bsa_version": (_i32, []),
    "bsa_status_string": (ctypes.c_char_p, [_i32]),
    "bsa_mask_blocks": (_i32, [ctypes.POINTER(MaskDesc)]),
    "bsa_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "bsa_build_mask": (_i32, [ctypes.POINTER(MaskDesc), _vp, _vp, _i64, _vp, _vp]),
    "bsa_precompute": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp,
                              _vp, _vp, _sz, _vp, _vp]),
    "bsa_route": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _f32, _f32,
                         _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "bsa_forward": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i64,
                           _i32, _i32, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "bsa_forward_noalloc": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
                                   _i64, _i32, _i32, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp]),
    "bsa_selftest_wait_timeout": (_i32, [_i64, _vp, _vp]),
    "bsa_selftest_forward_timeout": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                            _vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _sz,
                                            _i64, _vp, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libbsattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m piecewise_attention_diffusion_b200.build`")
        so = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(so, name)
            fn.restype = res
            fn.argtypes = args
        _lib = so
    return _lib


def status_string(code: int) -> str:
    return lib().bsa_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise BsaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _desc(desc) -> MaskDesc:
    if isinstance(desc, MaskDesc):
        return desc
    return MaskDesc(int(desc["n_text_blocks"]), int(desc["grid_h"]), int(desc["grid_w"]),
                    int(desc["radius"]), int(desc["global_stride"]),
                    int(desc.get("global_rows_full", 0)))


# ------------------------------------------------------------------ C entry points
def bsa_version() -> int:
    return int(lib().bsa_version())


def bsa_mask_blocks(desc) -> int:
    d = _desc(desc)
    return int(lib().bsa_mask_blocks(ctypes.byref(d)))


def bsa_workspace_bytes(call: int, Bt: int, H: int, L: int, d: int, block: int) -> int:
    return int(lib().bsa_workspace_bytes(call, Bt, H, L, d, block))


def bsa_build_mask(desc, row_ptr, col_idx, status=None, stream=None):
    d = _desc(desc)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(col_idx, torch.int32, "col_idx")
    _check(lib().bsa_build_mask(ctypes.byref(d), _ptr(row_ptr), _ptr(col_idx),
                                col_idx.numel(), _ptr(status), _stream(stream)),
           "bsa_build_mask")


def _bhld(x, name):
    _need(x, torch.bfloat16, name)
    if x.dim() != 4:
        raise ValueError(f"{name} must be [Bt, H, L, d]")
    return x.shape


def _key_valid(key_valid, L, block):
    """Check the per-block real-token counts (int32[L/block], shared by all heads)."""
    if key_valid is not None:
        _need(key_valid, torch.int32, "key_valid", (L // block,))
    return _ptr(key_valid)


def bsa_precompute(K, V, block, kbar, vsum, Hbar, Mnorm, Hblk=None, workspace=None,
                   status=None, stream=None, key_valid=None):
    Bt, H, L, d = _bhld(K, "K")
    _need(V, torch.bfloat16, "V", K.shape)
    M = L // block
    _need(kbar, torch.float32, "kbar", (Bt * H, M, d))
    _need(vsum, torch.float32, "vsum", (Bt * H, M, d))
    _need(Hbar, torch.float32, "Hbar", (Bt * H, d, d))
    _need(Mnorm, torch.float32, "Mnorm", (Bt * H, M))
    if Hblk is not None:
        _need(Hblk, torch.float32, "Hblk", (Bt * H, M, d, d))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bsa_precompute(_ptr(K), _ptr(V), Bt, H, L, d, block,
                                _key_valid(key_valid, L, block), _ptr(kbar), _ptr(vsum),
                                _ptr(Hbar), _ptr(Mnorm), _ptr(Hblk), _ptr(workspace), ws_bytes,
                                _ptr(status), _stream(stream)), "bsa_precompute")


def bsa_route(Q, kbar, Mnorm, block, k_top, lam, scale, row_ptr, col_idx, scores=None,
              workspace=None, status=None, stream=None, key_valid=None):
    Bt, H, L, d = _bhld(Q, "Q")
    M = L // block
    _need(kbar, torch.float32, "kbar", (Bt * H, M, d))
    _need(Mnorm, torch.float32, "Mnorm", (Bt * H, M))
    _need(row_ptr, torch.int32, "row_ptr", (Bt * H * (M + 1),))
    _need(col_idx, torch.int32, "col_idx", (Bt * H * M * k_top,))
    if scores is not None:
        _need(scores, torch.float32, "scores", (Bt * H, M, M))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bsa_route(_ptr(Q), _ptr(kbar), _ptr(Mnorm), Bt, H, L, d, block,
                           _key_valid(key_valid, L, block), k_top,
                           float(lam), float(scale), _ptr(row_ptr), _ptr(col_idx),
                           _ptr(scores), _ptr(workspace), ws_bytes, _ptr(status),
                           _stream(stream)), "bsa_route")


def bsa_forward(Q, K, V, block, row_ptr, col_idx, csr_per_head, mode, kbar, vsum, Hbar, scale,
                O, lse=None, workspace=None, status=None, stream=None, key_valid=None):
    Bt, H, L, d = _bhld(Q, "Q")
    _need(K, torch.bfloat16, "K", Q.shape)
    _need(V, torch.bfloat16, "V", Q.shape)
    _need(O, torch.bfloat16, "O", Q.shape)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(col_idx, torch.int32, "col_idx")
    M = L // block
    if mode == MODE_PISA:
        _need(kbar, torch.float32, "kbar", (Bt * H, M, d))
        _need(vsum, torch.float32, "vsum", (Bt * H, M, d))
        _need(Hbar, torch.float32, "Hbar", (Bt * H, d, d))
    if lse is not None:
        _need(lse, torch.float32, "lse", (Bt * H, L))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bsa_forward(_ptr(Q), _ptr(K), _ptr(V), Bt, H, L, d, block,
                             _key_valid(key_valid, L, block), _ptr(row_ptr), _ptr(col_idx),
                             col_idx.numel(), int(csr_per_head), int(mode),
                             _ptr(kbar), _ptr(vsum), _ptr(Hbar), float(scale), _ptr(O),
                             _ptr(lse), _ptr(workspace), ws_bytes, _ptr(status),
                             _stream(stream)), "bsa_forward")


def bsa_forward_noalloc(Q, K, V, block, row_ptr, col_idx, csr_per_head, mode, kbar, vsum, Hbar,
                        scale, O, lse=None, status=None, stream=None, key_valid=None):
    """bsa_forward without a workspace argument: the library's built-in device scratch
    array is used instead, for callers that cannot allocate device memory."""
    Bt, H, L, d = _bhld(Q, "Q")
    _need(K, torch.bfloat16, "K", Q.shape)
    _need(V, torch.bfloat16, "V", Q.shape)
    _need(O, torch.bfloat16, "O", Q.shape)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(col_idx, torch.int32, "col_idx")
    M = L // block
    if mode == MODE_PISA:
        _need(kbar, torch.float32, "kbar", (Bt * H, M, d))
        _need(vsum, torch.float32, "vsum", (Bt * H, M, d))
        _need(Hbar, torch.float32, "Hbar", (Bt * H, d, d))
    if lse is not None:
        _need(lse, torch.float32, "lse", (Bt * H, L))
    _check(lib().bsa_forward_noalloc(_ptr(Q), _ptr(K), _ptr(V), Bt, H, L, d, block,
                                     _key_valid(key_valid, L, block), _ptr(row_ptr),
                                     _ptr(col_idx), col_idx.numel(),
                                     int(csr_per_head), int(mode), _ptr(kbar), _ptr(vsum),
                                     _ptr(Hbar), float(scale), _ptr(O), _ptr(lse),
                                     _ptr(status), _stream(stream)), "bsa_forward_noalloc")


def bsa_selftest_wait_timeout(timeout_ns, status, stream=None):
    """Launch the bounded-wait self-test: the kernel's wait runs out after timeout_ns and
    BSA_ERR_TIMEOUT is written to `status` (device int32)."""
    _need(status, torch.int32, "status")
    _check(lib().bsa_selftest_wait_timeout(int(timeout_ns), _ptr(status), _stream(stream)),
           "bsa_selftest_wait_timeout")


def bsa_selftest_forward_timeout(Q, K, V, block, row_ptr, col_idx, mode, kbar, vsum, Hbar, O,
                                 workspace, wait_ns, status, stream=None):
    """bsa_forward (per-head lists) with every bounded wait of the attention kernel limited
    to wait_ns: the kernel's abort and drain path, reported as BSA_ERR_TIMEOUT in `status`."""
    Bt, H, L, d = _bhld(Q, "Q")
    _need(K, torch.bfloat16, "K", Q.shape)
    _need(V, torch.bfloat16, "V", Q.shape)
    _need(O, torch.bfloat16, "O", Q.shape)
    _need(row_ptr, torch.int32, "row_ptr")
    _need(col_idx, torch.int32, "col_idx")
    _need(status, torch.int32, "status")
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().bsa_selftest_forward_timeout(
        _ptr(Q), _ptr(K), _ptr(V), Bt, H, L, d, block, _ptr(row_ptr), _ptr(col_idx),
        col_idx.numel(), int(mode), _ptr(kbar), _ptr(vsum), _ptr(Hbar), _ptr(O),
        _ptr(workspace), ws_bytes, int(wait_ns), _ptr(status), _stream(stream)),
        "bsa_selftest_forward_timeout")


# ------------------------------------------------------------ allocating helpers
def workspace(call, Bt, H, L, d, block, device="cuda"):
    n = bsa_workspace_bytes(call, Bt, H, L, d, block)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def build_mask(desc, device="cuda", status=None):
    """Return (row_ptr int32[M+1], col_idx int32[nnz]) on `device`."""
    M = bsa_mask_blocks(desc)
    if M < 0:
        raise BsaError(ERR_INVALID_ARG, "build_mask")
    row_ptr = torch.empty(M + 1, dtype=torch.int32, device=device)
    col_idx = torch.empty(M * M, dtype=torch.int32, device=device)
    bsa_build_mask(desc, row_ptr, col_idx, status=status)
    nnz = int(row_ptr[-1].item())
    return row_ptr, col_idx[:nnz].clone()


def precompute(K, V, block, want_blocks=False, status=None, ws=None, key_valid=None):
    Bt, H, L, d = K.shape
    BH, M = Bt * H, L // block
    f = dict(dtype=torch.float32, device=K.device)
    out = dict(kbar=torch.empty(BH, M, d, **f), vsum=torch.empty(BH, M, d, **f),
               Hbar=torch.empty(BH, d, d, **f), Mnorm=torch.empty(BH, M, **f))
    out["Hblk"] = torch.empty(BH, M, d, d, **f) if want_blocks else None
    if ws is None:
        ws = workspace(CALL_PRECOMPUTE, Bt, H, L, d, block, K.device)
    bsa_precompute(K, V, block, out["kbar"], out["vsum"], out["Hbar"], out["Mnorm"],
                   out["Hblk"], ws, status, key_valid=key_valid)
    return out


def route(Q, kbar, Mnorm, block, k_top, lam=1.0, scale=0.0, want_scores=False, status=None,
          key_valid=None, ws=None):
    Bt, H, L, d = Q.shape
    BH, M = Bt * H, L // block
    row_ptr = torch.empty(BH * (M + 1), dtype=torch.int32, device=Q.device)
    col_idx = torch.empty(BH * M * k_top, dtype=torch.int32, device=Q.device)
    scores = torch.empty(BH, M, M, dtype=torch.float32, device=Q.device) if want_scores \
        else None
    if ws is None:
        ws = workspace(CALL_ROUTE, Bt, H, L, d, block, Q.device)
    bsa_route(Q, kbar, Mnorm, block, k_top, lam, scale, row_ptr, col_idx, scores, ws, status,
              key_valid=key_valid)
    return row_ptr, col_idx, scores


def forward(Q, K, V, block, row_ptr, col_idx, csr_per_head, mode, stats=None, scale=0.0,
            want_lse=False, status=None, ws=None, out=None, key_valid=None):
    Bt, H, L, d = Q.shape
    O = torch.empty_like(Q) if out is None else out
    lse = torch.empty(Bt * H, L, dtype=torch.float32, device=Q.device) if want_lse else None
    if ws is None:
        ws = workspace(CALL_FORWARD, Bt, H, L, d, block, Q.device)
    st = stats or {}
    bsa_forward(Q, K, V, block, row_ptr, col_idx, csr_per_head, mode, st.get("kbar"),
                st.get("vsum"), st.get("Hbar"), scale, O, lse, ws, status, key_valid=key_valid)
    return O, lse


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
