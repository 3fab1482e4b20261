"""Python binding of the svconv C ABI (include/svconv.h).

Argument marshalling only: every step runs in libsvconv.so's CUDA kernels.
PyTorch supplies device memory and the current CUDA stream.  There is no CPU
fallback: if the library is missing or no CUDA device is present, every call
raises.

Function names match the C entry points.  Output tensors may be passed in
(``out=``-style keyword arguments); otherwise they are allocated with torch on
the input's device.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

F32, BF16, E4M3 = 0, 1, 2
OK = 0
STATUS_BAD_COORD, STATUS_DUPLICATE, STATUS_BAD_FRAME, STATUS_BAD_OFFSETS = 1, 2, 4, 8
STATUS_TIMEOUT, STATUS_BAD_INDEX, STATUS_CHUNK_OVERFLOW = 16, 32, 64

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvconv.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "svconv.h")
_lib = None


class SvconvError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({status_str(code)})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libsvconv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_convolution_pruned_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.svconv_build_index.argtypes = [P, P, I, I, I, I, P, P, P, P]
        L.svconv_fwd.argtypes = [I, P, P, I, I, I, P, P, P, P]
        L.svconv_bwd_data.argtypes = [I, P, P, I, I, I, P, P, P]
        L.svconv_bwd_weight.argtypes = [I, P, P, P, I, I, I, P, P, P, Z, P]
        L.svconv_bwd.argtypes = [I, P, P, P, I, I, I, P, P, P, P, P, Z, P]
        L.svconv_bwd.restype = I
        L.svconv_bwd_single_pass.argtypes = [P, P, P, I, P, P, P, P, P, Z, P]
        L.svconv_bwd_single_pass.restype = I
        L.svconv_bwd_single_pass_workspace_size.argtypes = [I]
        L.svconv_bwd_single_pass_workspace_size.restype = Z
        L.svconv_bwd_workspace_size.argtypes = [I, I, I, I]
        L.svconv_bwd_workspace_size.restype = Z
        L.svconv_bwd_weight_noalloc.argtypes = [I, P, P, P, I, I, I, P, P, P]
        L.svconv_bwd_weight_noalloc.restype = I
        L.svconv_bwd_weight_workspace_size.argtypes = [I, I, I, I]
        L.svconv_bwd_weight_workspace_size.restype = Z
        L.svconv_adapter_fwd.argtypes = [P, P, P, I, I, I, I, P, P, P, P, I, I, P, Z, P, P]
        L.svconv_adapter_workspace_size.argtypes = [I, I]
        L.svconv_adapter_workspace_size.restype = Z
        L.svconv_xattn_aux.argtypes = [P, I, I, P, I, I, P, I, I, P, P, Z, P, P]
        L.svconv_xattn_aux.restype = I
        L.svconv_xattn_workspace_size.argtypes = [I, I, I]
        L.svconv_xattn_workspace_size.restype = Z
        L.svconv_adapter_fwd_xattn.argtypes = [P, P, P, I, I, I, I, P, P, P, P, I, I, P, I, I, P, P, Z, P, P]
        L.svconv_adapter_fwd_xattn.restype = I
        L.svconv_adapter_xattn_workspace_size.argtypes = [I, I, I, I, I]
        L.svconv_adapter_xattn_workspace_size.restype = Z
        L.svconv_read_error_word.argtypes = [P]
        L.svconv_selftest_timeout.argtypes = [P, I, P]
        L.svconv_status_str.argtypes = [I]
        L.svconv_status_str.restype = ctypes.c_char_p
        L.svconv_version.argtypes = []
        for name in ("svconv_build_index", "svconv_fwd", "svconv_bwd_data", "svconv_bwd_weight",
                     "svconv_adapter_fwd", "svconv_read_error_word", "svconv_selftest_timeout",
                     "svconv_version"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def declared_symbols() -> list:
    """Entry points declared with SVCONV_API in include/svconv.h."""
    text = open(HEADER_PATH).read()
    return re.findall(r"SVCONV_API\s+[\w\s\*]+?\b(svconv_\w+)\s*\(", text)


def status_str(code: int) -> str:
    try:
        return lib().svconv_status_str(int(code)).decode()
    except Exception:  # pragma: no cover - message formatting only
        return "?"


def svconv_status_str(code: int) -> str:
    return status_str(code)


def svconv_version() -> int:
    return int(lib().svconv_version())


def _check(fn: str, rc: int):
    if rc != OK:
        raise SvconvError(fn, rc)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float8_e4m3fn:
        return E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("svconv operates on CUDA tensors only")
        if not t.is_contiguous():
            raise ValueError("svconv expects contiguous tensors")


def svconv_build_index(coords: torch.Tensor, frame_off: torch.Tensor, T: int, H: int, W: int, *,
                       nbr: Optional[torch.Tensor] = None, M: Optional[torch.Tensor] = None,
                       want_map: bool = False, status: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Neighbour table [n, 9] int32 (and the lookup map [T, H, W] if requested)."""
    _cuda(coords, frame_off, nbr, M, status)
    n = coords.shape[0]
    dev = coords.device
    if nbr is None:
        nbr = torch.empty((n, 9), dtype=torch.int32, device=dev)
    if M is None and want_map:
        M = torch.empty((T, H, W), dtype=torch.int32, device=dev)
    rc = lib().svconv_build_index(_ptr(coords), _ptr(frame_off), int(T), int(H), int(W), int(n), _ptr(nbr),
                                  _ptr(M), _ptr(status), _stream(coords, stream))
    _check("svconv_build_index", rc)
    return nbr, M


def svconv_fwd(X: torch.Tensor, nbr: torch.Tensor, Wt: torch.Tensor, bias: Optional[torch.Tensor] = None, *,
               Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[k] = bias + sum_j W_j X[N[k, j]]; Wt is [C_out, 9, C_in].  e4m3 X / Wt give a bf16 Y."""
    _cuda(X, nbr, Wt, bias, Y)
    n, Cin = X.shape
    Cout = Wt.shape[0]
    if Y is None:
        ydt = torch.bfloat16 if X.dtype == torch.float8_e4m3fn else X.dtype
        Y = torch.empty((n, Cout), dtype=ydt, device=X.device)
    rc = lib().svconv_fwd(_dtype_code(X), _ptr(X), _ptr(nbr), n, Cin, Cout, _ptr(Wt), _ptr(bias), _ptr(Y),
                          _stream(X, stream))
    _check("svconv_fwd", rc)
    return Y


def svconv_bwd_data(dY: torch.Tensor, nbr: torch.Tensor, Wt: torch.Tensor, *, dX: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """dX[k] = sum_j W_j^T dY[N[k, 8-j]]."""
    _cuda(dY, nbr, Wt, dX)
    n, Cout = dY.shape
    Cin = Wt.shape[2]
    if dX is None:
        dX = torch.empty((n, Cin), dtype=dY.dtype, device=dY.device)
    rc = lib().svconv_bwd_data(_dtype_code(dY), _ptr(dY), _ptr(nbr), n, Cin, Cout, _ptr(Wt), _ptr(dX),
                               _stream(dY, stream))
    _check("svconv_bwd_data", rc)
    return dX


def svconv_bwd_weight_workspace_size(dtype: int, n: int, Cin: int, Cout: int) -> int:
    return int(lib().svconv_bwd_weight_workspace_size(int(dtype), int(n), int(Cin), int(Cout)))


def svconv_bwd_weight(dY: torch.Tensor, X: torch.Tensor, nbr: torch.Tensor, *, dW: Optional[torch.Tensor] = None,
                      db: Optional[torch.Tensor] = None, want_db: bool = True,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """(dW [C_out, 9, C_in] fp32, db [C_out] fp32 or None)."""
    _cuda(dY, X, nbr, dW, db, workspace)
    n, Cout = dY.shape
    Cin = X.shape[1]
    dt = _dtype_code(X)
    if dW is None:
        dW = torch.empty((Cout, 9, Cin), dtype=torch.float32, device=X.device)
    if db is None and want_db:
        db = torch.empty((Cout,), dtype=torch.float32, device=X.device)
    need = svconv_bwd_weight_workspace_size(dt, n, Cin, Cout)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    rc = lib().svconv_bwd_weight(dt, _ptr(dY), _ptr(X), _ptr(nbr), n, Cin, Cout, _ptr(dW), _ptr(db),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(X, stream))
    _check("svconv_bwd_weight", rc)
    return dW, db


def svconv_bwd_weight_noalloc(dY: torch.Tensor, X: torch.Tensor, nbr: torch.Tensor, *,
                              dW: Optional[torch.Tensor] = None, db: Optional[torch.Tensor] = None,
                              want_db: bool = True, stream=None):
    """As svconv_bwd_weight, with the split partials in the library's fixed device array
    (no workspace; concurrent calls race, see include/svconv.h)."""
    _cuda(dY, X, nbr, dW, db)
    n, Cout = dY.shape
    Cin = X.shape[1]
    if dW is None:
        dW = torch.empty((Cout, 9, Cin), dtype=torch.float32, device=X.device)
    if db is None and want_db:
        db = torch.empty((Cout,), dtype=torch.float32, device=X.device)
    rc = lib().svconv_bwd_weight_noalloc(_dtype_code(X), _ptr(dY), _ptr(X), _ptr(nbr), n, Cin, Cout, _ptr(dW),
                                         _ptr(db), _stream(X, stream))
    _check("svconv_bwd_weight_noalloc", rc)
    return dW, db


def svconv_bwd_workspace_size(dtype: int, n: int, Cin: int, Cout: int) -> int:
    return int(lib().svconv_bwd_workspace_size(int(dtype), int(n), int(Cin), int(Cout)))


def svconv_bwd(dY: torch.Tensor, X: torch.Tensor, nbr: torch.Tensor, Wt: torch.Tensor, *,
               dX: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None, db: Optional[torch.Tensor] = None,
               want_db: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """(dX, dW, db): the data gradient and the weight / bias gradients in one call."""
    _cuda(dY, X, nbr, Wt, dX, dW, db, workspace)
    n, Cout = dY.shape
    Cin = X.shape[1]
    dt = _dtype_code(X)
    if dX is None:
        dX = torch.empty((n, Cin), dtype=dY.dtype, device=dY.device)
    if dW is None:
        dW = torch.empty((Cout, 9, Cin), dtype=torch.float32, device=X.device)
    if db is None and want_db:
        db = torch.empty((Cout,), dtype=torch.float32, device=X.device)
    need = svconv_bwd_workspace_size(dt, n, Cin, Cout)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    rc = lib().svconv_bwd(dt, _ptr(dY), _ptr(X), _ptr(nbr), n, Cin, Cout, _ptr(Wt), _ptr(dX), _ptr(dW), _ptr(db),
                          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(X, stream))
    _check("svconv_bwd", rc)
    return dX, dW, db


def svconv_bwd_single_pass(dY: torch.Tensor, X: torch.Tensor, nbr: torch.Tensor, Wt: torch.Tensor, *,
                           dX: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
                           db: Optional[torch.Tensor] = None, want_db: bool = True,
                           workspace: Optional[torch.Tensor] = None, stream=None):
    """(dX, dW, db) at C_in = C_out = 64 (bf16) from one pass over dY."""
    _cuda(dY, X, nbr, Wt, dX, dW, db, workspace)
    n = dY.shape[0]
    if dX is None:
        dX = torch.empty((n, 64), dtype=dY.dtype, device=dY.device)
    if dW is None:
        dW = torch.empty((64, 9, 64), dtype=torch.float32, device=X.device)
    if db is None and want_db:
        db = torch.empty((64,), dtype=torch.float32, device=X.device)
    need = int(lib().svconv_bwd_single_pass_workspace_size(int(n)))
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    rc = lib().svconv_bwd_single_pass(_ptr(dY), _ptr(X), _ptr(nbr), n, _ptr(Wt), _ptr(dX), _ptr(dW), _ptr(db),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(X, stream))
    _check("svconv_bwd_single_pass", rc)
    return dX, dW, db


def svconv_adapter_workspace_size(R: int, max_chunk_rows: int) -> int:
    return int(lib().svconv_adapter_workspace_size(int(R), int(max_chunk_rows)))


def svconv_adapter_fwd(X: torch.Tensor, nbr: torch.Tensor, frame_off: torch.Tensor, T: int, Wd: torch.Tensor,
                       Wc: torch.Tensor, Wu: torch.Tensor, bc: Optional[torch.Tensor] = None, *, chunk_T: int,
                       max_chunk_rows: int, workspace: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """X <- X + Linear_up(GELU(SparseConv(Linear_down(X)))), chunked over frames, in place."""
    _cuda(X, nbr, frame_off, Wd, Wc, Wu, bc, workspace, status)
    n, D = X.shape
    R = Wd.shape[0]
    need = svconv_adapter_workspace_size(R, max_chunk_rows)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    rc = lib().svconv_adapter_fwd(_ptr(X), _ptr(nbr), _ptr(frame_off), int(T), n, D, R, _ptr(Wd), _ptr(Wc),
                                  _ptr(bc), _ptr(Wu), int(chunk_T), int(max_chunk_rows), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(status), _stream(X, stream))
    _check("svconv_adapter_fwd", rc)
    return X


def svconv_xattn_workspace_size(G: int, max_group_rows: int, A: int) -> int:
    return int(lib().svconv_xattn_workspace_size(int(G), int(max_group_rows), int(A)))


def svconv_xattn_aux(H: torch.Tensor, group_off: torch.Tensor, aux: torch.Tensor, *, max_group_rows: int,
                     heads: int = 1, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                     status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """aux [G, A, R] bf16 attending over the rows of H [n, R] of their group -> fp32 [G, A, R]."""
    _cuda(H, group_off, aux, out, workspace, status)
    n, R = H.shape
    G, A, _ = aux.shape
    if out is None:
        out = torch.empty((G, A, R), dtype=torch.float32, device=aux.device)
    need = svconv_xattn_workspace_size(G, max_group_rows, A)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=aux.device)
    rc = lib().svconv_xattn_aux(_ptr(H), n, R, _ptr(group_off), G, int(max_group_rows), _ptr(aux), A, int(heads),
                                _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(status), _stream(aux, stream))
    _check("svconv_xattn_aux", rc)
    return out


def svconv_adapter_xattn_workspace_size(T: int, R: int, chunk_T: int, max_chunk_rows: int, A: int) -> int:
    return int(lib().svconv_adapter_xattn_workspace_size(int(T), int(R), int(chunk_T), int(max_chunk_rows), int(A)))


def svconv_adapter_fwd_xattn(X: torch.Tensor, nbr: torch.Tensor, frame_off: torch.Tensor, T: int, Wd: torch.Tensor,
                             Wc: torch.Tensor, Wu: torch.Tensor, aux: torch.Tensor, bc: Optional[torch.Tensor] = None, *,
                             chunk_T: int, max_chunk_rows: int, heads: int = 1,
                             aux_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None):
    """The chunked adapter forward (X in place) plus the auxiliary tokens aux [A, R] attending
    over the down-projected rows of the whole sequence -> (X, aux_out fp32 [A, R])."""
    _cuda(X, nbr, frame_off, Wd, Wc, Wu, aux, bc, aux_out, workspace, status)
    n, D = X.shape
    R = Wd.shape[0]
    A = aux.shape[0]
    if aux_out is None:
        aux_out = torch.empty((A, R), dtype=torch.float32, device=X.device)
    need = svconv_adapter_xattn_workspace_size(T, R, chunk_T, max_chunk_rows, A)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    rc = lib().svconv_adapter_fwd_xattn(_ptr(X), _ptr(nbr), _ptr(frame_off), int(T), n, D, R, _ptr(Wd), _ptr(Wc),
                                        _ptr(bc), _ptr(Wu), int(chunk_T), int(max_chunk_rows), _ptr(aux), A,
                                        int(heads), _ptr(aux_out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _ptr(status),
                                        _stream(X, stream))
    _check("svconv_adapter_fwd_xattn", rc)
    return X, aux_out


def svconv_read_error_word() -> int:
    out = ctypes.c_int32(0)
    _check("svconv_read_error_word", lib().svconv_read_error_word(ctypes.byref(out)))
    return int(out.value)


def svconv_selftest_timeout(status: torch.Tensor, timeout_us: int, stream=None) -> None:
    _cuda(status)
    _check("svconv_selftest_timeout", lib().svconv_selftest_timeout(_ptr(status), int(timeout_us),
                                                                     _stream(status, stream)))
