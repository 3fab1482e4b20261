"""CPU oracle for SparseConv2D (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of the
benchmark may import this package.  The product path (the CUDA library and its
Python binding) never loads it, and this package never imports the product.

The arithmetic lives in ``svconv_oracle.c`` (plain single-threaded C, double
precision); this file only compiles it, loads it with ctypes and converts numpy
arrays.  Every function follows the SV-TAD page (papernotes.org, "SV-TAD: Native
Sparse Convolutions for Efficient Temporal Action Detection", Key Designs 1-2);
see the C file's header for the readings taken where the page is silent.

Parity pins: every function here is checked by ``tests/test_oracle_pins.py``
against something other than itself (dense convolution through torch's conv2d
in float64, brute-force neighbour search, finite differences / adjoint
identities, a hand-worked fixture, bf16 rounding against torch's RNE cast).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svconv_oracle.c")
_LIB = os.path.join(_HERE, "libsvconv_oracle.so")
_lib = None

BAD_COORD, DUPLICATE, BAD_FRAME, BAD_OFFSETS = 1, 2, 4, 8


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE double, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.orc_build_index.argtypes = [P, P, I, I, I, I, P, P]
        lib.orc_build_index.restype = I
        lib.orc_fwd.argtypes = [P, P, I, I, I, P, P, P, I, P]
        lib.orc_bwd_data.argtypes = [P, P, I, I, I, P, P, I, P]
        lib.orc_bwd_weight.argtypes = [P, P, P, I, I, I, P, P]
        lib.orc_bwd_weight_entries.argtypes = [P, P, P, I, I, I, P, I, P]
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_round_bf16.restype = ctypes.c_double
        lib.orc_adapter_fwd.argtypes = [P, P, I, I, I, I, P, P, P, P, P]
        lib.orc_dense_conv.argtypes = [P, I, I, I, I, P, P, P]
        lib.orc_bwd_bias.argtypes = [P, I, I, P]
        lib.orc_xattn_aux.argtypes = [P, P, I, I, I, P, I, P]
        lib.orc_down_proj.argtypes = [P, I, I, I, P, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def build_index(coords, frame_off, T, H, W, want_map=True):
    """Returns (nbr [n,9] int32, M [T,H,W] int32 or None, status flags)."""
    lib = _load()
    coords = _i32(coords).reshape(-1, 3)
    frame_off = _i32(frame_off)
    n = coords.shape[0]
    nbr = np.empty((n, 9), dtype=np.int32)
    M = np.empty((T, H, W), dtype=np.int32) if want_map else None
    st = lib.orc_build_index(_p(coords), _p(frame_off), T, H, W, n, _p(nbr), _p(M))
    return nbr, M, int(st)


def fwd(X, nbr, Wt, bias=None, rows=None):
    lib = _load()
    X = _f64(X)
    Wt = _f64(Wt)
    nbr = _i32(nbr)
    n, Cin = X.shape
    Cout = Wt.shape[0]
    b = _f64(bias)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    cnt = n if r is None else r.shape[0]
    Y = np.empty((cnt, Cout), dtype=np.float64)
    lib.orc_fwd(_p(X), _p(nbr), n, Cin, Cout, _p(Wt), _p(b), _p(r), 0 if r is None else cnt, _p(Y))
    return Y


def bwd_data(dY, nbr, Wt, rows=None):
    lib = _load()
    dY = _f64(dY)
    Wt = _f64(Wt)
    nbr = _i32(nbr)
    n, Cout = dY.shape
    Cin = Wt.shape[2]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    cnt = n if r is None else r.shape[0]
    dX = np.empty((cnt, Cin), dtype=np.float64)
    lib.orc_bwd_data(_p(dY), _p(nbr), n, Cin, Cout, _p(Wt), _p(r), 0 if r is None else cnt, _p(dX))
    return dX


def bwd_weight(dY, X, nbr, with_bias=True):
    lib = _load()
    dY = _f64(dY)
    X = _f64(X)
    nbr = _i32(nbr)
    n, Cout = dY.shape
    Cin = X.shape[1]
    dW = np.empty((Cout, 9, Cin), dtype=np.float64)
    db = np.empty((Cout,), dtype=np.float64) if with_bias else None
    lib.orc_bwd_weight(_p(dY), _p(X), _p(nbr), n, Cin, Cout, _p(dW), _p(db))
    return dW, db


def bwd_weight_entries(dY, X, nbr, entries):
    lib = _load()
    dY = _f64(dY)
    X = _f64(X)
    nbr = _i32(nbr)
    ent = _i32(entries).reshape(-1, 3)
    n, Cout = dY.shape
    Cin = X.shape[1]
    out = np.empty((ent.shape[0],), dtype=np.float64)
    lib.orc_bwd_weight_entries(_p(dY), _p(X), _p(nbr), n, Cin, Cout, _p(ent), ent.shape[0], _p(out))
    return out


def bwd_bias(dY):
    lib = _load()
    dY = _f64(dY)
    n, Cout = dY.shape
    db = np.empty((Cout,), dtype=np.float64)
    lib.orc_bwd_bias(_p(dY), n, Cout, _p(db))
    return db


def round_bf16(v: float) -> float:
    return float(_load().orc_round_bf16(float(v)))


def adapter_fwd(X, nbr, r0, r1, Wd, Wc, Wu, bc=None):
    """Adapter output rows r0..r1-1 (whole frames)."""
    lib = _load()
    X = _f64(X)
    nbr = _i32(nbr)
    D = X.shape[1]
    R = Wd.shape[0]
    out = np.empty((r1 - r0, D), dtype=np.float64)
    lib.orc_adapter_fwd(_p(X), _p(nbr), int(r0), int(r1), D, R, _p(_f64(Wd)), _p(_f64(Wc)),
                        _p(_f64(bc)), _p(_f64(Wu)), _p(out))
    return out


def xattn_aux(Hf, goff, aux, heads=1):
    """Auxiliary tokens aux [G, A, R] updated by attention over the rows of their group
    (Key Design 3); Hf [n, R] are the keys and values, goff [G+1] the groups' row bounds."""
    lib = _load()
    Hf = _f64(Hf)
    goff = _i32(goff)
    aux = _f64(aux)
    G, A, R = aux.shape
    out = np.empty((G, A, R), dtype=np.float64)
    lib.orc_xattn_aux(_p(Hf), _p(goff), int(G), int(R), int(heads), _p(aux), int(A), _p(out))
    return out


def down_proj(X, Wd):
    """The adapter's first stage alone: bf16(X Wd^T), [n, R]."""
    lib = _load()
    X = _f64(X)
    Wd = _f64(Wd)
    n, D = X.shape
    R = Wd.shape[0]
    H1 = np.empty((n, R), dtype=np.float64)
    lib.orc_down_proj(_p(X), int(n), int(D), int(R), _p(Wd), _p(H1))
    return H1


def dense_conv(G, Wt, bias=None):
    """Dense zero-padded 3x3 cross-correlation of one frame G [H,W,Cin]."""
    lib = _load()
    G = _f64(G)
    H, W, Cin = G.shape
    Wt = _f64(Wt)
    Cout = Wt.shape[0]
    Y = np.empty((H, W, Cout), dtype=np.float64)
    lib.orc_dense_conv(_p(G), H, W, Cin, Cout, _p(Wt), _p(_f64(bias)), _p(Y))
    return Y
