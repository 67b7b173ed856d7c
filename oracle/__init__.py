"""ctypes wrapper around the plain C oracle (``intattn_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  The product library never
imports, links or calls anything here, and nothing here imports the product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "intattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no vector intrinsics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i8p = ctypes.POINTER(ctypes.c_int8)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        c_int, c_float, c_double = ctypes.c_int, ctypes.c_float, ctypes.c_double
        _lib.oracle_lut.argtypes = [c_double, i32p]
        _lib.oracle_index_params.argtypes = [c_double, c_double, c_int, c_double, i32p, i32p, i32p]
        _lib.oracle_requant_params.argtypes = [c_double, c_double, i32p, i32p]
        _lib.oracle_params.argtypes = [c_int, f32p, f32p, f32p, f32p, c_int, c_int, c_float,
                                       i32p, i32p]
        _lib.oracle_scores.argtypes = [i8p, i8p, c_int, c_int, i32p]
        _lib.oracle_scores.restype = None
        _lib.oracle_index.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        _lib.oracle_index.restype = ctypes.c_int32
        _lib.oracle_index_softmax.argtypes = [i32p, c_int, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_int32, i32p, u8p, i32p, i32p,
                                              ctypes.POINTER(ctypes.c_uint32)]
        _lib.oracle_index_softmax.restype = None
        _lib.oracle_requant.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        _lib.oracle_requant.restype = ctypes.c_int8
        _lib.oracle_forward.argtypes = [i8p, i8p, i8p, c_int, f32p, f32p, f32p, f32p, c_int,
                                        c_int, c_int, c_int, c_int, c_int, c_float, i8p, c_int]
        _lib.oracle_forward_rows.argtypes = [i8p, i8p, i8p, c_int, f32p, f32p, f32p, f32p,
                                             c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                                             i32p, ctypes.c_longlong, i8p, c_int]
        _lib.oracle_decode.argtypes = [i8p, i8p, i8p, c_int, f32p, f32p, f32p, f32p, c_int,
                                       c_int, c_int, c_int, c_int, c_float, i8p, c_int]
        vp = ctypes.c_void_p
        _lib.oracle_forward_zp.argtypes = [i8p, vp, vp, i32p, i32p, c_int, f32p, f32p, f32p, f32p,
                                           c_int, c_int, c_int, c_int, c_int, c_int, c_float, i8p, c_int]
        _lib.oracle_decode_zp.argtypes = [i8p, vp, vp, i32p, i32p, c_int, f32p, f32p, f32p, f32p,
                                          c_int, c_int, c_int, c_int, c_int, c_float, i8p, c_int]
    return _lib


class OracleError(RuntimeError):
    pass


def _p(a: np.ndarray, ct):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.atleast_1d(np.asarray(x, dtype=np.float32)))


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


def lut(c: float) -> np.ndarray:
    out = np.zeros(32, dtype=np.int32)
    _check(lib().oracle_lut(float(c), _p(out, ctypes.c_int32)), "oracle_lut")
    return out


def index_params(s_q: float, s_k: float, d: int, c: float):
    M, s, D = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().oracle_index_params(float(s_q), float(s_k), int(d), float(c),
                                     ctypes.byref(M), ctypes.byref(s), ctypes.byref(D)),
           "oracle_index_params")
    return M.value, s.value, D.value


def requant_params(s_v: float, s_o: float):
    Mo, so = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().oracle_requant_params(float(s_v), float(s_o), ctypes.byref(Mo),
                                       ctypes.byref(so)), "oracle_requant_params")
    return Mo.value, so.value


def params(per_head: bool, s_q, s_k, s_v, s_o, H: int, d: int, c: float):
    """(lut[32], [H, 5] array of M, s, D, Mo, so) with float32 scales."""
    sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
    L = np.zeros(32, dtype=np.int32)
    hp = np.zeros((H, 5), dtype=np.int32)
    rc = lib().oracle_params(int(per_head), _p(sq, ctypes.c_float), _p(sk, ctypes.c_float),
                             _p(sv, ctypes.c_float), _p(so, ctypes.c_float), H, d,
                             float(np.float32(c)), _p(L, ctypes.c_int32), _p(hp, ctypes.c_int32))
    _check(rc, "oracle_params")
    return L, hp


def scores(q_row: np.ndarray, k: np.ndarray) -> np.ndarray:
    q_row = np.ascontiguousarray(q_row, dtype=np.int8)
    k = np.ascontiguousarray(k, dtype=np.int8)
    n, d = k.shape
    S = np.zeros(n, dtype=np.int32)
    lib().oracle_scores(_p(q_row, ctypes.c_int8), _p(k, ctypes.c_int8), n, d,
                        _p(S, ctypes.c_int32))
    return S


def index(gap: int, M: int, s: int, D: int) -> int:
    return int(lib().oracle_index(int(gap), M, s, D))


def index_softmax(S: np.ndarray, M: int, s: int, D: int, lut_: np.ndarray):
    """u8 probabilities of one row of valid scores, plus (m, Z, R)."""
    S = np.ascontiguousarray(S, dtype=np.int32)
    L = np.ascontiguousarray(lut_, dtype=np.int32)
    P = np.zeros(S.shape[0], dtype=np.uint8)
    m, Z, R = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_uint32()
    lib().oracle_index_softmax(_p(S, ctypes.c_int32), S.shape[0], M, s, D,
                               _p(L, ctypes.c_int32), _p(P, ctypes.c_uint8),
                               ctypes.byref(m), ctypes.byref(Z), ctypes.byref(R))
    return P, m.value, Z.value, R.value


def requant(acc: int, Mo: int, so: int) -> int:
    return int(lib().oracle_requant(int(acc), Mo, so))


def _codes_and_zero_points(x, z):
    """K or V codes with their zero-points: u8 codes and an int32 array when
    z is given, else int8 codes and None (zero-point 0)."""
    if z is None:
        return np.ascontiguousarray(x, dtype=np.int8), None
    return (np.ascontiguousarray(x, dtype=np.uint8),
            np.ascontiguousarray(np.atleast_1d(np.asarray(z)), dtype=np.int32))


def _zp_ptr(z):
    return None if z is None else _p(z, ctypes.c_int32)


def forward(q, k, v, per_head, s_q, s_k, s_v, s_o, causal, clip_c, nthreads=None, z_k=None, z_v=None):
    """Prefill.  With z_k (z_v) given, k (v) holds u8 codes whose zero-points
    are z_k (z_v), one per head or one in all; else int8 codes."""
    if z_k is not None or z_v is not None:
        return _forward_zp(q, k, v, per_head, s_q, s_k, s_v, s_o, causal, clip_c, nthreads, z_k, z_v)
    q = np.ascontiguousarray(q, dtype=np.int8)
    k = np.ascontiguousarray(k, dtype=np.int8)
    v = np.ascontiguousarray(v, dtype=np.int8)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    out = np.zeros((B, H, Lq, d), dtype=np.int8)
    sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
    rc = lib().oracle_forward(_p(q, ctypes.c_int8), _p(k, ctypes.c_int8), _p(v, ctypes.c_int8),
                              int(per_head), _p(sq, ctypes.c_float), _p(sk, ctypes.c_float),
                              _p(sv, ctypes.c_float), _p(so, ctypes.c_float), B, H, Lq, Lk, d,
                              int(causal), float(np.float32(clip_c)), _p(out, ctypes.c_int8),
                              int(nthreads or os.cpu_count() or 1))
    _check(rc, "oracle_forward")
    return out


def _forward_zp(q, k, v, per_head, s_q, s_k, s_v, s_o, causal, clip_c, nthreads, z_k, z_v):
    q = np.ascontiguousarray(q, dtype=np.int8)
    k, zk = _codes_and_zero_points(k, z_k)
    v, zv = _codes_and_zero_points(v, z_v)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    out = np.zeros((B, H, Lq, d), dtype=np.int8)
    sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
    rc = lib().oracle_forward_zp(_p(q, ctypes.c_int8), k.ctypes.data, v.ctypes.data, _zp_ptr(zk), _zp_ptr(zv),
                                 int(per_head), _p(sq, ctypes.c_float), _p(sk, ctypes.c_float),
                                 _p(sv, ctypes.c_float), _p(so, ctypes.c_float), B, H, Lq, Lk, d,
                                 int(causal), float(np.float32(clip_c)), _p(out, ctypes.c_int8),
                                 int(nthreads or os.cpu_count() or 1))
    _check(rc, "oracle_forward_zp")
    return out


def forward_rows(q, k, v, per_head, s_q, s_k, s_v, s_o, causal, clip_c, rows, nthreads=None):
    """Output rows for the (b, h, i) triples in ``rows`` ([n, 3] int)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    k = np.ascontiguousarray(k, dtype=np.int8)
    v = np.ascontiguousarray(v, dtype=np.int8)
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    out = np.zeros((rows.shape[0], d), dtype=np.int8)
    sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
    rc = lib().oracle_forward_rows(_p(q, ctypes.c_int8), _p(k, ctypes.c_int8),
                                   _p(v, ctypes.c_int8), int(per_head), _p(sq, ctypes.c_float),
                                   _p(sk, ctypes.c_float), _p(sv, ctypes.c_float),
                                   _p(so, ctypes.c_float), B, H, Lq, Lk, d, int(causal),
                                   float(np.float32(clip_c)), _p(rows, ctypes.c_int32),
                                   rows.shape[0], _p(out, ctypes.c_int8),
                                   int(nthreads or os.cpu_count() or 1))
    _check(rc, "oracle_forward_rows")
    return out


def decode(q, k_cache, v_cache, per_head, s_q, s_k, s_v, s_o, Lk, clip_c, nthreads=None, z_k=None, z_v=None):
    """Decode over the first Lk rows of the caches; zero-points as in forward."""
    if z_k is not None or z_v is not None:
        q = np.ascontiguousarray(q, dtype=np.int8)
        kc, zk = _codes_and_zero_points(k_cache, z_k)
        vc, zv = _codes_and_zero_points(v_cache, z_v)
        B, H, one, d = q.shape
        assert one == 1
        out = np.zeros((B, H, 1, d), dtype=np.int8)
        sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
        rc = lib().oracle_decode_zp(_p(q, ctypes.c_int8), kc.ctypes.data, vc.ctypes.data, _zp_ptr(zk),
                                    _zp_ptr(zv), int(per_head), _p(sq, ctypes.c_float), _p(sk, ctypes.c_float),
                                    _p(sv, ctypes.c_float), _p(so, ctypes.c_float), B, H, int(Lk), kc.shape[2],
                                    d, float(np.float32(clip_c)), _p(out, ctypes.c_int8),
                                    int(nthreads or os.cpu_count() or 1))
        _check(rc, "oracle_decode_zp")
        return out
    q = np.ascontiguousarray(q, dtype=np.int8)
    kc = np.ascontiguousarray(k_cache, dtype=np.int8)
    vc = np.ascontiguousarray(v_cache, dtype=np.int8)
    B, H, one, d = q.shape
    assert one == 1
    Lmax = kc.shape[2]
    out = np.zeros((B, H, 1, d), dtype=np.int8)
    sq, sk, sv, so = _f32(s_q), _f32(s_k), _f32(s_v), _f32(s_o)
    rc = lib().oracle_decode(_p(q, ctypes.c_int8), _p(kc, ctypes.c_int8), _p(vc, ctypes.c_int8),
                             int(per_head), _p(sq, ctypes.c_float), _p(sk, ctypes.c_float),
                             _p(sv, ctypes.c_float), _p(so, ctypes.c_float), B, H, int(Lk),
                             Lmax, d, float(np.float32(clip_c)), _p(out, ctypes.c_int8),
                             int(nthreads or os.cpu_count() or 1))
    _check(rc, "oracle_decode")
    return out
