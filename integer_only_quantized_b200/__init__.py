"""Fully-integer attention forward (IntAttention, arXiv 2511.21513) on B200.

Python binding of the C ABI in ``include/intattn.h``: argument marshalling
only.  Every step of the computation runs in the CUDA kernels of
``libintattn.so``; torch supplies device memory and streams.  There is no CPU
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence, Union

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libintattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_PARAM_RANGE, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT = range(7)
MAX_HEADS = 128
MAX_CLIPS = 8

# every function declared in include/intattn.h
EXPORTED = ("intattn_derive_params", "intattn_forward", "intattn_forward_variant",
            "intattn_forward_host_workspace_size", "intattn_forward_fp_workspace_size", "intattn_forward_fp",
            "intattn_forward_fp_zp",
            "intattn_calibrate_workspace_size", "intattn_calibrate_clip",
            "intattn_forward_host", "intattn_decode_workspace_size",
            "intattn_decode", "intattn_decode_int4", "intattn_decode_static_scratch", "intattn_quantize",
            "intattn_quantize_zp",
            "intattn_gelu_derive_params", "intattn_gelu", "intattn_selftest_timeout", "intattn_device_error",
            "intattn_strerror")
DTYPE_FP16, DTYPE_BF16 = 0, 1
VARIANT_AUTO, VARIANT_THREE_PASS, VARIANT_SHORT_ROWS = 0, 1, 2
SHORT_ROWS_MAX_KEYS = 256


class _GeluParams(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("s", ctypes.c_int32), ("Mo", ctypes.c_int32), ("so", ctypes.c_int32),
                ("gate", ctypes.c_int32 * 32)]


class IntAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code) if _lib is not None else code} (code {code})")


class _Scales(ctypes.Structure):
    _fields_ = [("per_head", ctypes.c_int32),
                ("s_q", ctypes.POINTER(ctypes.c_float)),
                ("s_k", ctypes.POINTER(ctypes.c_float)),
                ("s_v", ctypes.POINTER(ctypes.c_float)),
                ("s_o", ctypes.POINTER(ctypes.c_float)),
                ("clip_c", ctypes.POINTER(ctypes.c_float)),
                ("z_k", ctypes.POINTER(ctypes.c_int32)),
                ("z_v", ctypes.POINTER(ctypes.c_int32))]


class _HeadParams(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("s", ctypes.c_int32), ("D", ctypes.c_int32),
                ("Mo", ctypes.c_int32), ("so", ctypes.c_int32)]


FloatArg = Union[float, Sequence[float], np.ndarray]


@dataclasses.dataclass
class Scales:
    """Quantisation scales (real = scale * code).  per_head: arrays of H.
    clip: optional per-head clip thresholds (same layout as the scales);
    None: the call's clip_c applies to every head.
    z_k / z_v: optional zero-points (same layout, 0..255): the K / V codes
    are then uint8 tensors and code c stands for c - z."""
    s_q: FloatArg
    s_k: FloatArg
    s_v: FloatArg
    s_o: FloatArg
    per_head: bool = False
    clip: Optional[FloatArg] = None
    z_k: Optional[FloatArg] = None
    z_v: Optional[FloatArg] = None

    def _c(self):
        arrs = [np.ascontiguousarray(np.atleast_1d(np.asarray(x, dtype=np.float32)))
                for x in (self.s_q, self.s_k, self.s_v, self.s_o)]
        fp = ctypes.POINTER(ctypes.c_float)
        clip = None
        if self.clip is not None:
            clip = np.ascontiguousarray(np.atleast_1d(np.asarray(self.clip, dtype=np.float32)))
            arrs.append(clip)
        ip = ctypes.POINTER(ctypes.c_int32)
        zs = []
        for z in (self.z_k, self.z_v):
            if z is None:
                zs.append(ip())
            else:
                za = np.ascontiguousarray(np.atleast_1d(np.asarray(z)).astype(np.int32))
                arrs.append(za)
                zs.append(za.ctypes.data_as(ip))
        s = _Scales(int(bool(self.per_head)), *[a.ctypes.data_as(fp) for a in arrs[:4]],
                    clip.ctypes.data_as(fp) if clip is not None else fp(), *zs)
        return s, arrs  # keep the arrays alive for the duration of the call


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m integer_only_quantized_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.intattn_derive_params.argtypes = [ctypes.POINTER(_Scales), i32, i32, f32,
                                            ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(_HeadParams)]
        L.intattn_forward.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32,
                                      i32, f32, vp, vp]
        L.intattn_forward_variant.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32,
                                              i32, f32, vp, i32, vp]
        L.intattn_forward_fp_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.intattn_forward_fp_workspace_size.restype = ctypes.c_size_t
        f32p = ctypes.POINTER(ctypes.c_float)
        L.intattn_forward_fp.argtypes = [vp, vp, vp, i32, i32, f32p, f32p, f32, i32, i32, i32, i32, i32, i32,
                                         vp, vp, vp, ctypes.c_size_t, vp]
        L.intattn_forward_fp_zp.argtypes = [vp, vp, vp, i32, i32, f32p, f32p, f32, i32, i32, i32, i32, i32, i32,
                                            vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.intattn_calibrate_workspace_size.argtypes = [i32, i32]
        L.intattn_calibrate_workspace_size.restype = ctypes.c_size_t
        L.intattn_calibrate_clip.argtypes = [vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32, i32, i32,
                                             i32, f32, f32, f32p, ctypes.POINTER(ctypes.c_int32), vp,
                                             ctypes.c_size_t, vp]
        L.intattn_forward_host_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.intattn_forward_host_workspace_size.restype = ctypes.c_size_t
        L.intattn_forward_host.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32,
                                           i32, f32, vp, vp, ctypes.c_size_t, vp]
        L.intattn_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        L.intattn_decode_workspace_size.restype = ctypes.c_size_t
        L.intattn_decode.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32,
                                     f32, vp, vp, ctypes.c_size_t, vp]
        L.intattn_decode_int4.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32, i32, i32,
                                          f32, vp, vp, ctypes.c_size_t, vp]
        L.intattn_decode_static_scratch.argtypes = [vp, vp, vp, ctypes.POINTER(_Scales), i32, i32, i32,
                                                    i32, i32, f32, vp, vp]
        L.intattn_quantize.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
        L.intattn_quantize_zp.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.intattn_gelu_derive_params.argtypes = [f32, f32, f32, ctypes.POINTER(_GeluParams)]
        L.intattn_gelu.argtypes = [vp, vp, ctypes.c_longlong, f32, f32, f32, vp]
        L.intattn_selftest_timeout.argtypes = [vp]
        L.intattn_device_error.argtypes = [vp]
        L.intattn_strerror.argtypes = [i32]
        L.intattn_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().intattn_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise IntAttnError(rc, what)


def derive_params(scales: Scales, H: int, d: int, clip_c: float):
    """(lut[32] int32, [H, 5] int32 of M, s, D, Mo, so) as the kernels use them."""
    sc, keep = scales._c()
    lut = np.zeros(32, dtype=np.int32)
    hp = (_HeadParams * H)()
    rc = lib().intattn_derive_params(ctypes.byref(sc), int(H), int(d), float(clip_c),
                                     lut.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), hp)
    _check(rc, "intattn_derive_params")
    del keep
    return lut, np.array([[p.M, p.s, p.D, p.Mo, p.so] for p in hp], dtype=np.int32)


def _stream_handle(stream, device) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_tensor(t, name: str):
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int8 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA int8 tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_codes(t, name: str, zero_point, cuda: bool = True):
    """K or V codes: uint8 when the tensor has a zero-point, else int8."""
    import torch
    want = torch.uint8 if zero_point is not None else torch.int8
    if not isinstance(t, torch.Tensor) or t.dtype != want or t.is_cuda != cuda:
        raise TypeError(f"{name} must be a {'CUDA' if cuda else 'CPU'} {want} tensor"
                        + (" (it has a zero-point)" if zero_point is not None else ""))
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def forward(q, k, v, scales: Scales, causal: bool, clip_c: float, out=None, stream=None, variant: int = 0):
    """out[B,H,Lq,d] int8 = IntAttention forward of int8 q[B,H,Lq,d], k/v[B,H,Lk,d].
    variant: VARIANT_AUTO (intattn_forward), VARIANT_THREE_PASS or
    VARIANT_SHORT_ROWS (intattn_forward_variant); the bytes are the same."""
    import torch
    _check_tensor(q, "q")
    _check_codes(k, "k", scales.z_k)
    _check_codes(v, "v", scales.z_v)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Lk, d] matching q")
    if out is None:
        out = torch.empty_like(q)
    _check_tensor(out, "out")
    if out.shape != q.shape:
        raise ValueError("out must match q")
    sc, keep = scales._c()
    if variant == VARIANT_AUTO:
        rc = lib().intattn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(sc), B, H, Lq, Lk,
                                   d, int(bool(causal)), float(clip_c), out.data_ptr(),
                                   _stream_handle(stream, q.device))
    else:
        rc = lib().intattn_forward_variant(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(sc), B, H,
                                           Lq, Lk, d, int(bool(causal)), float(clip_c), out.data_ptr(),
                                           int(variant), _stream_handle(stream, q.device))
    del keep
    _check(rc, "intattn_forward")
    return out


def forward_host_workspace_size(B: int, H: int, Lq: int, Lk: int, d: int) -> int:
    return int(lib().intattn_forward_host_workspace_size(B, H, Lq, Lk, d))


def forward_host(q, k, v, scales: Scales, causal: bool, clip_c: float, out=None, workspace=None, stream=None,
                 device=None):
    """forward on CPU int8 tensors (pinned for asynchronous copies): the
    library copies them in, runs the forward and copies the result out;
    consecutive calls with one workspace overlap.  Returns out (a CPU tensor,
    valid once `stream` has reached the end of the call)."""
    import torch
    if not isinstance(q, torch.Tensor) or q.dtype != torch.int8 or q.is_cuda or not q.is_contiguous():
        raise TypeError("q must be a contiguous CPU int8 tensor")
    _check_codes(k, "k", scales.z_k, cuda=False)
    _check_codes(v, "v", scales.z_v, cuda=False)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Lk, d]")
    dev = torch.device("cuda") if device is None else torch.device(device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.int8, pin_memory=True)
    if out.is_cuda or out.dtype != torch.int8 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU int8 tensor shaped like q")
    need = forward_host_workspace_size(B, H, Lq, Lk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    sc, keep = scales._c()
    rc = lib().intattn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(sc), B, H, Lq, Lk, d,
                                    int(bool(causal)), float(clip_c), out.data_ptr(), workspace.data_ptr(),
                                    workspace.numel(), _stream_handle(stream, dev))
    del keep
    _check(rc, "intattn_forward_host")
    return out


def forward_fp_workspace_size(B: int, H: int, Lq: int, Lk: int, d: int) -> int:
    return int(lib().intattn_forward_fp_workspace_size(B, H, Lq, Lk, d))


def forward_fp(q, k, v, per_head: bool, s_o, causal: bool, clip_c: float, clip=None, out=None, scales_out=None,
               workspace=None, stream=None, zero_points=False, zero_points_out=None):
    """intattn_forward_fp: fp16 / bf16 q [B,H,Lq,d], k, v [B,H,Lk,d] (CUDA)
    -> int8 out, quantising on the device.  s_o (and clip, optional): host
    floats, H entries per head or 1.  zero_points=True: intattn_forward_fp_zp
    (K and V quantised with zero-points; zero_points_out, optional CUDA int32
    [2 n], receives z_k then z_v)."""
    import torch
    dt = {torch.float16: DTYPE_FP16, torch.bfloat16: DTYPE_BF16}
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in dt or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous CUDA fp16 / bf16 tensor")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must have one dtype")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Lk, d] matching q")
    if out is None:
        out = torch.empty((B, H, Lq, d), dtype=torch.int8, device=q.device)
    _check_tensor(out, "out")
    so = np.ascontiguousarray(np.atleast_1d(np.asarray(s_o, dtype=np.float32)))
    cl = None if clip is None else np.ascontiguousarray(np.atleast_1d(np.asarray(clip, dtype=np.float32)))
    need = forward_fp_workspace_size(B, H, Lq, Lk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    f32p = ctypes.POINTER(ctypes.c_float)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), dt[q.dtype], int(bool(per_head)), so.ctypes.data_as(f32p),
            None if cl is None else cl.ctypes.data_as(f32p), float(clip_c), B, H, Lq, Lk, d, int(bool(causal)),
            out.data_ptr(), None if scales_out is None else scales_out.data_ptr())
    tail = (workspace.data_ptr(), workspace.numel(), _stream_handle(stream, q.device))
    if zero_points:
        zp = None if zero_points_out is None else zero_points_out.data_ptr()
        rc = lib().intattn_forward_fp_zp(*args, zp, *tail)
        _check(rc, "intattn_forward_fp_zp")
    else:
        rc = lib().intattn_forward_fp(*args, *tail)
        _check(rc, "intattn_forward_fp")
    return out


def calibrate_workspace_size(B: int, H: int) -> int:
    return int(lib().intattn_calibrate_workspace_size(int(B), int(H)))


def calibrate_clip(q, k, scales: Scales, causal: bool, keep: int, stride: int, c_min: float = 0.25,
                   c_max: float = 64.0, workspace=None, stream=None):
    """intattn_calibrate_clip: (thresholds float32 [H or 1], gaps int32 [H or 1])
    for int8 CUDA q [B,H,Lq,d], k [B,H,Lk,d].  Synchronises the stream."""
    import torch
    _check_tensor(q, "q")
    _check_tensor(k, "k")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if k.shape != (B, H, Lk, d):
        raise ValueError("k must be [B, H, Lk, d] matching q")
    n = H if scales.per_head else 1
    clip = np.zeros(n, dtype=np.float32)
    gaps = np.zeros(n, dtype=np.int32)
    if workspace is None:
        workspace = torch.empty(max(int(lib().intattn_calibrate_workspace_size(B, H)), 1), dtype=torch.uint8,
                                device=q.device)
    sc, keep_alive = scales._c()
    rc = lib().intattn_calibrate_clip(q.data_ptr(), k.data_ptr(), ctypes.byref(sc), B, H, Lq, Lk, d,
                                      int(bool(causal)), int(keep), int(stride), float(c_min), float(c_max),
                                      clip.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                      gaps.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), workspace.data_ptr(),
                                      workspace.numel(), _stream_handle(stream, q.device))
    del keep_alive
    _check(rc, "intattn_calibrate_clip")
    return clip, gaps


def decode_workspace_size(B: int, H: int, Lk: int, d: int) -> int:
    return int(lib().intattn_decode_workspace_size(int(B), int(H), int(Lk), int(d)))


def decode(q, k_cache, v_cache, scales: Scales, Lk: int, clip_c: float, out=None, workspace=None,
           stream=None):
    """out[B,H,1,d] int8: one query per (b, h) over the first Lk rows of the caches."""
    import torch
    _check_tensor(q, "q")
    _check_codes(k_cache, "k_cache", scales.z_k)
    _check_codes(v_cache, "v_cache", scales.z_v)
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query per (b, h): q is [B, H, 1, d]")
    Lmax = k_cache.shape[2]
    if k_cache.shape != (B, H, Lmax, d) or v_cache.shape != k_cache.shape:
        raise ValueError("caches must be [B, H, Lmax, d]")
    if out is None:
        out = torch.empty_like(q)
    _check_tensor(out, "out")
    need = decode_workspace_size(B, H, Lk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    sc, keep = scales._c()
    rc = lib().intattn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), ctypes.byref(sc), B,
                              H, int(Lk), Lmax, d, float(clip_c), out.data_ptr(), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(),
                              _stream_handle(stream, q.device))
    del keep
    _check(rc, "intattn_decode")
    return out


def _check_u8_tensor(t, name: str):
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA uint8 tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def decode_int4(q, k_cache, v_cache, scales: Scales, Lk: int, clip_c: float, out=None, workspace=None,
                stream=None):
    """out[B,H,1,d] int8 over an int4 KV cache: k_cache/v_cache are uint8
    [B, H, Lmax, d/2], two 4-bit two's-complement channels per byte (channel
    2t in the low nibble of byte t)."""
    import torch
    _check_tensor(q, "q")
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_u8_tensor(t, n)
    B, H, one, d = q.shape
    if one != 1:
        raise ValueError("decode takes one query per (b, h): q is [B, H, 1, d]")
    Lmax = k_cache.shape[2]
    if k_cache.shape != (B, H, Lmax, d // 2) or v_cache.shape != k_cache.shape:
        raise ValueError("int4 caches must be [B, H, Lmax, d/2] bytes")
    if out is None:
        out = torch.empty_like(q)
    _check_tensor(out, "out")
    need = decode_workspace_size(B, H, Lk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    sc, keep = scales._c()
    rc = lib().intattn_decode_int4(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), ctypes.byref(sc), B,
                                   H, int(Lk), Lmax, d, float(clip_c), out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream, q.device))
    del keep
    _check(rc, "intattn_decode_int4")
    return out


def quantize(x, per_head: bool, out=None, scales=None, stream=None):
    """int8 codes and device scales of an fp16 / bf16 CUDA tensor [B, H, L, d]
    (symmetric, dynamic: s = max|x| / 127 per tensor or per head)."""
    import torch
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("x must be a CUDA float16 or bfloat16 tensor")
    if not x.is_contiguous() or x.dim() != 4:
        raise ValueError("x must be a contiguous [B, H, L, d] tensor")
    B, H, L, d = x.shape
    if out is None:
        out = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    _check_tensor(out, "out")
    if out.shape != x.shape:
        raise ValueError("out must match x")
    n = H if per_head else 1
    if scales is None:
        scales = torch.empty(n, dtype=torch.float32, device=x.device)
    if scales.dtype != torch.float32 or not scales.is_cuda or scales.numel() < n:
        raise ValueError(f"scales must be a CUDA float32 tensor of at least {n} entries")
    dt = DTYPE_BF16 if x.dtype == torch.bfloat16 else DTYPE_FP16
    _check(lib().intattn_quantize(x.data_ptr(), dt, B, H, L, d, int(bool(per_head)), out.data_ptr(),
                                  scales.data_ptr(), _stream_handle(stream, x.device)), "intattn_quantize")
    return out, scales


def quantize_zp(x, per_head: bool, out=None, scales=None, zero_points=None, stream=None):
    """u8 codes, device scales and device zero-points of an fp16 / bf16 CUDA
    tensor [B, H, L, d] (asymmetric, dynamic, per tensor or per head)."""
    import torch
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("x must be a CUDA float16 or bfloat16 tensor")
    if not x.is_contiguous() or x.dim() != 4:
        raise ValueError("x must be a contiguous [B, H, L, d] tensor")
    B, H, L, d = x.shape
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if not isinstance(out, torch.Tensor) or out.dtype != torch.uint8 or not out.is_cuda or not out.is_contiguous():
        raise TypeError("out must be a contiguous CUDA uint8 tensor")
    if out.shape != x.shape:
        raise ValueError("out must match x")
    n = H if per_head else 1
    if scales is None:
        scales = torch.empty(n, dtype=torch.float32, device=x.device)
    if zero_points is None:
        zero_points = torch.empty(n, dtype=torch.int32, device=x.device)
    if scales.dtype != torch.float32 or not scales.is_cuda or scales.numel() < n:
        raise ValueError(f"scales must be a CUDA float32 tensor of at least {n} entries")
    if zero_points.dtype != torch.int32 or not zero_points.is_cuda or zero_points.numel() < n:
        raise ValueError(f"zero_points must be a CUDA int32 tensor of at least {n} entries")
    dt = DTYPE_BF16 if x.dtype == torch.bfloat16 else DTYPE_FP16
    _check(lib().intattn_quantize_zp(x.data_ptr(), dt, B, H, L, d, int(bool(per_head)), out.data_ptr(),
                                     scales.data_ptr(), zero_points.data_ptr(), _stream_handle(stream, x.device)),
           "intattn_quantize_zp")
    return out, scales, zero_points


def gelu_params(s_x: float, s_y: float, c: float):
    """(M, s, gate[32], Mo, so) of the integer GELU, as the kernel uses them."""
    p = _GeluParams()
    _check(lib().intattn_gelu_derive_params(float(s_x), float(s_y), float(c), ctypes.byref(p)),
           "intattn_gelu_derive_params")
    return p.M, p.s, list(p.gate), p.Mo, p.so


def gelu(x, s_x: float, s_y: float, c: float, out=None, stream=None):
    """Integer GELU of a contiguous CUDA int8 tensor (any shape): int8 codes
    of scale s_y for codes x of scale s_x; gate tabulated on [-c, c].
    out may be x itself (in place)."""
    _check_tensor(x, "x")
    if out is None:
        import torch
        out = torch.empty_like(x)
    _check_tensor(out, "out")
    if out.numel() != x.numel():
        raise ValueError("out must have as many elements as x")
    _check(lib().intattn_gelu(x.data_ptr(), out.data_ptr(), x.numel(), float(s_x), float(s_y), float(c),
                              _stream_handle(stream, x.device)), "intattn_gelu")
    return out


def device_error(stream=None) -> int:
    """Synchronise and return/clear the device error word (OK or ERR_TIMEOUT)."""
    import torch
    return int(lib().intattn_device_error(_stream_handle(stream, torch.device("cuda"))))


def selftest_timeout(stream=None) -> int:
    """Run the bounded-wait self-test; returns device_error() afterwards
    (ERR_TIMEOUT when failure detection works)."""
    import torch
    _check(lib().intattn_selftest_timeout(_stream_handle(stream, torch.device("cuda"))),
           "intattn_selftest_timeout")
    return device_error(stream)
