"""Plain numpy oracle of the quantisation prologue.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and ``bench.py``'s CPU
baseline; the product library never calls it.

Follows the forum page "IntAttention：面向边缘设备的纯整数注意力推理加速方案",
section 动态量化策略 (the quantisation range of a layer, or of a head, is taken
from the live activations), with the readings: symmetric (zero-point 0),
range = max |x|, 127 levels each side, round half to even.  Definition:
    amax = max |x| over the tensor, or over one head's [B, L, d] slice
    s    = amax / 127 and inv = min(127 / amax, FLT_MAX) in IEEE fp32 (both 1
           when amax = 0)
    code = clamp(rint(x * inv), -127, 127), the fp32 product rounded to nearest

The same page names a zero-point beside the scale; ``quantize_asym`` is that
form (u8 codes), with the readings: the range always holds 0 (so that 0 is a
code), 255 levels, the width in IEEE double, round half to even:
    hi   = max(max x, 0),  lo = min(min x, 0)  over the tensor or one head
    w    = hi - lo                      (double)
    s    = RN32(w / 255),  inv = RN32(min(255 / w, FLT_MAX))  (both 1 when w = 0)
    z    = clamp(rint(RN32(-lo * inv)), 0, 255)
    code = clamp(rint(RN32(x * inv)) + z, 0, 255)
A code c stands for s (c - z).
"""
import numpy as np


def quantize(x, per_head: bool):
    """x: float32 array [B, H, L, d] holding fp16 / bf16 values (exact).
    Returns (codes int8 [B, H, L, d], scales float32 [H] or [1])."""
    x = np.asarray(x, dtype=np.float32)
    B, H, L, d = x.shape
    if per_head:
        amax = np.abs(x).max(axis=(0, 2, 3)) if x.size else np.zeros(H, np.float32)
    else:
        amax = np.array([np.abs(x).max() if x.size else 0.0], dtype=np.float32)
    amax = amax.astype(np.float32)
    s = (amax / np.float32(127.0)).astype(np.float32)
    s[amax == 0] = np.float32(1.0)
    inv = np.ones_like(amax)
    nz = amax != 0
    with np.errstate(over="ignore", divide="ignore"):
        inv[nz] = np.minimum(np.float32(127.0) / amax[nz], np.finfo(np.float32).max).astype(np.float32)
    per = inv if per_head else np.repeat(inv, H)
    q = np.rint(x * per[None, :, None, None].astype(np.float32))  # float32 product, half-even
    return np.clip(q, -127, 127).astype(np.int8), s


def quantize_asym(x, per_head: bool):
    """x: float32 [B, H, L, d] holding fp16 / bf16 values.  Returns (codes
    uint8 [B, H, L, d], scales float32 [H] or [1], zero-points int32 [H] or [1])."""
    x = np.asarray(x, dtype=np.float32)
    B, H, L, d = x.shape
    axes = (0, 2, 3) if per_head else None
    n = H if per_head else 1
    if x.size:
        hi = np.maximum(np.asarray(x.max(axis=axes), np.float32).reshape(n), np.float32(0))
        lo = np.minimum(np.asarray(x.min(axis=axes), np.float32).reshape(n), np.float32(0))
    else:
        hi = np.zeros(n, np.float32)
        lo = np.zeros(n, np.float32)
    w = hi.astype(np.float64) - lo.astype(np.float64)
    s = np.ones(n, np.float32)
    inv = np.ones(n, np.float32)
    nz = w != 0
    s[nz] = (w[nz] / 255.0).astype(np.float32)
    inv[nz] = np.minimum(255.0 / w[nz], float(np.finfo(np.float32).max)).astype(np.float32)
    z = np.clip(np.rint((-lo) * inv), 0, 255).astype(np.int32)  # float32 product, half-even
    per_inv = inv if per_head else np.repeat(inv, H)
    per_z = z if per_head else np.repeat(z, H)
    p = np.rint(x * per_inv[None, :, None, None].astype(np.float32))  # float32 product, half-even
    codes = np.clip(p + per_z[None, :, None, None], 0, 255).astype(np.uint8)
    return codes, s, z
