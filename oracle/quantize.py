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
