"""Plain Python oracle of the integer GELU (one int8 code in, one out).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and ``bench.py``'s CPU
baseline; the product library never calls it, and it shares no code, table
or constant generator with the CUDA library.

The pages name GELU only as future work: the euno.news summary
"[Paper] IntAttention：全整数注意力流水线用于高效边缘推理", section
局限性与未来工作 (and its Korean twin, Limitations & Future Work), lists
extending the method to further nonlinear operators such as GELU.  Nothing
about the operator is fixed there, so everything below is this
implementation's reading, built from the same three pieces as IndexSoftmax
(Methodology item 2 of the same page): an integer index by multiply and
shift, a 32-entry integer table, and a requantising multiply and shift.

GELU(x) = x * Phi(x), Phi the standard normal CDF.  The gate Phi is tabulated
on 32 points spread evenly over [-c, c]; outside the table the gate is
exactly 0 (left) or 1 (right), so very negative inputs give 0 and large
positive ones pass through unchanged.

Host parameters (IEEE double, in this order; s_x, s_y, c are fp32 values):
    r      = (s_x * 31) / (2 * c)           table steps per input code
    s      = 26; while (s > 1 and llround(r * 2^s) > 2^24) s -= 1
    M      = llround(r * 2^s)               need 1 <= M <= 2^24
    t_i    = ((2i - 31) * c) / 31           i = 0..31: -c .. c
    G[i]   = llround(32768 * (0.5 * erfc(-t_i / sqrt(2))))   i = 1..30
    G[0]   = 0,  G[31] = 32768
    m      = s_x / (32768 * s_y) = f * 2^e, f in [0.5, 1)
    Mo     = llround(f * 2^31) (2^31 -> 2^30 and e + 1);  so = 31 - e in [1, 62]
Per element (q an int8 code, real value s_x * q):
    idx = clamp(16 + floor(q * M / 2^s), 0, 31)    round-half-up of q*r + 15.5
    y   = q * G[idx]                               |y| <= 2^22
    out = clamp(floor((y * Mo + 2^(so-1)) / 2^so), -127, 127)   real s_y * out
llround rounds half away from zero.
"""
from __future__ import annotations

import math

import numpy as np


class ParamRange(ValueError):
    """A scale or threshold the definition cannot represent."""


def llround(x: float) -> int:
    """Nearest integer, halves away from zero (C's llround), exact."""
    if x < 0:
        return -llround(-x)
    f = math.floor(x)
    return int(f) + (1 if x - f >= 0.5 else 0)  # x - floor(x) is exact for doubles


def _f32(v) -> float:
    return float(np.float32(v))


def gelu_params(s_x, s_y, c):
    """(M, s, G[32], Mo, so) for input scale s_x, output scale s_y and gate
    range c.  Raises ParamRange for non-finite or non-positive inputs and for
    multipliers or shifts out of range."""
    s_x, s_y, c = _f32(s_x), _f32(s_y), _f32(c)
    for v in (s_x, s_y, c):
        if not (math.isfinite(v) and v > 0.0):
            raise ParamRange("scales and c must be finite and > 0")
    r = (s_x * 31.0) / (2.0 * c)
    s = 26
    while s > 1 and llround(math.ldexp(r, s)) > 1 << 24:
        s -= 1
    M = llround(math.ldexp(r, s))
    if M < 1 or M > 1 << 24:
        raise ParamRange("index multiplier out of range")
    G = [0] * 32
    G[31] = 32768
    for i in range(1, 31):
        t = ((2 * i - 31) * c) / 31.0
        G[i] = llround(32768.0 * (0.5 * math.erfc(-t / math.sqrt(2.0))))
    m = s_x / (32768.0 * s_y)
    f, e = math.frexp(m)
    Mo = llround(f * 2.0 ** 31)
    if Mo == 1 << 31:
        Mo, e = 1 << 30, e + 1
    so = 31 - e
    if not 1 <= so <= 62:
        raise ParamRange("requant shift out of range")
    return M, s, G, Mo, so


def gelu_index(q, M: int, s: int):
    """Table index of int8 codes q (numpy int64 arithmetic, >> is floor)."""
    q = np.asarray(q, dtype=np.int64)
    return np.clip(16 + ((q * M) >> s), 0, 31)


def gelu_codes(q, params):
    """Integer GELU of int8 codes q (any shape) -> int8 codes."""
    M, s, G, Mo, so = params
    q = np.asarray(q, dtype=np.int64)
    y = q * np.asarray(G, dtype=np.int64)[gelu_index(q, M, s)]
    out = (y * Mo + (1 << (so - 1))) >> so
    return np.clip(out, -127, 127).astype(np.int8)


def gelu(q, s_x, s_y, c):
    """gelu_codes with the parameters derived from (s_x, s_y, c)."""
    return gelu_codes(q, gelu_params(s_x, s_y, c))


def gelu_real(x: float) -> float:
    """The real GELU, x * Phi(x) (for error bounds in the tests)."""
    return x * 0.5 * math.erfc(-x / math.sqrt(2.0))
