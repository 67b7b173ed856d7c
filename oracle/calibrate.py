"""Plain numpy oracle of the adaptive clip threshold.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` (and nothing in the product
library calls it).

The summary pages ("[Paper] IntAttention：全整数注意力流水线用于高效边缘推理" and
its Korean edition, sections 概览 / Overview and 局限性与未来工作 / Limitations &
Future Work) describe the clip as sparsity-aware, limiting extreme
activations dynamically, and name an adaptive / learned threshold as future
work; they give no rule.  The reading implemented here chooses each head's
threshold from the integer scores of a sample of query rows:

    rows    i = stride - 1, 2 stride - 1, ... < Lq   (every stride-th row)
    G_i     = m_i - S_i,(K): the gap from the row max to the K-th largest
              score over the row's valid keys (causal: j <= i + Lk - Lq);
              with fewer than K valid keys, the gap to the smallest one
    G       = max of G_i over the sampled rows of the head (and over the
              batch; over all heads for per-tensor scales)
    c       = clamp(alpha * G * 31 / 30, c_min, c_max),  alpha = s_q s_k / sqrt(d)
              (IEEE double in that order, then rounded to float)

so that in every sampled row at least K keys keep an index <= 30 (the
index of a gap g is round(g alpha 31 / c) <= round(30 g / G) <= 30), while
the threshold is as small, and the exp table as fine (spacing c / 31), as
that allows.
"""
import numpy as np


def gaps(q, k, causal, keep, stride):
    """G per (batch, head): int64 [B, H]."""
    q = np.asarray(q, dtype=np.int64)
    k = np.asarray(k, dtype=np.int64)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    rows = np.arange(stride - 1, Lq, stride)
    G = np.zeros((B, H), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            S = q[b, h, rows] @ k[b, h].T          # exact integer scores [rows, Lk]
            for r, i in enumerate(rows):
                n = min(Lk, i + (Lk - Lq) + 1) if causal else Lk
                s = np.sort(S[r, :n])[::-1]          # descending
                kth = s[min(keep, n) - 1]
                G[b, h] = max(G[b, h], s[0] - kth)
    return G


def thresholds(q, k, per_head, s_q, s_k, causal, keep, stride, c_min, c_max):
    """Per-head (or one per-tensor) clip thresholds as float32."""
    G = gaps(q, k, causal, keep, stride)
    d = q.shape[-1]
    Gh = G.max(axis=0) if per_head else np.array([G.max()])
    sq = np.atleast_1d(np.asarray(s_q, dtype=np.float32)).astype(np.float64)
    sk = np.atleast_1d(np.asarray(s_k, dtype=np.float32)).astype(np.float64)
    out = np.empty(Gh.shape[0], dtype=np.float32)
    for h in range(Gh.shape[0]):
        alpha = (sq[h] * sk[h]) / np.sqrt(np.float64(d))
        c = ((alpha * np.float64(Gh[h])) * 31.0) / 30.0
        out[h] = np.float32(min(max(c, float(np.float32(c_min))), float(np.float32(c_max))))
    return out, Gh
