"""Seeded synthetic workloads for the integer attention forward.

This module only draws random numbers and quantises them to int8.  It holds
none of the attention arithmetic (scores, IndexSoftmax, P.V, requantisation):
both the CUDA path and the CPU oracle receive its outputs as plain inputs.

Recipe (the same for every workload):
  * fp32 draws from numpy ``Generator(PCG64(seed))`` with
    ``seed = 20251126 + workload index``; one child generator per tensor and
    per batch entry (``SeedSequence.spawn``), so large tensors are generated
    chunk by chunk with identical results.
  * values are N(0, 1), or Student-t with 4 degrees of freedom;
  * outlier channels: ``round(frac * H * d)`` distinct (head, channel) pairs
    drawn per tensor, multiplied by a constant factor;
  * symmetric int8 quantisation with zero-point 0:
    ``s = max|x| / 127`` over the whole tensor (per-tensor) or over each head
    (per-head), ``q = clamp(rint(x / s), -127, 127)``;
  * output scale ``s_o = max|O| / 127`` where O is fp64 softmax attention of
    the de-quantised int8 inputs (scaled by 1/sqrt(d), causal mask applied),
    evaluated on an evenly spaced sample of at most 64 query rows per
    (batch, head).  Rows outside the sample may saturate at +-127, which the
    requantisation clamp handles.

The shapes are those of single attention layers of BERT-base, ViT-B/16,
GPT-2 small and LLaMA-7B; no dataset or trained weight is involved.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SEED_BASE = 20251126


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    Lq: int
    Lk: int
    d: int
    causal: bool
    dist: str                  # "normal" or "student_t4"
    outlier_frac: float
    outlier_scale: float
    outlier_tensors: str       # subset of "qkv"
    per_head: bool
    clip_c: float
    decode: bool = False
    Lmax: int = 0              # decode: cache capacity (rows per (b, h))
    kv_bits: int = 8           # 4: K and V codes in [-7, 7], stored as packed nibbles

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def effective_ops(self) -> float:
        """4*B*H*Lq*Lk*d, halved for a causal mask."""
        ops = 4.0 * self.B * self.H * self.Lq * self.Lk * self.d
        return ops / 2 if self.causal else ops

    @property
    def decode_bytes(self) -> int:
        """K and V cache rows read plus the q and out vectors."""
        kv = 2 * self.B * self.H * self.Lk * self.d * self.kv_bits // 8
        return kv + 2 * self.B * self.H * self.d

    @property
    def kv_qmax(self) -> int:
        """Largest K/V code magnitude of the symmetric quantisation."""
        return 7 if self.kv_bits == 4 else 127


WORKLOADS = {
    w.name: w
    for w in [
        Workload("bert_base_l128", 0, 1, 12, 128, 128, 64, False, "normal",
                 0.02, 8.0, "qkv", False, 8.0),
        Workload("bert_base_b8_l512", 1, 8, 12, 512, 512, 64, False, "normal",
                 0.02, 8.0, "qkv", False, 8.0),
        Workload("vit_b16_l197", 2, 32, 12, 197, 197, 64, False, "student_t4",
                 0.0, 1.0, "", True, 6.0),
        Workload("gpt2_small_causal_l2048", 3, 4, 12, 2048, 2048, 64, True,
                 "normal", 0.02, 8.0, "qkv", False, 8.0),
        Workload("llama7b_causal_l8192", 4, 1, 32, 8192, 8192, 128, True,
                 "normal", 0.01, 16.0, "k", True, 10.0),
        Workload("llama7b_decode_b64_lk4096", 5, 64, 32, 1, 4096, 128, False,
                 "normal", 0.01, 16.0, "k", True, 10.0, decode=True, Lmax=4096),
        Workload("llama7b_decode_int4_b64_lk4096", 6, 64, 32, 1, 4096, 128, False,
                 "normal", 0.01, 16.0, "k", True, 10.0, decode=True, Lmax=4096, kv_bits=4),
    ]
}


def custom_workload(name: str, B: int, H: int, Lq: int, Lk: int, d: int,
                    causal: bool, *, per_head: bool = False, clip_c: float = 8.0,
                    dist: str = "normal", outlier_frac: float = 0.02,
                    outlier_scale: float = 8.0, outlier_tensors: str = "qkv",
                    index: int = 100, decode: bool = False,
                    Lmax: int = 0, kv_bits: int = 8) -> Workload:
    return Workload(name, index, B, H, Lq, Lk, d, causal, dist, outlier_frac,
                    outlier_scale, outlier_tensors, per_head, clip_c, decode,
                    Lmax if Lmax else Lk, kv_bits)


@dataclasses.dataclass
class Inputs:
    w: Workload
    q: np.ndarray          # int8 [B, H, Lq, d]
    k: np.ndarray          # int8 [B, H, Lk | Lmax, d]
    v: np.ndarray          # int8 [B, H, Lk | Lmax, d]
    s_q: np.ndarray        # float32 [1] or [H]
    s_k: np.ndarray
    s_v: np.ndarray
    s_o: np.ndarray


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape, dtype=np.float32)
    if dist == "student_t4":
        return rng.standard_t(4.0, size=shape).astype(np.float32)
    raise ValueError(dist)


def _tensor_chunks(w: Workload, which: str, L: int, nthreads: int):
    """fp32 draws of one tensor, one [H, L, d] chunk per batch entry."""
    ss = np.random.SeedSequence([w.seed, "qkv".index(which)])
    kids = ss.spawn(w.B + 1)
    # outlier (head, channel) pairs: drawn from the extra child
    pairs = np.zeros((0, 2), dtype=np.int64)
    if which in w.outlier_tensors and w.outlier_frac > 0:
        n = int(round(w.outlier_frac * w.H * w.d))
        flat = np.random.Generator(np.random.PCG64(kids[-1])).choice(
            w.H * w.d, size=n, replace=False)
        pairs = np.stack([flat // w.d, flat % w.d], axis=1)

    def one(b):
        x = _draw(np.random.Generator(np.random.PCG64(kids[b])), (w.H, L, w.d),
                  w.dist)
        for h, t in pairs:
            x[h, :, t] *= np.float32(w.outlier_scale)
        return x

    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        for b, x in enumerate(ex.map(one, range(w.B))):
            yield b, x


def _quantise(w: Workload, which: str, L: int, nthreads: int, qmax: int = 127):
    """Two passes over the seeded chunks: max|x| first, then codes in
    [-qmax, qmax] (int8 storage)."""
    amax = np.zeros(w.H, dtype=np.float64)
    for _, x in _tensor_chunks(w, which, L, nthreads):
        amax = np.maximum(amax, np.abs(x).max(axis=(1, 2)).astype(np.float64))
    if not w.per_head:
        amax = np.array([amax.max()])
    scale = (amax / float(qmax)).astype(np.float32)
    scale[scale == 0] = np.float32(1.0)
    out = np.empty((w.B, w.H, L, w.d), dtype=np.int8)
    sc = scale.astype(np.float64)
    sc_h = sc if w.per_head else np.repeat(sc, w.H)
    for b, x in _tensor_chunks(w, which, L, nthreads):
        y = np.rint(x.astype(np.float64) / sc_h[:, None, None])
        out[b] = np.clip(y, -qmax, qmax).astype(np.int8)
    return out, scale


def _sample_rows(Lq: int, n: int = 64) -> np.ndarray:
    if Lq <= n:
        return np.arange(Lq)
    return np.unique(np.round(np.linspace(0, Lq - 1, n)).astype(np.int64))


def _output_scale(w: Workload, q, k, v, s_q, s_k, s_v) -> np.ndarray:
    """max|O|/127 of fp64 softmax attention on de-quantised inputs (row sample)."""
    rows = _sample_rows(w.Lq)
    amax = np.zeros(w.H, dtype=np.float64)
    sq = np.broadcast_to(s_q.astype(np.float64), (w.H,)) if w.per_head else np.full(w.H, float(s_q[0]))
    sk = np.broadcast_to(s_k.astype(np.float64), (w.H,)) if w.per_head else np.full(w.H, float(s_k[0]))
    sv = np.broadcast_to(s_v.astype(np.float64), (w.H,)) if w.per_head else np.full(w.H, float(s_v[0]))
    off = w.Lk - w.Lq
    for b in range(w.B):
        qf = q[b][:, rows, :].astype(np.float64) * sq[:, None, None]
        kf = k[b][:, :w.Lk, :].astype(np.float64) * sk[:, None, None]
        vf = v[b][:, :w.Lk, :].astype(np.float64) * sv[:, None, None]
        logits = np.einsum("hid,hjd->hij", qf, kf) / math.sqrt(w.d)
        if w.causal:
            mask = np.arange(w.Lk)[None, :] > (rows[:, None] + off)
            logits = np.where(mask[None], -np.inf, logits)
        logits -= logits.max(axis=-1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=-1, keepdims=True)
        o = np.einsum("hij,hjd->hid", p, vf)
        amax = np.maximum(amax, np.abs(o).max(axis=(1, 2)))
    if not w.per_head:
        amax = np.array([amax.max()])
    s_o = (amax / 127.0).astype(np.float32)
    s_o[s_o == 0] = np.float32(1.0)
    return s_o


def make_inputs(w: Workload, nthreads: int = 8) -> Inputs:
    Lkv = w.Lmax if w.decode else w.Lk
    q, s_q = _quantise(w, "q", w.Lq, nthreads)
    k, s_k = _quantise(w, "k", Lkv, nthreads, w.kv_qmax)
    v, s_v = _quantise(w, "v", Lkv, nthreads, w.kv_qmax)
    s_o = _output_scale(w, q, k, v, s_q, s_k, s_v)
    return Inputs(w, q, k, v, s_q, s_k, s_v, s_o)


def pack_int4(x: np.ndarray) -> np.ndarray:
    """int8 codes in [-8, 7], [..., d] -> uint8 [..., d/2]: byte t holds
    channel 2t in bits 0-3 and channel 2t+1 in bits 4-7 (two's complement)."""
    x = np.asarray(x)
    if x.shape[-1] % 2 or x.min(initial=0) < -8 or x.max(initial=0) > 7:
        raise ValueError("int4 packing needs an even last dimension and codes in [-8, 7]")
    u = x.astype(np.uint8) & np.uint8(0x0F)
    return (u[..., 0::2] | (u[..., 1::2] << np.uint8(4))).astype(np.uint8)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    """Inverse of pack_int4: uint8 [..., d/2] -> int8 codes [..., d]."""
    p = np.asarray(p, dtype=np.uint8)
    lo = (p & np.uint8(0x0F)).astype(np.int16)
    hi = (p >> np.uint8(4)).astype(np.int16)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out).astype(np.int8)


@dataclasses.dataclass
class DeviceInputs:
    w: Workload
    q: "object"            # torch int8 tensors on the device
    k: "object"
    v: "object"
    s_q: np.ndarray
    s_k: np.ndarray
    s_v: np.ndarray
    s_o: np.ndarray


def make_inputs_torch(w: Workload, device) -> DeviceInputs:
    """Same recipe drawn with torch's generator on the device (for benchmark
    inputs too large to draw quickly with numpy; a different random stream
    from make_inputs, and never compared with the oracle)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    Lkv = w.Lmax if w.decode else w.Lk

    def one(which, L, qmax=127):
        x = torch.randn((w.B, w.H, L, w.d), generator=g, device=device, dtype=torch.float32)
        if w.dist == "student_t4":
            chi = torch.randn((4, w.B, w.H, L, w.d), generator=g, device=device).pow(2).sum(0)
            x = x / torch.sqrt(chi / 4.0)
        if which in w.outlier_tensors and w.outlier_frac > 0:
            n = int(round(w.outlier_frac * w.H * w.d))
            flat = torch.randperm(w.H * w.d, generator=g, device=device)[:n]
            for f in flat.tolist():
                x[:, f // w.d, :, f % w.d] *= w.outlier_scale
        amax = x.abs().amax(dim=(0, 2, 3)).double()
        if not w.per_head:
            amax = amax.max().reshape(1)
        scale = (amax / float(qmax)).float()
        scale[scale == 0] = 1.0
        sh = scale.double() if w.per_head else scale.double().expand(w.H)
        q = torch.clamp(torch.round(x.double() / sh.view(1, -1, 1, 1)), -qmax, qmax).to(torch.int8)
        return q, scale.cpu().numpy().astype(np.float32)

    q, s_q = one("q", w.Lq)
    k, s_k = one("k", Lkv, w.kv_qmax)
    v, s_v = one("v", Lkv, w.kv_qmax)
    # output scale from an fp64 row sample, as in make_inputs
    rows = torch.as_tensor(_sample_rows(w.Lq), device=device)
    sq = torch.as_tensor(np.array(np.broadcast_to(s_q, (w.H,))) if w.per_head else np.full(w.H, s_q[0]),
                         device=device, dtype=torch.float64)
    sk = torch.as_tensor(np.array(np.broadcast_to(s_k, (w.H,))) if w.per_head else np.full(w.H, s_k[0]),
                         device=device, dtype=torch.float64)
    sv = torch.as_tensor(np.array(np.broadcast_to(s_v, (w.H,))) if w.per_head else np.full(w.H, s_v[0]),
                         device=device, dtype=torch.float64)
    amax = torch.zeros(w.H, dtype=torch.float64, device=device)
    for b in range(w.B):
        qf = q[b][:, rows].double() * sq.view(-1, 1, 1)
        kf = k[b][:, :w.Lk].double() * sk.view(-1, 1, 1)
        vf = v[b][:, :w.Lk].double() * sv.view(-1, 1, 1)
        logits = torch.einsum("hid,hjd->hij", qf, kf) / math.sqrt(w.d)
        if w.causal:
            mask = torch.arange(w.Lk, device=device)[None, :] > (rows[:, None] + (w.Lk - w.Lq))
            logits = logits.masked_fill(mask[None], float("-inf"))
        o = torch.einsum("hij,hjd->hid", torch.softmax(logits, dim=-1), vf)
        amax = torch.maximum(amax, o.abs().amax(dim=(1, 2)))
    if not w.per_head:
        amax = amax.max().reshape(1)
    s_o = (amax / 127.0).float().cpu().numpy().astype(np.float32)
    s_o[s_o == 0] = np.float32(1.0)
    return DeviceInputs(w, q.contiguous(), k.contiguous(), v.contiguous(), s_q, s_k, s_v, s_o)


def pack_int4_torch(x):
    """pack_int4 for a torch int8 tensor on any device (same byte layout)."""
    import torch
    u = (x.to(torch.int16) & 0x0F).to(torch.uint8)
    return (u[..., 0::2] | (u[..., 1::2] << 4)).contiguous()


# ------------------------------------------------------------- integer GELU
# GELU input: the pre-activation of a transformer MLP (GPT-2 small: hidden
# 768 -> 3072).  Recipe: N(0, 1.5) draws, 1 % of the 3072 channels scaled by
# 4 (outlier channels), per-tensor symmetric int8 with s_x = max|x| / 127,
# s_y = s_x (GELU(x) <= max(x, 0)), gate range c = 4.
GELU_WORKLOADS = {
    "gpt2_small_mlp_gelu_b16_l1024_f3072": dict(tokens=16 * 1024, features=3072, c=4.0),
    "gelu_small_t512_f768": dict(tokens=512, features=768, c=4.0),
}


def gelu_inputs_torch(tokens: int, features: int, seed: int, device):
    """(codes int8 [tokens, features], s_x) drawn on `device`."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((tokens, features), generator=g, device=device, dtype=torch.float32) * 1.5
    n_out = max(1, round(0.01 * features))
    ch = torch.randperm(features, generator=g, device=device)[:n_out]
    x[:, ch] *= 4.0
    amax = float(x.abs().max())
    s_x = float(np.float32(amax / 127.0)) if amax > 0 else 1.0
    codes = torch.clamp(torch.round(x / s_x), -127, 127).to(torch.int8)
    return codes, s_x
