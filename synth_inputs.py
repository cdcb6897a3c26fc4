"""Seeded synthetic inputs for the ISPA hot path.

This module is shared by the fp64 oracle tests, the CUDA parity tests and
``bench.py``.  It holds none of the method's arithmetic: only random draws,
round-to-nearest-even conversion of those draws to bf16, and the frame/token
bookkeeping of each workload.  Every generator takes an explicit key so that
the same tensor is reproduced bit for bit by every caller.

Workload shapes follow the autoregressive video generators the ISPA pages
compress (1.3B-class: 12 heads x 128, 30 layers; 14B-class: 40 heads x 128,
40 layers; 1560 tokens per latent frame; chunks of 3 latent frames; a sink of
initial frames that stays in the local group).  The pages' own evaluation
(VBench-Long on MovieGen prompts with trained generators) cannot run here;
these seeded tensors stand in for the attention inputs of those models.
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Dict, Iterable, Optional

import numpy as np

ROOT_SEED = 20260702


# ---------------------------------------------------------------------------
# seeding
# ---------------------------------------------------------------------------
def _key_int(part) -> int:
    if isinstance(part, (int, np.integer)):
        return int(part) & 0xFFFFFFFF
    return zlib.crc32(str(part).encode("utf-8"))


def rng(*key) -> np.random.Generator:
    """A PCG64 generator seeded by ROOT_SEED and an arbitrary key tuple."""
    ss = np.random.SeedSequence([ROOT_SEED] + [_key_int(k) for k in key])
    return np.random.Generator(np.random.PCG64(ss))


# ---------------------------------------------------------------------------
# bf16 rounding of draws (host side, so both sides see identical values)
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # u + 0x7FFF + (bit 16 of u), in place in one uint32 temporary: only NaN
    # patterns (overwritten below) can carry out of 32 bits
    r = u >> 16
    r &= 1
    r += 0x7FFF
    r += u
    r >>= 16
    out = r.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 array holding exactly the bf16 values nearest to x."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# ---------------------------------------------------------------------------
# shapes
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class AttnShape:
    """Frame layout of one attention call.

    The K/V buffer of each instance holds ``kv_frames`` frames in order
    sink | history | current.  Queries are the current chunk's tokens.
    Group ranges are half-open frame intervals.
    """

    B: int
    H: int
    d: int
    tpf: int
    sink_frames: int
    hist_begin: int
    hist_end: int
    cur_begin: int
    cur_end: int
    kv_frames: int

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def Lq(self) -> int:
        return (self.cur_end - self.cur_begin) * self.tpf

    @property
    def Lkv(self) -> int:
        return self.kv_frames * self.tpf

    @property
    def local_rows(self) -> np.ndarray:
        """Token rows of the local group: sink frames union current frames."""
        f = set(range(0, self.sink_frames)) | set(range(self.cur_begin, self.cur_end))
        return np.array([r for fr in sorted(f) for r in range(fr * self.tpf, (fr + 1) * self.tpf)],
                        dtype=np.int64)

    @property
    def hist_rows(self) -> np.ndarray:
        return np.arange(self.hist_begin * self.tpf, self.hist_end * self.tpf, dtype=np.int64)

    def with_batch(self, B: int) -> "AttnShape":
        return dataclasses.replace(self, B=B)


def video_shape(H: int, hist_frames: int, *, B: int = 1, d: int = 128, tpf: int = 1560,
                sink: int = 3, chunk: int = 3) -> AttnShape:
    """Sink | history | current layout used by the 1.3B- and 14B-shaped workloads."""
    hb, he = sink, sink + hist_frames
    return AttnShape(B=B, H=H, d=d, tpf=tpf, sink_frames=sink, hist_begin=hb, hist_end=he,
                     cur_begin=he, cur_end=he + chunk, kv_frames=he + chunk)


# Tiny fp32 case: 2 heads x 32, 16 tokens/frame, sink 1, history 6, current 1.
TINY = AttnShape(B=1, H=2, d=32, tpf=16, sink_frames=1, hist_begin=1, hist_end=7,
                 cur_begin=7, cur_end=8, kv_frames=8)
# 1.3B-shaped layer: 12 x 128, 1560 tokens/frame, sink 3, history 15, chunk 3.
SHAPE_1P3B = video_shape(12, 15)
# 14B-shaped layer: 40 x 128, sink 3, history 60, chunk 3.
SHAPE_14B = video_shape(40, 60)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: AttnShape
    dtype: str                 # "f32" or "bf16" for Q/K/V
    layers: int
    warmup_chunks: int
    post_chunks: int
    x: float                   # ISPA-x, fraction of layers converted
    lambda_rel: float          # lambda = lambda_rel * tr(G) / D
    history: str               # "iid" or "drift"


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", TINY, "f32", 1, 4, 0, 0.0, 1e-4, "iid"),
    "layer_1p3b": Workload("layer_1p3b", SHAPE_1P3B, "bf16", 1, 1, 0, 0.0, 1e-4, "iid"),
    "model_1p3b": Workload("model_1p3b", SHAPE_1P3B, "bf16", 30, 8, 16, 0.5, 1e-4, "drift"),
    "model_14b": Workload("model_14b", SHAPE_14B, "bf16", 40, 8, 0, 0.5, 1e-4, "drift"),
}


# ---------------------------------------------------------------------------
# tensors
# ---------------------------------------------------------------------------
def _normal(g: np.random.Generator, shape, std: float) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _finish(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16(x) if dtype == "bf16" else np.ascontiguousarray(x, np.float32)


def qkv_std(shape: AttnShape, dtype: str) -> float:
    """N(0,1)/sqrt(d) for the tiny fp32 case, N(0,1) for the bf16 video shapes."""
    return 1.0 / math.sqrt(shape.d) if dtype == "f32" else 1.0


def iid_qkv(shape: AttnShape, dtype: str, key: Iterable) -> Dict[str, np.ndarray]:
    """Q [B,Lq,H,d], K/V [B,Lkv,H,d] with i.i.d. normal entries (float32 holding exact values)."""
    key = tuple(key)
    std = qkv_std(shape, dtype)
    out = {}
    for name, rows in (("q", shape.Lq), ("k", shape.Lkv), ("v", shape.Lkv)):
        g = rng(*key, name)
        out[name] = _finish(_normal(g, (shape.B, rows, shape.H, shape.d), std), dtype)
    return out


def projection_weight(D: int, Dout: int, key: Iterable, dtype: str = "f32") -> np.ndarray:
    """Output projection W [D, Dout] (row-vector convention y = a W), entries N(0, 1/D)."""
    g = rng(*tuple(key), "W")
    return _finish(_normal(g, (D, Dout), 1.0 / math.sqrt(D)), dtype)


def drift_layer_kv(shape: AttnShape, dtype: str, layer: int, key: Iterable = ()) -> Dict[str, np.ndarray]:
    """Sink + history K/V of one layer, history as a low-rank drift of the sink.

    For every head and for X in {K, V}: U, Vr ~ N(0, 1/d) of size d x 64 and a
    per-layer amplitude alpha ~ U[0.5, 2].  History frame j (1-based) copies sink
    frame b = (j-1) mod S and adds alpha * (j/Hf) * X_sink[b] U Vr^T plus
    N(0, 0.1^2) noise.  Returns K/V [B, hist_end*tpf, H, d] (current frames are
    drawn per chunk by :func:`chunk_qkv`).
    """
    key = tuple(key)
    S, Hf, tpf, d = shape.sink_frames, shape.hist_end - shape.hist_begin, shape.tpf, shape.d
    alpha = float(rng(*key, "alpha", layer).uniform(0.5, 2.0))
    out = {}
    std = qkv_std(shape, dtype)
    for name in ("k", "v"):
        g = rng(*key, "drift", layer, name)
        sink = _normal(g, (shape.B, S * tpf, shape.H, d), std)
        hist = np.empty((shape.B, Hf * tpf, shape.H, d), np.float32)
        for h in range(shape.H):
            U = _normal(g, (d, 64), 1.0 / math.sqrt(d))
            Vr = _normal(g, (d, 64), 1.0 / math.sqrt(d))
            P = (U @ Vr.T).astype(np.float32)
            for j in range(1, Hf + 1):
                b = (j - 1) % S
                base = sink[:, b * tpf:(b + 1) * tpf, h, :]
                noise = _normal(g, base.shape, 0.1)
                hist[:, (j - 1) * tpf:j * tpf, h, :] = base + np.float32(alpha * j / Hf) * (base @ P) + noise
        out[name] = _finish(np.concatenate([sink, hist], axis=1), dtype)
    out["alpha"] = alpha
    return out


def chunk_qkv(shape: AttnShape, dtype: str, layer: int, chunk: int, key: Iterable = ()) -> Dict[str, np.ndarray]:
    """Q [B,Lq,H,d] and the current frames' K/V [B,Lq,H,d] of one chunk of one layer."""
    key = tuple(key)
    std = qkv_std(shape, dtype)
    out = {}
    for name in ("q", "k", "v"):
        g = rng(*key, "chunk", layer, chunk, name)
        out[name] = _finish(_normal(g, (shape.B, shape.Lq, shape.H, shape.d), std), dtype)
    return out


def assemble_kv(prefix: np.ndarray, current: np.ndarray, shape: AttnShape) -> np.ndarray:
    """K/V buffer [B, kv_frames*tpf, H, d] = frames [0, cur_begin) from prefix, then current."""
    assert prefix.shape[1] == shape.cur_begin * shape.tpf
    return np.ascontiguousarray(np.concatenate([prefix, current], axis=1))


def random_groups_shape(g: np.random.Generator, *, max_frames: int = 12, d: Optional[int] = None,
                        H: Optional[int] = None, tpf: Optional[int] = None, B: Optional[int] = None) -> AttnShape:
    """A random valid frame layout (possibly empty history, sink overlapping current)."""
    tpf = tpf or int(g.integers(1, 9))
    d = d or int(g.choice([32, 64, 128]))
    H = H or int(g.integers(1, 4))
    B = B or int(g.integers(1, 3))
    S = int(g.integers(0, 3))
    Hf = int(g.integers(0, max_frames))
    C = int(g.integers(1, 4))
    hb, he = S, S + Hf
    return AttnShape(B=B, H=H, d=d, tpf=tpf, sink_frames=S, hist_begin=hb, hist_end=he,
                     cur_begin=he, cur_end=he + C, kv_frames=he + C)


def activation_rows(M: int, K: int, key: Iterable) -> np.ndarray:
    """Activation-like rows [M, K] in bf16 values for the 8-bit quantisers.

    Row magnitudes log-uniform over 1e-4 .. 1e2 (so some rows reach the e4m3
    subnormal range after scaling), a few outlier channels at 20x, row 0 all
    zeros and row 1 a single nonzero entry when M allows.
    """
    g = rng(*tuple(key), "act")
    x = _normal(g, (M, K), 1.0)
    x *= (10.0 ** g.uniform(-4.0, 2.0, size=(M, 1))).astype(np.float32)
    if K >= 8:
        x[:, g.choice(K, size=max(1, K // 128), replace=False)] *= np.float32(20.0)
    if M >= 1:
        x[0] = 0.0
    if M >= 2:
        x[1] = 0.0
        x[1, K // 3] = -3.0
    return round_to_bf16(x)


# ---------------------------------------------------------------------------
# device-side draws of the same recipes (timing runs only: the values come
# from torch's generator, not from the PCG64 streams above, so no oracle
# comparison uses them)
# ---------------------------------------------------------------------------
def torch_generator(device, *key):
    """A torch generator on `device` seeded from ROOT_SEED and a key tuple."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([ROOT_SEED] + [_key_int(k) for k in key]).generate_state(1)[0]))
    return g


def device_normal_bf16(shape, device, gen, std: float = 1.0):
    """N(0, std^2) draws in fp32 on the device, rounded to bf16."""
    import torch
    x = torch.randn(shape, device=device, dtype=torch.float32, generator=gen)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def drift_layer_kv_device(shape: AttnShape, layer: int, key: Iterable, device):
    """The drift history recipe of :func:`drift_layer_kv` drawn on the device:
    K, V [B, hist_end*tpf, H, d] in bf16 (sink frames, then every history frame
    as its base sink frame plus alpha (j/Hf) X U Vr^T and N(0, 0.1^2) noise)."""
    import torch
    key = tuple(key)
    S, Hf, tpf, d, H = shape.sink_frames, shape.hist_end - shape.hist_begin, shape.tpf, shape.d, shape.H
    alpha = float(rng(*key, "alpha", layer).uniform(0.5, 2.0))
    out = {}
    for name in ("k", "v"):
        g = torch_generator(device, *key, "drift", layer, name)
        sink = torch.randn((shape.B, S * tpf, H, d), device=device, dtype=torch.float32, generator=g)
        U = torch.randn((H, d, 64), device=device, generator=g) / math.sqrt(d)
        Vr = torch.randn((H, d, 64), device=device, generator=g) / math.sqrt(d)
        P = torch.matmul(U, Vr.transpose(1, 2))                      # [H, d, d]
        buf = torch.empty((shape.B, (S + Hf) * tpf, H, d), device=device, dtype=torch.bfloat16)
        buf[:, :S * tpf] = sink.to(torch.bfloat16)
        for j in range(1, Hf + 1):
            b = (j - 1) % S
            base = sink[:, b * tpf:(b + 1) * tpf]                     # [B, tpf, H, d]
            drift = torch.einsum("bthd,hde->bthe", base, P)
            noise = torch.randn(base.shape, device=device, generator=g) * 0.1
            buf[:, (S + j - 1) * tpf:(S + j) * tpf] = (base + (alpha * j / Hf) * drift + noise).to(torch.bfloat16)
        out[name] = buf
    out["alpha"] = alpha
    return out
