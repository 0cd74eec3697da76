"""Seeded synthetic inputs shaped like the workloads of RTR-DiT's streaming
rerenderer.

This module holds only random-number generation and storage-format
conversion; none of the method's arithmetic.  Both the CUDA path's tests and
the oracle's tests draw their inputs here, so the two sides see the same bits.

Recipe: ``numpy.random.default_rng(seed)``, ``standard_normal(dtype=float32)``
times a scale, then rounded to bfloat16 with round-to-nearest-even (or kept
as float32 for the fp32 workload).  Tensors are [tokens, heads, head_dim].
Per workload the reference K, V (and text K, V) are drawn first, then the
window frames (K then V per frame), then per chunk Q, K, V.

The pages' evaluation clips (50 Pexels videos at 832x640, 24 fps, 5 s) are
not available here; these tensors stand in for the projected Q/K/V such clips
produce in a Wan-style DiT.
"""
from dataclasses import dataclass, field

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits.
    Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact float32 value of bfloat16 bit patterns."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(rng: np.random.Generator, shape, scale: float, dtype: str) -> np.ndarray:
    """N(0,1)*scale in the storage format: uint16 bf16 bits or float32."""
    x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(scale)
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    if dtype == "f32":
        return x
    raise ValueError(dtype)


@dataclass(frozen=True)
class Workload:
    """Shape of one streaming / prefill workload."""
    name: str
    dtype: str            # "bf16" | "f32"
    layers: int
    heads: int
    head_dim: int
    k: int                # tokens per latent frame
    ref_frames: int
    window_frames: int
    chunk_frames: int
    scale: float          # std of the synthetic Q/K/V
    seed: int
    frames_total: int = 0
    steps_per_chunk: int = 1
    text_tokens: int = 0
    switch_every: int = 0


# The five workloads: a tiny fp32 stream; one Wan-1.3B-shaped layer (a chunk
# of 3 latent frames against 1 reference + 21 window frames); a block-causal
# prefill of 22 frames; a 30-layer, 120-frame stream; a 40-head stream with
# text cross-attention and a style switch every 16 frames.
TINY_F32 = Workload("tiny fp32 stream: H=2 d=64 k=16 ref=1 W=4, 10 frames one at a time",
                    "f32", 1, 2, 64, 16, 1, 4, 1, 1.0, 0, frames_total=10)
WAN13_LAYER = Workload("Wan-1.3B-like layer: H=12 d=128 k=1560, chunk of 3 frames vs ref 1 + window 21",
                       "bf16", 1, 12, 128, 1560, 1, 21, 3, 0.5, 1)
PREFILL_22 = Workload("block-causal prefill: H=12 d=128 k=1560, 1 ref + 21 frames = 34320 tokens",
                      "bf16", 1, 12, 128, 1560, 0, 22, 22, 0.5, 2)
LONG_STREAM = Workload("long stream: 30 layers x H=12 d=128 k=1560, 120 frames in chunks of 3, 2 steps, W=21",
                       "bf16", 30, 12, 128, 1560, 1, 21, 3, 0.5, 3, frames_total=120,
                       steps_per_chunk=2)
SWITCH_14B = Workload("14B-like with switching: H=40 d=128 k=1560, W=21, text 512, switch every 16 of 64 frames",
                      "bf16", 1, 40, 128, 1560, 1, 21, 1, 0.5, 4, frames_total=64,
                      text_tokens=512, switch_every=16)

WORKLOADS = [TINY_F32, WAN13_LAYER, PREFILL_22, LONG_STREAM, SWITCH_14B]


def tokens(w: Workload, frames: int) -> tuple:
    return (frames * w.k, w.heads, w.head_dim)


@dataclass
class StreamInputs:
    """Inputs of one streaming attention call after a pre-filled window."""
    ref_k: np.ndarray
    ref_v: np.ndarray
    window_k: list = field(default_factory=list)   # per frame [k, H, d]
    window_v: list = field(default_factory=list)
    q: np.ndarray = None                            # [C*k, H, d]
    k_cur: np.ndarray = None
    v_cur: np.ndarray = None


def stream_layer_inputs(w: Workload, window_fill: int = None, seed: int = None) -> StreamInputs:
    """Reference K, V; ``window_fill`` frames of K, V to append; one chunk of
    Q, K, V -- drawn in that order from ``default_rng(seed)``."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    fill = w.window_frames if window_fill is None else window_fill
    out = StreamInputs(normal(rng, tokens(w, w.ref_frames), w.scale, w.dtype),
                       normal(rng, tokens(w, w.ref_frames), w.scale, w.dtype))
    for _ in range(fill):
        out.window_k.append(normal(rng, tokens(w, 1), w.scale, w.dtype))
        out.window_v.append(normal(rng, tokens(w, 1), w.scale, w.dtype))
    shape = tokens(w, w.chunk_frames)
    out.q = normal(rng, shape, w.scale, w.dtype)
    out.k_cur = normal(rng, shape, w.scale, w.dtype)
    out.v_cur = normal(rng, shape, w.scale, w.dtype)
    return out


def prefill_inputs(w: Workload, n_tokens: int = None, seed: int = None):
    """Q, K, V of one whole sequence [n, H, d] (default: all frames of w)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    n = w.chunk_frames * w.k if n_tokens is None else n_tokens
    shape = (n, w.heads, w.head_dim)
    return (normal(rng, shape, w.scale, w.dtype), normal(rng, shape, w.scale, w.dtype),
            normal(rng, shape, w.scale, w.dtype))


def random_qkv(seed: int, n: int, heads: int, d: int, dtype: str = "bf16", scale: float = 1.0):
    """Three independent [n, heads, d] tensors from one seed (small tests)."""
    rng = np.random.default_rng(seed)
    return tuple(normal(rng, (n, heads, d), scale, dtype) for _ in range(3))
