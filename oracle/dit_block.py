"""Oracle of one DiT block around the frame-causal attention (TEST
INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's oracle legs, never by the library's product path).

Sources: papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
Architecture (the patchified tokens of the reference and the video frames go
through the DiT blocks, whose 3D attention carries the temporal causal
mask; the clean latent is noised at a timestep t that conditions the model),
Key Designs 1 (text enters through cross attention); gist.science explainer
"Adapting VACE for Real-Time Autoregressive Video Diffusion", section 1
(rotary position encodings are baked into the cached keys).  The pages name
a Wan DiT but give no block internals, so the block below is the plainest
transformer block that has those parts; every choice the pages leave open
is marked "reading":

  h  = LN(x) * (1 + scale1) + shift1                       (reading: timestep
                                                             modulation as six
                                                             per-channel vectors)
  q, k, v = split(h Wqkv + bqkv);  q, k <- RoPE3D(q, k)    (reading: 3D rotary
                                                             encoding, below)
  o  = frame-causal attention of q against the cache's [ref | window] and the
       chunk's own k, v                                     (Key Designs 2, 4)
  x1 = x + gate1 * (o Wo + bo)
  o2 = attention of (LN(x1) Wq2 + bq2) against the text cache (Key Designs 1)
  x2 = x1 + (o2 Wo2 + bo2)
  x3 = x2 + gate2 * (GELU(h3 W1 + b1) W2 + b2),  h3 = LN(x2) * (1 + scale2) + shift2

LN: mean and variance over the model dimension, eps 1e-6, no affine
(reading).  GELU: the tanh form 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715
x^3))) (reading).  RoPE3D (reading): each head's d channels split into a
temporal part of d - 2P and two spatial parts of P = 2 floor(d/6) channels
(height, width); within a part of size S, channel pair (2j, 2j+1) is rotated
by the angle pos * 10000^(-2j/S), the rotary form of Su et al., "RoFormer"
(2021), eq. 13-15.  Token i of a chunk of frames is at frame t0 + i // k,
row (i % k) // grid_w, column i % grid_w.

Precision (reading of "bf16 operands, fp32 accumulation"): the block's
inputs are bf16 values; every tensor the next step consumes as an operand
(h, q, k, v, o, x1, the cross-attention query and output, x2, h3, the GELU
output, x3) is rounded to bf16, round-to-nearest-even; everything else is
fp64.  Weights are [in, out] (y = x W + b).
"""
import math

import numpy as np

from .attention import decode

EPS = 1e-6
ROPE_BASE = 10000.0


def round_bf16(a):
    """Nearest bfloat16 value (8 significant bits), ties to even, in fp64."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                  # a = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0), e - 8)


def bf16_bits(values):
    """Bit patterns (uint16) of values that are already bfloat16 numbers."""
    v = np.ascontiguousarray(values, np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def layer_norm(x, eps=EPS):
    """(x - mean) / sqrt(var + eps) over the last axis (biased variance)."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def gelu_tanh(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def rope_parts(d):
    """Channel counts of the (temporal, height, width) parts of a head."""
    p = 2 * (d // 6)
    return d - 2 * p, p, p


def token_positions(n_frames, grid_h, grid_w, t0):
    """(frame, row, column) of every token of a chunk of n_frames frames."""
    k = grid_h * grid_w
    i = np.arange(n_frames * k, dtype=np.int64)
    r = i % k
    return t0 + i // k, r // grid_w, r % grid_w


def rope3d(x, t, y, xc, base=ROPE_BASE):
    """Rotate x [n, H, d] by the 3D rotary encoding of positions (t, y, xc)
    ([n] each); returns fp64 [n, H, d]."""
    x = np.asarray(x, np.float64)
    n, H, d = x.shape
    out = x.copy()
    c0 = 0
    for size, pos in zip(rope_parts(d), (t, y, xc)):
        j = np.arange(size // 2)
        theta = base ** (-2.0 * j / size)
        ang = np.asarray(pos, np.float64)[:, None] * theta[None, :]          # [n, size/2]
        cos, sin = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
        a = x[:, :, c0 + 2 * j]
        b = x[:, :, c0 + 2 * j + 1]
        out[:, :, c0 + 2 * j] = a * cos - b * sin
        out[:, :, c0 + 2 * j + 1] = a * sin + b * cos
        c0 += size
    return out


def dit_block(x, mod, w, cache, xcache, n_cur_frames, grid_h, grid_w, t0, eps=EPS, rows=None):
    """One block on the current chunk.

    x: bf16 bits [n, D] (n = n_cur_frames * grid_h * grid_w, D = H d); mod:
    bf16 bits [6, D] (shift1, scale1, gate1, shift2, scale2, gate2); w: dict
    of bf16 bits: wqkv [D, 3D], bqkv [3D], wo [D, D], bo [D], wq2 [D, D],
    bq2 [D], wo2 [D, D], bo2 [D], w1 [D, F], b1 [F], w2 [F, D], b2 [D].
    cache: oracle.ReferenceCache holding the layer's reference and window
    (keys already rotary-encoded); xcache: oracle.CrossCache with the text
    keys and values.  Returns a dict with "out" (fp64 values of the bf16
    result [n, D]) and "k", "v" (bf16 bits [n, H, d], the chunk's rotated
    keys and values, which a commit appends to the cache).  ``rows``
    selects output rows: every token's keys and values are still formed (the
    attention needs them), the rest only for those rows, so "out" then has
    one row per selected token."""
    H, d = cache.H, cache.d
    X = decode(x, "bf16")
    n, D = X.shape
    M = decode(mod, "bf16")
    W = {name: decode(a, "bf16") for name, a in w.items()}
    r = round_bf16

    rows = np.arange(n, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    m = rows.size
    h = r(layer_norm(X, eps) * (1.0 + M[1]) + M[0])
    qkv = h @ W["wqkv"] + W["bqkv"]
    q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(n, H, d) for i in range(3))
    t, yy, xx = token_positions(n_cur_frames, grid_h, grid_w, t0)
    qb = np.zeros((n, H, d), np.uint16)
    qb[rows] = bf16_bits(r(rope3d(q[rows], t[rows], yy[rows], xx[rows])))
    kb = bf16_bits(r(rope3d(k, t, yy, xx)))
    vb = bf16_bits(r(v))
    o = r(cache.stream_attention(qb, kb, vb, n_cur_frames, rows=rows)).reshape(m, D)
    X = X[rows]
    x1 = r(X + M[2] * (o @ W["wo"] + W["bo"]))
    q2 = r(r(layer_norm(x1, eps)) @ W["wq2"] + W["bq2"])
    o2 = r(xcache.attention(bf16_bits(q2).reshape(m, H, d))).reshape(m, D)
    x2 = r(x1 + (o2 @ W["wo2"] + W["bo2"]))
    h3 = r(layer_norm(x2, eps) * (1.0 + M[4]) + M[3])
    f = r(gelu_tanh(h3 @ W["w1"] + W["b1"]))
    x3 = r(x2 + M[5] * (f @ W["w2"] + W["b2"]))
    return {"out": x3, "k": kb, "v": vb}


def dit_block_flops(n_tokens, d_model, d_ffn):
    """Matmul flops of the block's six projections per call (2 per multiply-add)."""
    return 2.0 * n_tokens * (6.0 * d_model * d_model + 2.0 * d_model * d_ffn)
