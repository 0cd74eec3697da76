"""GPU parity of the frame-causal attention against the fp64 oracle, through
the C ABI: streaming chunk attention over [reference | window | chunk], block-
causal prefill and unmasked cross-attention (papernotes.org note "DiT as
Real-Time Rerenderer", Method > Key Designs 2 and 4).

Small cases compare every output element and cover one or several tiles, ragged
frame and tile tails, frames smaller and larger than a tile, a wrapped ring
window, TV2V (no reference), an empty window and the degenerate k = 1 (token
causal) and k >= n (bidirectional) masks.  Full-size cases run the launch the
benchmark times and compare sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def rtr():
    from causal_attention_rtr_b200 import rtr as lib
    return lib


def build_stream(dtype, H, d, k, R, W, ref_on, appends, retain=None, seed=0, scale=1.0):
    """Create a library cache and an oracle cache with the same history."""
    lib = rtr()
    rng = np.random.default_rng(seed)
    c = lib.rtr_kvcache_create(1, H, d, k, R, W, dtype, 0)
    o = oracle.ReferenceCache(H, d, k, R, W, dtype)
    if ref_on and R > 0:
        kr = synth.normal(rng, (R * k, H, d), scale, dtype)
        vr = synth.normal(rng, (R * k, H, d), scale, dtype)
        lib.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
    for n in appends:
        kn = synth.normal(rng, (n * k, H, d), scale, dtype)
        vn = synth.normal(rng, (n * k, H, d), scale, dtype)
        lib.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), n)
        o.append(kn, vn, n)
    if retain is not None:
        lib.rtr_kvcache_retain_last(c, 0, retain)
        o.retain_last(retain)
    return c, o, rng


def run_stream_attention(c, dtype, H, d, k, C, rng, scale=1.0):
    shape = (C * k, H, d)
    q = synth.normal(rng, shape, scale, dtype)
    kc = synth.normal(rng, shape, scale, dtype)
    vc = synth.normal(rng, shape, scale, dtype)
    out = torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    rtr().rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), C, out)
    torch.cuda.synchronize()
    return q, kc, vc, out


STREAM_CASES = [
    # dtype, H, d, k, R, W, C, ref, appends, retain
    ("bf16", 2, 128, 16, 1, 4, 1, True, [1] * 6, None),        # wrapped ring, one tile
    ("bf16", 2, 128, 17, 1, 4, 3, True, [2], None),            # partial window, 3-frame chunk
    ("bf16", 3, 128, 1, 1, 4, 5, True, [1] * 7, None),         # k = 1: token-causal chunk
    ("bf16", 2, 128, 200, 1, 3, 2, True, [2, 3, 1], None),     # frames span tiles, ragged tails
    ("bf16", 2, 128, 128, 1, 3, 2, True, [3, 1], None),        # tile-aligned frames
    ("bf16", 2, 128, 100, 1, 4, 3, False, [3, 3], None),       # TV2V: no reference
    ("bf16", 2, 128, 60, 1, 5, 2, True, [4, 4], 1),            # switch bridge: retain_last(1)
    ("bf16", 2, 128, 60, 1, 5, 2, True, [], None),             # reference only, empty window
    ("bf16", 1, 128, 300, 0, 2, 1, False, [], None),           # nothing cached: chunk only
    ("bf16", 2, 128, 45, 2, 4, 2, True, [3, 3], 2),            # two reference frames
    ("bf16", 2, 64, 50, 1, 4, 3, True, [2, 3], None),          # head_dim 64
    ("bf16", 4, 128, 520, 1, 4, 3, True, [2, 2, 2], None),     # several query-tile pairs
    ("f32", 2, 64, 16, 1, 4, 1, True, [1] * 6, None),          # fp32 storage
    ("f32", 2, 128, 33, 1, 3, 2, True, [2, 2], None),
]


@pytest.mark.parametrize("case", STREAM_CASES, ids=lambda c: "-".join(str(x) for x in c[:8]))
def test_stream_attention_parity(case):
    dtype, H, d, k, R, W, C, ref_on, appends, retain = case
    c, o, rng = build_stream(dtype, H, d, k, R, W, ref_on, appends, retain, seed=len(appends) * 31 + k)
    try:
        q, kc, vc, out = run_stream_attention(c, dtype, H, d, k, C, rng)
        want = o.stream_attention(q, kc, vc, C)
        assert_close(host_f64(out), want, str(case))
    finally:
        rtr().rtr_kvcache_destroy(c)
    assert rtr().rtr_get_device_status(0) == rtr().RTR_OK


PREFILL_CASES = [
    # dtype, H, d, n, k
    ("bf16", 2, 128, 700, 100),
    ("bf16", 2, 128, 600, 1),      # token-causal: every key tile on the diagonal is partial
    ("bf16", 2, 128, 513, 600),    # k >= n: full bidirectional attention
    ("bf16", 3, 128, 300, 37),
    ("bf16", 1, 128, 1, 5),        # single token
    ("bf16", 2, 128, 257, 256),
    ("bf16", 2, 64, 400, 50),
    ("f32", 2, 64, 96, 16),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_prefill_parity(case):
    dtype, H, d, n, k = case
    q, kk, v = synth.random_qkv(n + k, n, H, d, dtype)
    out = torch.empty((n, H, d), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    rtr().rtr_attn_block_causal_prefill(dev(q), dev(kk), dev(v), n, H, d, k, dtype, out)
    torch.cuda.synchronize()
    want = oracle.prefill(*(oracle.decode(x, dtype) for x in (q, kk, v)), k)
    assert_close(host_f64(out), want, str(case))


def test_prefill_empty_is_noop():
    rtr().rtr_attn_block_causal_prefill(None, None, None, 0, 2, 128, 4, "bf16", None)


def _growing_score_qkv(n, H, d, jumps, step_log2, seed):
    """Q, K, V (bf16 bits, [n, H, d]) whose scaled scores rise by about
    ``step_log2`` (log2 units) at every key position in ``jumps``:
    Q ~ 1 + 0.05 N(0,1), K_j ~ a_j + 0.05 N(0,1) with a_j stepping up by
    step_log2 / (log2(e) sqrt(d)) at each jump, V ~ N(0,1)."""
    rng = np.random.default_rng(seed)
    da = step_log2 / (np.log2(np.e) * np.sqrt(d))
    a = da * np.searchsorted(np.sort(np.asarray(jumps)), np.arange(n), side="right")
    q = 1.0 + 0.05 * rng.standard_normal((n, H, d))
    k = a[:, None, None] + 0.05 * rng.standard_normal((n, H, d))
    v = rng.standard_normal((n, H, d))
    return tuple(synth.f32_to_bf16_bits(x.astype(np.float32)) for x in (q, k, v))


GROWTH_CASES = [
    # d, n, k_per_frame, key positions where every row's score jumps
    (128, 700, 1000, [5, 128, 296, 454, 639, 690]),   # all keys visible; a jump in each 32-column chunk
    (128, 700, 150, [5, 128, 296, 454, 639, 690]),    # frame-causal: rows see different prefixes
    (64, 520, 520, [0, 160, 200, 383, 500]),          # head_dim 64, jump at a tile's first and last column
]


@pytest.mark.parametrize("case", GROWTH_CASES, ids=lambda c: f"d{c[0]}-n{c[1]}-k{c[2]}")
def test_prefill_parity_scores_growing_along_keys(case):
    """Row maxima that grow by about 10 (log2 units) part-way through key
    tiles, at each of the four 32-column positions and in the ragged last tile:
    the kernel's running max, the rescale of O, of the row sum and of the P
    already formed for the tile stay exact, so outputs and the row log-sum-exp
    match the oracle.  (With N(0,1) inputs the max rarely grows this much after
    the first tile.)"""
    d, n, kpf, jumps = case
    H = 2
    q, k, v = _growing_score_qkv(n, H, d, jumps, 10.0, seed=n + d + kpf)
    out = torch.empty((n, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, n), dtype=torch.float32, device="cuda")
    rtr().rtr_attn_block_causal_prefill_lse(dev(q), dev(k), dev(v), n, H, d, kpf, "bf16", out, lse)
    torch.cuda.synchronize()
    Q, K, V = (oracle.decode(x, "bf16") for x in (q, k, v))
    assert_close(host_f64(out), oracle.prefill(Q, K, V, kpf), str(case))
    want_lse = oracle.prefill_lse(Q, K, kpf)
    assert np.max(np.abs(lse.cpu().numpy().T.astype(np.float64) - want_lse)) <= 2e-3 * max(1.0, np.max(np.abs(want_lse)))
    assert rtr().rtr_get_device_status(0) == rtr().RTR_OK


@pytest.mark.parametrize("T,nq,H", [(512, 300, 4), (77, 129, 2), (1, 5, 1)])
def test_cross_attention_parity(T, nq, H):
    lib = rtr()
    d = 128
    rng = np.random.default_rng(T + nq)
    x = lib.rtr_crossattn_create(1, H, d, 512, "bf16", 0)
    ox = oracle.CrossCache(H, d, 512, "bf16")
    try:
        kt = synth.normal(rng, (T, H, d), 1.0, "bf16")
        vt = synth.normal(rng, (T, H, d), 1.0, "bf16")
        lib.rtr_crossattn_set_text(x, 0, dev(kt), dev(vt), T)
        ox.set_text(kt, vt, T)
        q = synth.normal(rng, (nq, H, d), 1.0, "bf16")
        out = torch.empty((nq, H, d), dtype=torch.bfloat16, device="cuda")
        lib.rtr_attn_cross(x, 0, dev(q), nq, out)
        torch.cuda.synchronize()
        assert_close(host_f64(out), ox.attention(q), f"cross T={T}")
    finally:
        lib.rtr_crossattn_destroy(x)


def test_tiny_fp32_stream_all_frames():
    """The tiny fp32 workload end to end: reference, then 10 frames each
    attended and appended one at a time through a 4-frame window."""
    w = synth.TINY_F32
    lib = rtr()
    rng = np.random.default_rng(w.seed)
    c = lib.rtr_kvcache_create(1, w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, "f32", 0)
    o = oracle.ReferenceCache(w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, "f32")
    try:
        kr = synth.normal(rng, (w.k, w.heads, w.head_dim), w.scale, "f32")
        vr = synth.normal(rng, (w.k, w.heads, w.head_dim), w.scale, "f32")
        lib.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        for f in range(w.frames_total):
            q, kc, vc, out = run_stream_attention(c, "f32", w.heads, w.head_dim, w.k, 1, rng, w.scale)
            want = o.stream_attention(q, kc, vc, 1)
            got = host_f64(out)
            assert_close(got, want, f"frame {f}")
            assert np.max(np.abs(got - want)) < 1e-4      # fp32 arithmetic
            lib.rtr_kvcache_append_frame(c, 0, dev(kc), dev(vc), 1)
            o.append(kc, vc, 1)
    finally:
        lib.rtr_kvcache_destroy(c)


def test_no_future_frame_bitwise_gpu():
    """Changing the chunk's later frames leaves earlier frames' outputs bit-
    identical on the GPU: masked keys contribute exactly nothing."""
    lib = rtr()
    H, d, k, C = 2, 128, 150, 3
    c, o, rng = build_stream("bf16", H, d, k, 1, 3, True, [1, 1], seed=4)
    try:
        shape = (C * k, H, d)
        q = synth.normal(rng, shape, 1.0, "bf16")
        kc = synth.normal(rng, shape, 1.0, "bf16")
        vc = synth.normal(rng, shape, 1.0, "bf16")
        out0 = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        lib.rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), C, out0)
        for f in (1, 2):
            k2, v2 = kc.copy(), vc.copy()
            k2[f * k:] ^= np.uint16(0x0100)
            v2[f * k:] ^= np.uint16(0x0100)
            out1 = torch.empty_like(out0)
            lib.rtr_attn_frame_causal(c, 0, dev(q), dev(k2), dev(v2), C, out1)
            torch.cuda.synchronize()
            a, b = host_bits(out0), host_bits(out1)
            assert np.array_equal(a[: f * k], b[: f * k])
            assert not np.array_equal(a[f * k:], b[f * k:])
    finally:
        lib.rtr_kvcache_destroy(c)


# ---------------------------------------------------------------- full size
def _sample_rows(n, k, extra, seed):
    rows = {0, 1, 127, 128, 255, 256, n - 1, n - 2}
    for f in range(0, n, k):
        rows.update({f, f + 1, f - 1})
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, n, extra).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)


def test_full_wan13_layer_sampled():
    """One Wan-1.3B-shaped layer: chunk of 3 frames (4680 queries, 12 heads,
    d = 128) against 1 reference + 21 window frames -- the launch the
    benchmark times -- on sampled rows."""
    w = synth.WAN13_LAYER
    lib = rtr()
    x = synth.stream_layer_inputs(w)
    c = lib.rtr_kvcache_create(1, w.heads, w.head_dim, w.k, 1, w.window_frames, "bf16", 0)
    o = oracle.ReferenceCache(w.heads, w.head_dim, w.k, 1, w.window_frames, "bf16")
    try:
        lib.rtr_kvcache_set_reference(c, 0, dev(x.ref_k), dev(x.ref_v))
        o.set_reference(x.ref_k, x.ref_v)
        for fk, fv in zip(x.window_k, x.window_v):
            lib.rtr_kvcache_append_frame(c, 0, dev(fk), dev(fv), 1)
            o.append(fk, fv, 1)
        shape = x.q.shape
        out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        lib.rtr_attn_frame_causal(c, 0, dev(x.q), dev(x.k_cur), dev(x.v_cur), w.chunk_frames, out)
        torch.cuda.synchronize()
        rows = _sample_rows(shape[0], w.k, 40, 1)
        want = o.stream_attention(x.q, x.k_cur, x.v_cur, w.chunk_frames, rows=rows)
        got = host_f64(out)[rows]
        assert_close(got, want, "wan13 layer")
    finally:
        lib.rtr_kvcache_destroy(c)
    assert lib.rtr_get_device_status(0) == lib.RTR_OK


def test_full_prefill_sampled():
    """Block-causal prefill of 22 frames x 1560 tokens (34,320), 12 heads."""
    w = synth.PREFILL_22
    q, k, v = synth.prefill_inputs(w)
    n = q.shape[0]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    rtr().rtr_attn_block_causal_prefill(dev(q), dev(k), dev(v), n, w.heads, w.head_dim, w.k, "bf16", out)
    torch.cuda.synchronize()
    rows = _sample_rows(n, w.k, 24, 2)
    want = oracle.prefill(oracle.decode(q, "bf16"), oracle.decode(k, "bf16"), oracle.decode(v, "bf16"),
                          w.k, rows=rows)
    assert_close(host_f64(out)[rows], want, "prefill 34320")


def test_full_14b_frame_and_cross_sampled():
    """40 heads, one frame against 1 reference + 21 window frames, then the
    same queries against 512 text tokens."""
    w = synth.SWITCH_14B
    lib = rtr()
    rng = np.random.default_rng(w.seed)
    H, d, k = w.heads, w.head_dim, w.k
    c = lib.rtr_kvcache_create(1, H, d, k, 1, w.window_frames, "bf16", 0)
    x = lib.rtr_crossattn_create(1, H, d, w.text_tokens, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, w.window_frames, "bf16")
    ox = oracle.CrossCache(H, d, w.text_tokens, "bf16")
    try:
        kt = synth.normal(rng, (w.text_tokens, H, d), w.scale, "bf16")
        vt = synth.normal(rng, (w.text_tokens, H, d), w.scale, "bf16")
        lib.rtr_crossattn_set_text(x, 0, dev(kt), dev(vt), w.text_tokens)
        ox.set_text(kt, vt, w.text_tokens)
        kr = synth.normal(rng, (k, H, d), w.scale, "bf16")
        vr = synth.normal(rng, (k, H, d), w.scale, "bf16")
        lib.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        for _ in range(w.window_frames):
            fk = synth.normal(rng, (k, H, d), w.scale, "bf16")
            fv = synth.normal(rng, (k, H, d), w.scale, "bf16")
            lib.rtr_kvcache_append_frame(c, 0, dev(fk), dev(fv), 1)
            o.append(fk, fv, 1)
        q = synth.normal(rng, (k, H, d), w.scale, "bf16")
        kc = synth.normal(rng, (k, H, d), w.scale, "bf16")
        vc = synth.normal(rng, (k, H, d), w.scale, "bf16")
        out = torch.empty((k, H, d), dtype=torch.bfloat16, device="cuda")
        lib.rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), 1, out)
        xout = torch.empty_like(out)
        lib.rtr_attn_cross(x, 0, dev(q), k, xout)
        torch.cuda.synchronize()
        rows = _sample_rows(k, k, 12, 4)
        assert_close(host_f64(out)[rows], o.stream_attention(q, kc, vc, 1, rows=rows), "14B self")
        assert_close(host_f64(xout)[rows], ox.attention(q, rows=rows), "14B cross")
    finally:
        lib.rtr_kvcache_destroy(c)
        lib.rtr_crossattn_destroy(x)
