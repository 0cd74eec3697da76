"""GPU: the bf16 frame-causal attention with an fp32 output
(rtr_attn_frame_causal_f32out), the run that shows the bf16 path's error
without the final rounding of the output.

For every case the fp32 output, rounded to bf16 (nearest even), equals the
bf16 call's output bit for bit: both come from the same normalised rows, the
bf16 call only rounds them.  Against the fp64 oracle the fp32 output is
within the attention tolerance and its relative L2 error is below the bf16
output's (the bf16 rounding of the output is one of the error's parts).
Cases cover whole units, units split across CTAs (merged by the combine
kernel, which writes fp32 too), ragged tails and head_dim 64, and the
Wan-1.3B layer on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, errors, host_f64

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _build(H, d, k, W, appends, seed):
    lib = _rtr()
    rng = np.random.default_rng(seed)
    c = lib.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    kr, vr = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
    lib.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
    o.set_reference(kr, vr)
    for n in appends:
        kn, vn = (synth.normal(rng, (n * k, H, d), 1.0, "bf16") for _ in range(2))
        lib.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), n)
        o.append(kn, vn, n)
    return c, o, rng


CASES = [
    # H, d, k, W, C, appends
    (2, 128, 200, 3, 2, [2, 1]),        # 4 units on 148 CTAs: split units, merged in fp32
    (12, 128, 300, 4, 3, [3, 1]),       # whole units in full rounds
    (3, 128, 77, 4, 3, [2, 2]),         # ragged frame and tile tails
    (2, 64, 150, 3, 2, [1, 2]),         # head_dim 64
]


@pytest.mark.parametrize("H,d,k,W,C,appends", CASES, ids=lambda c: str(c))
def test_f32_output_is_the_unrounded_bf16_output(H, d, k, W, C, appends):
    lib = _rtr()
    c, o, rng = _build(H, d, k, W, appends, seed=H * 1000 + k)
    try:
        shape = (C * k, H, d)
        q, kc, vc = (synth.normal(rng, shape, 1.0, "bf16") for _ in range(3))
        Q, K, V = dev(q), dev(kc), dev(vc)
        out16 = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        out32 = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        lib.rtr_attn_frame_causal(c, 0, Q, K, V, C, out16)
        lib.rtr_attn_frame_causal_f32out(c, 0, Q, K, V, C, out32)
        torch.cuda.synchronize()
        assert lib.rtr_get_device_status(0) == lib.RTR_OK
        assert not torch.isnan(out32).any()
        assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
        want = o.stream_attention(q, kc, vc, C)
        got32, got16 = host_f64(out32), host_f64(out16)
        assert_close(got32, want, "fp32 output")
        e32, e16 = errors(got32, want), errors(got16, want)
        assert e32[1] < e16[1], f"rel-L2 fp32 {e32[1]:.3e} vs bf16 {e16[1]:.3e}"
    finally:
        lib.rtr_kvcache_destroy(c)


def test_f32_output_wan13_layer_sampled():
    """The benchmark's layer (4680 queries, 12 heads, 1 reference + 21 window
    frames) on sampled rows: the fp32 output's error against the bf16
    output's."""
    lib = _rtr()
    w = synth.WAN13_LAYER
    x = synth.stream_layer_inputs(w)
    c = lib.rtr_kvcache_create(1, w.heads, w.head_dim, w.k, 1, w.window_frames, "bf16", 0)
    o = oracle.ReferenceCache(w.heads, w.head_dim, w.k, 1, w.window_frames, "bf16")
    try:
        lib.rtr_kvcache_set_reference(c, 0, dev(x.ref_k), dev(x.ref_v))
        o.set_reference(x.ref_k, x.ref_v)
        for fk, fv in zip(x.window_k, x.window_v):
            lib.rtr_kvcache_append_frame(c, 0, dev(fk), dev(fv), 1)
            o.append(fk, fv, 1)
        Q, K, V = dev(x.q), dev(x.k_cur), dev(x.v_cur)
        out16 = torch.empty(x.q.shape, dtype=torch.bfloat16, device="cuda")
        out32 = torch.empty(x.q.shape, dtype=torch.float32, device="cuda")
        lib.rtr_attn_frame_causal(c, 0, Q, K, V, w.chunk_frames, out16)
        lib.rtr_attn_frame_causal_f32out(c, 0, Q, K, V, w.chunk_frames, out32)
        torch.cuda.synchronize()
        assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
        rows = np.array(sorted(set(np.random.default_rng(7).integers(0, x.q.shape[0], 40).tolist())
                               | {0, w.k - 1, w.k, x.q.shape[0] - 1}))
        want = o.stream_attention(x.q, x.k_cur, x.v_cur, w.chunk_frames, rows=rows)
        e32 = errors(host_f64(out32)[rows], want)
        e16 = errors(host_f64(out16)[rows], want)
        print(f"wan13 sampled rows: fp32 out max_abs={e32[0]:.3e} rel_l2={e32[1]:.3e}; "
              f"bf16 out max_abs={e16[0]:.3e} rel_l2={e16[1]:.3e}")
        assert_close(host_f64(out32)[rows], want, "fp32 output")
        assert e32[1] < e16[1]
    finally:
        lib.rtr_kvcache_destroy(c)
    assert lib.rtr_get_device_status(0) == lib.RTR_OK


def test_f32_output_rejects_misaligned_output():
    lib = _rtr()
    c = lib.rtr_kvcache_create(1, 2, 128, 16, 1, 2, "bf16", 0)
    try:
        x = torch.zeros((16, 2, 128), dtype=torch.bfloat16, device="cuda")
        o = torch.zeros((16 * 2 * 128 + 4,), dtype=torch.float32, device="cuda")
        st = lib.raw_status("rtr_attn_frame_causal_f32out", c, 0, x.data_ptr(), x.data_ptr(), x.data_ptr(), 1,
                            o.data_ptr() + 4, 0.0, None)
        assert st == lib.RTR_E_INVAL
    finally:
        lib.rtr_kvcache_destroy(c)
