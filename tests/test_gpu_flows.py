"""GPU parity of whole streaming flows against the oracle's state machines
(papernotes.org note "DiT as Real-Time Rerenderer", Method > Key Designs 2 and
4): frames attended and committed one chunk at a time through eviction, with
several layers and two denoising steps per chunk, and a live style switch
(cross-attention cache reset and refilled, 3D cache cut to its most recent
frame, reference overwritten in place) in the middle of a stream."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def test_switching_stream_flow():
    """Frames one at a time with self- and cross-attention; a switch at
    frame 6 and another at frame 11."""
    rtr = _rtr()
    H, d, k, W, T = 4, 128, 200, 4, 64
    rng = np.random.default_rng(55)
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    x = rtr.rtr_crossattn_create(1, H, d, T, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    ox = oracle.CrossCache(H, d, T, "bf16")
    try:
        def new_condition(n_text):
            kt, vt = (synth.normal(rng, (n_text, H, d), 0.5, "bf16") for _ in range(2))
            kr, vr = (synth.normal(rng, (k, H, d), 0.5, "bf16") for _ in range(2))
            return kt, vt, kr, vr

        kt, vt, kr, vr = new_condition(T)
        rtr.rtr_crossattn_set_text(x, 0, dev(kt), dev(vt), T)
        ox.set_text(kt, vt, T)
        rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        for f in range(14):
            if f in (6, 11):
                n_text = T if f == 6 else 37          # a shorter prompt on the second switch
                kt, vt, kr, vr = new_condition(n_text)
                rtr.rtr_crossattn_reset(x)
                ox.reset()
                rtr.rtr_crossattn_set_text(x, 0, dev(kt), dev(vt), n_text)
                ox.set_text(kt, vt, n_text)
                rtr.rtr_kvcache_retain_last(c, 0, 1)
                o.retain_last(1)
                rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
                o.set_reference(kr, vr)
            q, kc, vc = (synth.normal(rng, (k, H, d), 0.5, "bf16") for _ in range(3))
            out = torch.empty((k, H, d), dtype=torch.bfloat16, device="cuda")
            xout = torch.empty_like(out)
            rtr.rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), 1, out)
            rtr.rtr_attn_cross(x, 0, dev(q), k, xout)
            rtr.rtr_kvcache_append_frame(c, 0, dev(kc), dev(vc), 1)
            torch.cuda.synchronize()
            assert_close(host_f64(out), o.stream_attention(q, kc, vc, 1), f"self frame {f}")
            assert_close(host_f64(xout), ox.attention(q), f"cross frame {f}")
            o.append(kc, vc, 1)
            assert rtr.rtr_kvcache_get_index_map(c, 0, W) == (*o.index_map(), o.count)
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK


def test_multilayer_chunked_stream_flow():
    """3 layers, chunks of 2 frames, 2 denoising steps per chunk (attend twice,
    commit the last step's K/V), 8 chunks through a 5-frame window."""
    rtr = _rtr()
    L, H, d, k, W, C = 3, 2, 128, 160, 5, 2
    rng = np.random.default_rng(66)
    c = rtr.rtr_kvcache_create(L, H, d, k, 1, W, "bf16", 0)
    os_ = [oracle.ReferenceCache(H, d, k, 1, W, "bf16") for _ in range(L)]
    try:
        for l in range(L):
            kr, vr = (synth.normal(rng, (k, H, d), 0.5, "bf16") for _ in range(2))
            rtr.rtr_kvcache_set_reference(c, l, dev(kr), dev(vr))
            os_[l].set_reference(kr, vr)
        for ch in range(8):
            for l in range(L):
                for step in range(2):
                    q, kc, vc = (synth.normal(rng, (C * k, H, d), 0.5, "bf16") for _ in range(3))
                    out = torch.empty((C * k, H, d), dtype=torch.bfloat16, device="cuda")
                    rtr.rtr_attn_frame_causal(c, l, dev(q), dev(kc), dev(vc), C, out)
                    torch.cuda.synchronize()
                    if step == 1 or ch in (0, 7):
                        assert_close(host_f64(out), os_[l].stream_attention(q, kc, vc, C),
                                     f"chunk {ch} layer {l} step {step}")
                rtr.rtr_kvcache_append_frame(c, l, dev(kc), dev(vc), C)
                os_[l].append(kc, vc, C)
        for l in range(L):
            assert rtr.rtr_kvcache_get_index_map(c, l, W) == (*os_[l].index_map(), os_[l].count)
    finally:
        rtr.rtr_kvcache_destroy(c)


def test_full_long_stream_layer_after_eviction_sampled():
    """One layer of the long-stream workload (12 heads, k = 1560, window 21)
    after 10 chunks of 3 frames -- the window has wrapped -- on sampled rows."""
    rtr = _rtr()
    w = synth.LONG_STREAM
    H, d, k, W, C = w.heads, w.head_dim, w.k, w.window_frames, w.chunk_frames
    rng = np.random.default_rng(w.seed)
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    try:
        kr, vr = (synth.normal(rng, (k, H, d), w.scale, "bf16") for _ in range(2))
        rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        for _ in range(10):
            kc, vc = (synth.normal(rng, (C * k, H, d), w.scale, "bf16") for _ in range(2))
            rtr.rtr_kvcache_append_frame(c, 0, dev(kc), dev(vc), C)
            o.append(kc, vc, C)
        q, kc, vc = (synth.normal(rng, (C * k, H, d), w.scale, "bf16") for _ in range(3))
        out = torch.empty((C * k, H, d), dtype=torch.bfloat16, device="cuda")
        rtr.rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), C, out)
        torch.cuda.synchronize()
        rows = np.array(sorted({0, 1, 127, 128, 1559, 1560, 1561, 3119, 3120, 4679}
                               | set(np.random.default_rng(3).integers(0, C * k, 20).tolist())))
        assert_close(host_f64(out)[rows], o.stream_attention(q, kc, vc, C, rows=rows), "long stream")
        assert rtr.rtr_kvcache_get_index_map(c, 0, W) == (*o.index_map(), o.count)
    finally:
        rtr.rtr_kvcache_destroy(c)
