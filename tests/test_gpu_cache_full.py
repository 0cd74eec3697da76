"""GPU: KV-cache bytes at the full sizes of the long-stream and the 14B-like
switching workloads, bit for bit against the oracle's state machine
(papernotes.org note "DiT as Real-Time Rerenderer", Method > Key Designs 4:
the anchored reference survives eviction; a switch keeps the most recent
frame and anchors the new reference in place).

Frame data: one seeded bf16 draw per tensor (the workloads' recipe, N(0,1)
* 0.5), and frame f of layer l is that draw with the low 7 mantissa bits of
every element XOR-ed with a pattern unique to (l, f).  The caches copy bits,
so any pattern is as good as a fresh draw for a copy test, and every frame
differs from every other in every element: a frame written to the wrong
slot, layer or head cannot match.  The same XOR is applied on the device
(the library's input) and in numpy (the oracle's input).
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import dev
from test_gpu_cache import compare_cache

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _pattern(layer, frame):
    return np.uint16(((layer * 131 + frame * 7 + 1) % 127) + 1)   # 1..127: low mantissa bits only


def _variant_host(base, pat):
    return base ^ pat


def _variant_dev(base_dev, pat):
    return torch.bitwise_xor(base_dev, int(pat) if int(pat) < 32768 else int(pat) - 65536)


def test_long_stream_cache_all_layers_bit_exact():
    """30 layers x 12 heads x k = 1560, reference + W = 21: every layer gets
    its reference and 8 chunks of 3 frames (the window wraps after 7), then
    layers 0, 1, 14, 28 and 29 are compared byte for byte (layer 29 starts
    6.1 GB into the buffer: its offset is far above 2^31 bytes) and every
    layer's index map is checked; the guard bands are intact."""
    rtr = _rtr()
    w = synth.LONG_STREAM
    L, H, d, k, R, W, C = w.layers, w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames, w.chunk_frames
    chunks = 8
    rng = np.random.default_rng(w.seed)
    ref_k, ref_v = (synth.normal(rng, (R * k, H, d), w.scale, "bf16") for _ in range(2))
    ck, cv = (synth.normal(rng, (C * k, H, d), w.scale, "bf16") for _ in range(2))
    d_ref_k, d_ref_v, d_ck, d_cv = (dev(a).view(torch.int16) for a in (ref_k, ref_v, ck, cv))
    compared = (0, 1, 14, 28, 29)
    refs = {l: oracle.ReferenceCache(H, d, k, R, W, "bf16") for l in compared}
    c = rtr.rtr_kvcache_create(L, H, d, k, R, W, "bf16", 0)
    try:
        for l in range(L):
            pat = _pattern(l, 10_000)
            rk, rv = _variant_dev(d_ref_k, pat), _variant_dev(d_ref_v, pat)
            rtr.rtr_kvcache_set_reference(c, l, rk, rv)
            if l in refs:
                refs[l].set_reference(_variant_host(ref_k, pat), _variant_host(ref_v, pat))
        torch.cuda.synchronize()
        for ch in range(chunks):
            for l in range(L):
                pat = _pattern(l, ch)
                kn, vn = _variant_dev(d_ck, pat), _variant_dev(d_cv, pat)
                rtr.rtr_kvcache_append_frame(c, l, kn, vn, C)
                if l in refs:
                    refs[l].append(_variant_host(ck, pat), _variant_host(cv, pat), C)
            torch.cuda.synchronize()
        assert refs[0].g == chunks * C > W                      # the window has wrapped
        for l in range(L):
            slots, ref_valid, g, count = rtr.rtr_kvcache_get_index_map(c, l, W)
            assert (ref_valid, g, count) == (1, chunks * C, W)
        for l in compared:
            compare_cache(c, refs[l], layer=l)
        assert rtr.rtr_kvcache_check_guards(c) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK


def test_switching_cache_40_heads_bit_exact():
    """40 heads x k = 1560, reference + W = 21, frames one at a time: 16
    frames, a switch (retain_last(1), a new reference written in place over
    the old one), compared right after the switch, then 25 more frames (the
    window wraps) and a second switch, compared after each."""
    rtr = _rtr()
    w = synth.SWITCH_14B
    H, d, k, R, W = w.heads, w.head_dim, w.k, w.ref_frames, w.window_frames
    rng = np.random.default_rng(w.seed)
    ref_k, ref_v = (synth.normal(rng, (R * k, H, d), w.scale, "bf16") for _ in range(2))
    fk, fv = (synth.normal(rng, (k, H, d), w.scale, "bf16") for _ in range(2))
    d_ref_k, d_ref_v, d_fk, d_fv = (dev(a).view(torch.int16) for a in (ref_k, ref_v, fk, fv))
    o = oracle.ReferenceCache(H, d, k, R, W, "bf16")
    c = rtr.rtr_kvcache_create(1, H, d, k, R, W, "bf16", 0)

    def set_reference(epoch):
        pat = _pattern(epoch, 20_000)
        rtr.rtr_kvcache_set_reference(c, 0, _variant_dev(d_ref_k, pat), _variant_dev(d_ref_v, pat))
        o.set_reference(_variant_host(ref_k, pat), _variant_host(ref_v, pat))

    try:
        set_reference(0)
        frame = 0
        for epoch, n_frames in ((1, 16), (2, 25)):
            for _ in range(n_frames):
                pat = _pattern(0, frame)
                rtr.rtr_kvcache_append_frame(c, 0, _variant_dev(d_fk, pat), _variant_dev(d_fv, pat), 1)
                o.append(_variant_host(fk, pat), _variant_host(fv, pat), 1)
                frame += 1
            torch.cuda.synchronize()
            compare_cache(c, o)
            # the switch: keep the most recent frame, anchor the new reference in place
            rtr.rtr_kvcache_retain_last(c, 0, 1)
            o.retain_last(1)
            set_reference(epoch)
            torch.cuda.synchronize()
            compare_cache(c, o)
            assert rtr.rtr_kvcache_get_index_map(c, 0, W)[3] == 1
        assert o.g == 41 > W
        assert rtr.rtr_kvcache_check_guards(c) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
