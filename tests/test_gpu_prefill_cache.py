"""GPU parity of the prefill that also fills the cache
(rtr_attn_block_causal_prefill_cache): a sequence attended under the
block-causal mask whose K/V become the reference slot and the window the
stream continues from (papernotes.org note "DiT as Real-Time Rerenderer",
Method > Key Designs 2 and 4).  Outputs are compared with the oracle's prefill
and, bit for bit, with rtr_attn_block_causal_prefill; the cache with the
oracle's state machine after set_reference + append; then one streamed chunk
attends to the filled cache."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_bits, host_f64
from test_gpu_cache import compare_cache

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _empty(shape, dtype):
    return torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")


CASES = [
    # dtype, H, d, k, R, W, commit room, with_reference, n_frames, appends before
    ("bf16", 2, 128, 200, 1, 4, 0, True, 5, []),          # fresh cache, TMA writes, window filled
    ("bf16", 2, 128, 77, 1, 4, 0, True, 3, []),           # k not a multiple of 8: warp-copy writes
    ("bf16", 2, 128, 120, 1, 4, 2, False, 3, [1, 2]),     # no reference part, ring position 3 of 6
    ("bf16", 2, 128, 200, 1, 4, 0, False, 4, [1] * 5),    # no reference part, wraps the ring, evicts
    ("bf16", 2, 128, 96, 1, 3, 0, True, 3, [2]),          # reference part with g = 2 not a multiple of S
    ("bf16", 2, 128, 96, 1, 3, 0, True, 4, [3]),          # reference part with g = S: one launch
    ("bf16", 2, 64, 64, 2, 3, 0, True, 5, []),            # two reference frames, head_dim 64
    ("bf16", 1, 128, 600, 1, 2, 0, True, 3, []),          # frames longer than a tile, several query pairs
    ("bf16", 2, 128, 40, 1, 4, 0, True, 1, []),           # the reference alone
    ("f32", 2, 64, 16, 1, 4, 0, True, 5, []),             # fp32 storage: attention, then the copy kernels
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c[:9]))
def test_prefill_cache_parity(case):
    dtype, H, d, k, R, W, room, with_ref, F, before = case
    rtr = _rtr()
    rng = np.random.default_rng(k * 10 + F + len(before))
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, R, W, room, dtype, 0)
    o = oracle.ReferenceCache(H, d, k, R, W, dtype, slots=W + room)
    try:
        if R > 0 and not with_ref:
            kr, vr = (synth.normal(rng, (R * k, H, d), 0.5, dtype) for _ in range(2))
            rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
            o.set_reference(kr, vr)
        for n in before:
            kn, vn = (synth.normal(rng, (n * k, H, d), 0.5, dtype) for _ in range(2))
            rtr.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), n)
            o.append(kn, vn, n)
        n_tok = F * k
        q, kk, vv = (synth.normal(rng, (n_tok, H, d), 0.5, dtype) for _ in range(3))
        out = _empty((n_tok, H, d), dtype)
        rtr.rtr_attn_block_causal_prefill_cache(c, 0, dev(q), dev(kk), dev(vv), F, with_ref, out)
        plain = _empty((n_tok, H, d), dtype)
        rtr.rtr_attn_block_causal_prefill(dev(q), dev(kk), dev(vv), n_tok, H, d, k, dtype, plain)
        torch.cuda.synchronize()
        Q, K, V = (oracle.decode(x, dtype) for x in (q, kk, vv))
        assert_close(host_f64(out), oracle.prefill(Q, K, V, k), str(case))
        assert np.array_equal(host_bits(out), host_bits(plain)), "differs from the plain prefill"
        nref = R if with_ref else 0
        if nref:
            o.set_reference(kk[: nref * k], vv[: nref * k])
        if F > nref:
            o.append(kk[nref * k:], vv[nref * k:], F - nref)
        compare_cache(c, o)
        # the stream continues from the filled cache
        q2, k2, v2 = (synth.normal(rng, (k, H, d), 0.5, dtype) for _ in range(3))
        out2 = _empty((k, H, d), dtype)
        rtr.rtr_attn_frame_causal(c, 0, dev(q2), dev(k2), dev(v2), 1, out2)
        torch.cuda.synchronize()
        assert_close(host_f64(out2), o.stream_attention(q2, k2, v2, 1), "chunk after the prefill")
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)


def test_prefill_cache_rejects_bad_arguments():
    """Invalid calls return their status and leave the cache as it was."""
    rtr = _rtr()
    H, d, k, W = 1, 128, 16, 3
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    c0 = rtr.rtr_kvcache_create(1, H, d, k, 0, W, "bf16", 0)
    try:
        x = torch.zeros((5 * k, H, d), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(x)
        cases = [
            (c, 5, True, rtr.RTR_E_INVAL),     # 4 window frames > W = 3
            (c, 4, False, rtr.RTR_E_INVAL),    # 4 window frames > W = 3
            (c0, 2, True, rtr.RTR_E_STATE),    # no reference slot
            (c, 0, True, rtr.RTR_E_INVAL),     # no frames
        ]
        for cache, F, with_ref, want in cases:
            with pytest.raises(rtr.RtrError) as e:
                rtr.rtr_attn_block_causal_prefill_cache(cache, 0, x, x, x, F, with_ref, out)
            assert e.value.status == want, (F, with_ref)
        st = rtr._lib.rtr_attn_block_causal_prefill_cache(c, 0, x.data_ptr(), x.data_ptr(), x.data_ptr(), 2, 2,
                                                           out.data_ptr(), 0.0, None)
        assert st == rtr.RTR_E_INVAL                                       # with_reference not 0 / 1
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_attn_block_causal_prefill_cache(c, 1, x, x, x, 2, True, out)
        assert e.value.status == rtr.RTR_E_INVAL                           # no such layer
        assert rtr.rtr_kvcache_get_index_map(c, 0, W) == ([-1] * W, 0, 0, 0)
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_kvcache_destroy(c0)


def test_full_prefill_22_into_wan13_cache_sampled():
    """The 22-frame prefill (1 reference + 21 frames, 12 heads, k = 1560) into a
    Wan-1.3B-shaped cache in one launch: sampled rows against the oracle, the
    whole cache bit-exact, then the layer's 3-frame chunk attends to it."""
    rtr = _rtr()
    w = synth.WAN13_LAYER
    H, d, k, W, C = w.heads, w.head_dim, w.k, w.window_frames, w.chunk_frames
    F = 1 + W
    rng = np.random.default_rng(22)
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    try:
        q, kk, vv = (synth.normal(rng, (F * k, H, d), w.scale, "bf16") for _ in range(3))
        out = torch.empty((F * k, H, d), dtype=torch.bfloat16, device="cuda")
        rtr.rtr_attn_block_causal_prefill_cache(c, 0, dev(q), dev(kk), dev(vv), F, True, out)
        torch.cuda.synchronize()
        rows = np.array(sorted({0, 1559, 1560, 17000, F * k - 1}
                               | set(np.random.default_rng(5).integers(0, F * k, 20).tolist())))
        Q, K, V = (oracle.decode(x, "bf16") for x in (q, kk, vv))
        assert_close(host_f64(out)[rows], oracle.prefill(Q, K, V, k, rows=rows), "prefill rows")
        o.set_reference(kk[:k], vv[:k])
        o.append(kk[k:], vv[k:], W)
        compare_cache(c, o)
        q2, k2, v2 = (synth.normal(rng, (C * k, H, d), w.scale, "bf16") for _ in range(3))
        out2 = torch.empty((C * k, H, d), dtype=torch.bfloat16, device="cuda")
        rtr.rtr_attn_frame_causal(c, 0, dev(q2), dev(k2), dev(v2), C, out2)
        torch.cuda.synchronize()
        rows2 = np.array([0, 127, 1560, 3119, 4679])
        assert_close(host_f64(out2)[rows2], o.stream_attention(q2, k2, v2, C, rows=rows2), "chunk rows")
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)
