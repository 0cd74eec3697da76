"""GPU parity of the fused chunk commit (rtr_attn_frame_causal_commit): the
chunk's attention and the write of its K/V into the rolling cache in one
launch (papernotes.org note "DiT as Real-Time Rerenderer", Method > Key
Designs 4: a generated chunk enters the fixed-length cache and the oldest
frames leave it).  Outputs are compared with the oracle's stream attention.
The ring contents and the index map are compared bit for bit with the
oracle's state machine, which is given the same number of physical slots."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64
from test_gpu_cache import _raw_view, compare_cache

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _out(shape, dtype):
    return torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")


CASES = [
    # dtype, H, d, k, W, C, chunks, ref
    ("bf16", 2, 128, 200, 4, 2, 7, True),     # frames straddle tiles, ring wraps mid-chunk
    ("bf16", 2, 128, 128, 3, 3, 5, True),     # tile-aligned frames, C == W
    ("bf16", 3, 128, 77, 5, 1, 9, False),     # one frame per chunk, TV2V (no reference)
    ("bf16", 2, 64, 90, 4, 3, 5, True),       # head_dim 64
    ("bf16", 2, 128, 600, 2, 2, 4, True),     # several query-tile pairs per chunk
    ("f32", 2, 64, 16, 4, 2, 5, True),        # fp32 storage: attention, then the scatter kernel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_commit_stream_parity(case):
    """Chunks through eviction, two denoising steps each: step 1 attends only,
    step 2 attends and commits; every output against the oracle, the ring and
    the index map bit-exact after every commit."""
    dtype, H, d, k, W, C, chunks, ref = case
    rtr = _rtr()
    rng = np.random.default_rng(H * 100 + k + C)
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, W, C, dtype, 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, dtype, slots=W + C)
    try:
        if ref:
            kr, vr = (synth.normal(rng, (k, H, d), 0.5, dtype) for _ in range(2))
            rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
            o.set_reference(kr, vr)
        for ch in range(chunks):
            for step in range(2):
                q, kc, vc = (synth.normal(rng, (C * k, H, d), 0.5, dtype) for _ in range(3))
                out = _out((C * k, H, d), dtype)
                if step == 0:
                    rtr.rtr_attn_frame_causal(c, 0, dev(q), dev(kc), dev(vc), C, out)
                else:
                    rtr.rtr_attn_frame_causal_commit(c, 0, dev(q), dev(kc), dev(vc), C, out)
                torch.cuda.synchronize()
                assert_close(host_f64(out), o.stream_attention(q, kc, vc, C), f"chunk {ch} step {step}")
            o.append(kc, vc, C)
            compare_cache(c, o)
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)


def test_commit_after_switch_and_plain_appends():
    """Fused commits mixed with plain appends, a retain_last(1) switch and a
    reference overwrite: the state machine stays in step with the oracle."""
    rtr = _rtr()
    H, d, k, W, C = 2, 128, 150, 5, 2
    rng = np.random.default_rng(5)
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, W, C, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16", slots=W + C)
    try:
        for it in range(10):
            if it in (0, 6):
                kr, vr = (synth.normal(rng, (k, H, d), 0.5, "bf16") for _ in range(2))
                rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
                o.set_reference(kr, vr)
            if it == 6:
                rtr.rtr_kvcache_retain_last(c, 0, 1)
                o.retain_last(1)
            n = 1 if it % 3 == 0 else C
            q, kc, vc = (synth.normal(rng, (n * k, H, d), 0.5, "bf16") for _ in range(3))
            if it % 4 == 3:
                rtr.rtr_kvcache_append_frame(c, 0, dev(kc), dev(vc), n)
            else:
                out = _out((n * k, H, d), "bf16")
                rtr.rtr_attn_frame_causal_commit(c, 0, dev(q), dev(kc), dev(vc), n, out)
                torch.cuda.synchronize()
                assert_close(host_f64(out), o.stream_attention(q, kc, vc, n), f"iteration {it}")
            o.append(kc, vc, n)
            compare_cache(c, o)
    finally:
        rtr.rtr_kvcache_destroy(c)


def test_commit_rejects_chunk_larger_than_commit_room():
    rtr = _rtr()
    H, d, k = 1, 128, 16
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, 4, 1, "bf16", 0)
    plain = rtr.rtr_kvcache_create(1, H, d, k, 1, 4, "bf16", 0)
    try:
        x = torch.zeros((2 * k, H, d), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(x)
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_attn_frame_causal_commit(c, 0, x, x, x, 2, out)
        assert e.value.status == rtr.RTR_E_INVAL
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_attn_frame_causal_commit(plain, 0, x[:k], x[:k], x[:k], 1, out[:k])
        assert e.value.status == rtr.RTR_E_INVAL
        # a rejected call leaves the state untouched
        assert rtr.rtr_kvcache_get_index_map(c, 0, 5) == ([-1] * 5, 0, 0, 0)
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_kvcache_destroy(plain)


def test_full_layer_commit_sampled():
    """The Wan-1.3B-like layer (12 heads, k = 1560, window 21, chunks of 3)
    with commit room 3, after 9 committed chunks (the window has wrapped):
    sampled output rows against the oracle; the ring against the oracle."""
    rtr = _rtr()
    w = synth.WAN13_LAYER
    H, d, k, W, C = w.heads, w.head_dim, w.k, w.window_frames, w.chunk_frames
    rng = np.random.default_rng(w.seed)
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, W, C, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16", slots=W + C)
    try:
        kr, vr = (synth.normal(rng, (k, H, d), w.scale, "bf16") for _ in range(2))
        rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        rows = np.array(sorted({0, 127, 128, 255, 256, 1559, 1560, 3119, 3120, 4679}
                               | set(np.random.default_rng(4).integers(0, C * k, 12).tolist())))
        for ch in range(9):
            q, kc, vc = (synth.normal(rng, (C * k, H, d), w.scale, "bf16") for _ in range(3))
            out = torch.empty((C * k, H, d), dtype=torch.bfloat16, device="cuda")
            rtr.rtr_attn_frame_causal_commit(c, 0, dev(q), dev(kc), dev(vc), C, out)
            torch.cuda.synchronize()
            if ch in (0, 8):
                assert_close(host_f64(out)[rows], o.stream_attention(q, kc, vc, C, rows=rows), f"chunk {ch}")
            o.append(kc, vc, C)
        compare_cache(c, o)
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)


@pytest.mark.parametrize("k", [200, 77])
def test_commit_equals_attention_then_append_bitwise(k):
    """On two caches with the same commit room and history, the fused call
    and attention followed by append give bit-identical outputs, rings and
    index maps (TMA chunk write for k a multiple of 8, warp copy otherwise)."""
    rtr = _rtr()
    H, d, W, C = 2, 128, 4, 3
    rng = np.random.default_rng(k)
    a = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, W, C, "bf16", 0)
    b = rtr.rtr_kvcache_create_ex(1, H, d, k, 1, W, C, "bf16", 0)
    nbytes = H * (1 + W + C) * k * d * 2
    try:
        kr, vr = (synth.normal(rng, (k, H, d), 0.5, "bf16") for _ in range(2))
        for c in (a, b):
            rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        for step in range(6):
            n = 1 + step % C
            q, kc, vc = (synth.normal(rng, (n * k, H, d), 0.5, "bf16") for _ in range(3))
            oa, ob = (torch.empty((n * k, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2))
            rtr.rtr_attn_frame_causal_commit(a, 0, dev(q), dev(kc), dev(vc), n, oa)
            rtr.rtr_attn_frame_causal(b, 0, dev(q), dev(kc), dev(vc), n, ob)
            rtr.rtr_kvcache_append_frame(b, 0, dev(kc), dev(vc), n)
            torch.cuda.synchronize()
            assert torch.equal(oa.view(torch.int16), ob.view(torch.int16)), f"step {step}"
            assert rtr.rtr_kvcache_get_index_map(a, 0, W + C) == rtr.rtr_kvcache_get_index_map(b, 0, W + C)
        slots = rtr.rtr_kvcache_get_index_map(a, 0, W + C)[0]
        for pa, pb in zip(rtr.rtr_kvcache_device_ptrs(a, 0), rtr.rtr_kvcache_device_ptrs(b, 0)):
            ta = _raw_view(pa, nbytes).view(H, 1 + W + C, k * d * 2)
            tb = _raw_view(pb, nbytes).view(H, 1 + W + C, k * d * 2)
            for s_, f in enumerate(slots):
                if f >= 0:
                    assert torch.equal(ta[:, 1 + s_], tb[:, 1 + s_]), f"slot {s_}"
    finally:
        rtr.rtr_kvcache_destroy(a)
        rtr.rtr_kvcache_destroy(b)
