"""GPU: KV-cache and cross-attention-cache contents and index maps are
bit-exact against the oracle's state machine (papernotes.org note "DiT as
Real-Time Rerenderer", Method > Key Designs 4), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import dev, host_bits

pytestmark = pytest.mark.gpu


class _DevArray:
    """__cuda_array_interface__ view of a library-owned device buffer."""

    def __init__(self, ptr, n, typestr):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


def gpu_view(c, layer, H, rows, d, dtype, which):
    """Host copy of layer ``layer``'s K or V cache buffer [H][rows][d]."""
    from causal_attention_rtr_b200 import rtr
    kp, vp = rtr.rtr_kvcache_device_ptrs(c, layer)
    ptr = kp if which == "k" else vp
    n = H * rows * d
    torch.cuda.synchronize()
    t = torch.as_tensor(_DevArray(ptr, n, "<i2" if dtype == "bf16" else "<f4"), device="cuda")
    a = t.cpu().numpy()
    a = a.view(np.uint16) if dtype == "bf16" else a
    return a.reshape(H, rows, d)


def compare_cache(c, ref: oracle.ReferenceCache, layer=0):
    from causal_attention_rtr_b200 import rtr
    rtr.rtr_kvcache_check_guards(c)                   # no kernel wrote outside the buffers
    slots, ref_valid, g, count = rtr.rtr_kvcache_get_index_map(c, layer, ref.S)
    want_slots, want_ref, want_g = ref.index_map()
    assert (slots, ref_valid, g, count) == (want_slots, want_ref, want_g, ref.count)
    rows = (ref.R + ref.S) * ref.k
    for which in ("k", "v"):
        buf = gpu_view(c, layer, ref.H, rows, ref.d, ref.dtype, which)
        if ref.ref_valid:
            want = (ref.ref_k if which == "k" else ref.ref_v).transpose(1, 0, 2)
            assert np.array_equal(buf[:, : ref.R * ref.k], want), "reference slot differs"
        for s, f in enumerate(slots):
            if f >= 0:
                data = (ref.slots_k if which == "k" else ref.slots_v)[s].transpose(1, 0, 2)
                lo = (ref.R + s) * ref.k
                assert np.array_equal(buf[:, lo: lo + ref.k], data), f"slot {s} (frame {f}) differs"


@pytest.mark.parametrize("dtype,H,d,k,R,W", [("bf16", 2, 128, 16, 1, 4), ("bf16", 3, 64, 17, 1, 5),
                                             ("f32", 2, 64, 16, 1, 4), ("bf16", 12, 128, 1560, 1, 3),
                                             ("bf16", 2, 128, 5, 2, 3)])
def test_cache_random_ops_bit_exact(dtype, H, d, k, R, W):
    from causal_attention_rtr_b200 import rtr
    rng = np.random.default_rng(H * 1000 + k)
    c = rtr.rtr_kvcache_create(1, H, d, k, R, W, dtype, 0)
    ref = oracle.ReferenceCache(H, d, k, R, W, dtype)
    try:
        compare_cache(c, ref)
        steps = 12 if k > 1000 else 40
        for _ in range(steps):
            op = rng.integers(0, 8)
            if op == 0:
                kr = synth.normal(rng, (R * k, H, d), 1.0, dtype)
                vr = synth.normal(rng, (R * k, H, d), 1.0, dtype)
                rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
                ref.set_reference(kr, vr)
            elif op == 1:
                r = int(rng.integers(0, 3))
                rtr.rtr_kvcache_retain_last(c, 0, r)
                ref.retain_last(r)
            elif op == 2 and rng.integers(0, 3) == 0:
                rtr.rtr_kvcache_clear_reference(c, 0)
                ref.clear_reference()
            else:
                n = int(rng.integers(1, W + 1))
                kn = synth.normal(rng, (n * k, H, d), 1.0, dtype)
                vn = synth.normal(rng, (n * k, H, d), 1.0, dtype)
                rtr.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), n)
                ref.append(kn, vn, n)
            torch.cuda.synchronize()
            compare_cache(c, ref)
    finally:
        rtr.rtr_kvcache_destroy(c)
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK


def test_reference_survives_many_appends_gpu():
    from causal_attention_rtr_b200 import rtr
    H, d, k, W = 2, 128, 8, 3
    rng = np.random.default_rng(77)
    c = rtr.rtr_kvcache_create(2, H, d, k, 1, W, "bf16", 0)
    ref = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    try:
        kr = synth.normal(rng, (k, H, d), 1.0, "bf16")
        vr = synth.normal(rng, (k, H, d), 1.0, "bf16")
        rtr.rtr_kvcache_set_reference(c, 1, dev(kr), dev(vr))
        ref.set_reference(kr, vr)
        for _ in range(200):
            n = int(rng.integers(1, W + 1))
            kn = synth.normal(rng, (n * k, H, d), 1.0, "bf16")
            rtr.rtr_kvcache_append_frame(c, 1, dev(kn), dev(kn), n)
            ref.append(kn, kn, n)
        torch.cuda.synchronize()
        compare_cache(c, ref, layer=1)
        # layer 0 untouched: no reference, nothing appended
        assert rtr.rtr_kvcache_get_index_map(c, 0, W) == ([-1] * W, 0, 0, 0)
    finally:
        rtr.rtr_kvcache_destroy(c)


def test_cross_cache_bit_exact():
    from causal_attention_rtr_b200 import rtr
    H, d, T = 4, 128, 77
    rng = np.random.default_rng(5)
    x = rtr.rtr_crossattn_create(2, H, d, 100, "bf16", 0)
    try:
        kt = synth.normal(rng, (T, H, d), 1.0, "bf16")
        vt = synth.normal(rng, (T, H, d), 1.0, "bf16")
        rtr.rtr_crossattn_set_text(x, 1, dev(kt), dev(vt), T)
        q = dev(synth.normal(rng, (5, H, d), 1.0, "bf16"))
        out = torch.empty_like(q)
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_attn_cross(x, 0, q, 5, out)
        assert e.value.status == rtr.RTR_E_STATE
        rtr.rtr_attn_cross(x, 1, q, 5, out)
        rtr.rtr_crossattn_reset(x)
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_attn_cross(x, 1, q, 5, out)
        assert e.value.status == rtr.RTR_E_STATE
        torch.cuda.synchronize()
    finally:
        rtr.rtr_crossattn_destroy(x)


def test_argument_errors_leave_state_unchanged():
    from causal_attention_rtr_b200 import rtr
    H, d, k, W = 2, 128, 4, 3
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    try:
        kn = dev(np.zeros((4 * k, H, d), np.uint16))
        with pytest.raises(rtr.RtrError) as e:
            rtr.rtr_kvcache_append_frame(c, 0, kn, kn, W + 1)
        assert e.value.status == rtr.RTR_E_INVAL
        with pytest.raises(rtr.RtrError):
            rtr.rtr_kvcache_append_frame(c, 1, kn, kn, 1)
        with pytest.raises(rtr.RtrError):
            rtr.rtr_kvcache_append_frame(c, 0, kn.data_ptr() + 2, kn, 1)   # misaligned
        assert rtr.rtr_kvcache_get_index_map(c, 0, W) == ([-1] * W, 0, 0, 0)
    finally:
        rtr.rtr_kvcache_destroy(c)


def _raw_view(ptr, nbytes):
    """uint8 device tensor over library-owned memory (no copy)."""
    return torch.as_tensor(_DevArray(ptr, nbytes, "|u1"), device="cuda")


def test_guard_bands_intact_after_every_kind_of_update():
    """Appends through eviction and wrap, reference overwrites, fused commits
    and text set/reset leave the 64 KB guard bands around every buffer
    untouched (no kernel writes outside its buffer)."""
    from causal_attention_rtr_b200 import rtr
    H, d, k, W, C = 3, 128, 200, 4, 2
    rng = np.random.default_rng(8)
    c = rtr.rtr_kvcache_create_ex(2, H, d, k, 1, W, C, "bf16", 0)
    x = rtr.rtr_crossattn_create(2, H, d, 64, "bf16", 0)
    try:
        for layer in range(2):
            kr, vr = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
            rtr.rtr_kvcache_set_reference(c, layer, dev(kr), dev(vr))
            for i in range(7):
                n = 1 + i % C
                q, kk, vv = (synth.normal(rng, (n * k, H, d), 1.0, "bf16") for _ in range(3))
                out = torch.empty((n * k, H, d), dtype=torch.bfloat16, device="cuda")
                if i % 2:
                    rtr.rtr_attn_frame_causal_commit(c, layer, dev(q), dev(kk), dev(vv), n, out)
                else:
                    rtr.rtr_kvcache_append_frame(c, layer, dev(kk), dev(vv), n)
            kt, vt = (synth.normal(rng, (64, H, d), 1.0, "bf16") for _ in range(2))
            rtr.rtr_crossattn_set_text(x, layer, dev(kt), dev(vt), 64)
        rtr.rtr_crossattn_reset(x)
        rtr.rtr_kvcache_check_guards(c)
        rtr.rtr_crossattn_check_guards(x)
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)


def test_allocation_failures_return_nomem():
    """Injected device-allocation failures: cache and text-cache creation and
    the attention scratch of a new stream return RTR_E_NOMEM, leave nothing
    behind, and the library works normally once the hook is cleared."""
    from causal_attention_rtr_b200 import rtr
    try:
        for after in (0, 1):
            rtr.rtr_test_fail_allocs(after, 1)
            with pytest.raises(rtr.RtrError) as e:
                rtr.rtr_kvcache_create(1, 2, 128, 16, 1, 4, "bf16", 0)
            assert e.value.status == rtr.RTR_E_NOMEM
            rtr.rtr_test_fail_allocs(after, 1)
            with pytest.raises(rtr.RtrError) as e:
                rtr.rtr_crossattn_create(1, 2, 128, 16, "bf16", 0)
            assert e.value.status == rtr.RTR_E_NOMEM
        rtr.rtr_test_fail_allocs(0, 0)
        c = rtr.rtr_kvcache_create(1, 2, 128, 16, 1, 4, "bf16", 0)
        try:
            q = torch.zeros((16, 2, 128), dtype=torch.bfloat16, device="cuda")
            out = torch.empty_like(q)
            torch.cuda.synchronize()
            s = torch.cuda.Stream()
            rtr.rtr_test_fail_allocs(0, 1)
            with pytest.raises(rtr.RtrError) as e:
                rtr.rtr_attn_frame_causal(c, 0, q, q, q, 1, out, 0.0, s)
            assert e.value.status == rtr.RTR_E_NOMEM
            rtr.rtr_test_fail_allocs(0, 0)
            rtr.rtr_attn_frame_causal(c, 0, q, q, q, 1, out, 0.0, s)
            s.synchronize()
            assert rtr.rtr_kvcache_get_index_map(c, 0, 4) == ([-1] * 4, 0, 0, 0)
        finally:
            rtr.rtr_kvcache_destroy(c)
    finally:
        rtr.rtr_test_fail_allocs(0, 0)


def test_snapshot_and_restore_resume_the_stream():
    """A cache saved (index map + a copy of its buffers) and restored into a
    new cache (bytes copied back, rtr_kvcache_set_index_map) continues the
    stream exactly: bit-identical attention and the same index maps."""
    from causal_attention_rtr_b200 import rtr
    H, d, k, R, W = 2, 128, 150, 1, 4
    rng = np.random.default_rng(21)
    a = rtr.rtr_kvcache_create(1, H, d, k, R, W, "bf16", 0)
    b = rtr.rtr_kvcache_create(1, H, d, k, R, W, "bf16", 0)
    nbytes = H * (R + W) * k * d * 2
    try:
        kr, vr = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
        rtr.rtr_kvcache_set_reference(a, 0, dev(kr), dev(vr))
        for _ in range(6):
            kk, vv = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
            rtr.rtr_kvcache_append_frame(a, 0, dev(kk), dev(vv), 1)
        torch.cuda.synchronize()
        slots, ref_valid, g, count = rtr.rtr_kvcache_get_index_map(a, 0, W)
        ka, va = rtr.rtr_kvcache_device_ptrs(a, 0)
        snap = [_raw_view(p, nbytes).clone() for p in (ka, va)]          # the saved state
        kb, vb = rtr.rtr_kvcache_device_ptrs(b, 0)
        for p, saved in zip((kb, vb), snap):
            _raw_view(p, nbytes).copy_(saved)
        rtr.rtr_kvcache_set_index_map(b, 0, g, count, ref_valid)
        assert rtr.rtr_kvcache_get_index_map(b, 0, W) == (slots, ref_valid, g, count)
        for step in range(3):
            q, kk, vv = (synth.normal(rng, (2 * k, H, d), 1.0, "bf16") for _ in range(3))
            oa, ob = (torch.empty((2 * k, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2))
            rtr.rtr_attn_frame_causal(a, 0, dev(q), dev(kk), dev(vv), 2, oa)
            rtr.rtr_attn_frame_causal(b, 0, dev(q), dev(kk), dev(vv), 2, ob)
            torch.cuda.synchronize()
            assert torch.equal(oa.view(torch.int16), ob.view(torch.int16)), f"step {step}"
            rtr.rtr_kvcache_append_frame(a, 0, dev(kk), dev(vv), 2)
            rtr.rtr_kvcache_append_frame(b, 0, dev(kk), dev(vv), 2)
            assert rtr.rtr_kvcache_get_index_map(a, 0, W) == rtr.rtr_kvcache_get_index_map(b, 0, W)
        with pytest.raises(rtr.RtrError):
            rtr.rtr_kvcache_set_index_map(b, 0, 3, 4, 1)                 # count > frames appended
        with pytest.raises(rtr.RtrError):
            rtr.rtr_kvcache_set_index_map(b, 0, 30, W + 1, 1)            # count > window
    finally:
        rtr.rtr_kvcache_destroy(a)
        rtr.rtr_kvcache_destroy(b)
