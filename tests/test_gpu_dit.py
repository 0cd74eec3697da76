"""GPU parity of one DiT block around the frame-causal attention
(rtr_dit_block_forward) against the block oracle (oracle/dit_block.py;
papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
Architecture, Key Designs 1, 2 and 4).

Tolerance: the block's output passes through about ten bf16 storage points
and two attentions; both sides store at the same points, so they differ by
fp32-versus-fp64 accumulation and the attention's bf16 P.  The bar is the
attention's relative L2 of 5e-3 and, elementwise, the attention's 2e-2
absolute or four bf16 units in the last place of the oracle's value,
whichever is larger.  The output is the residual stream after three
residual additions (gated self attention, cross attention, gated
feed-forward), each rounded to bf16 on both sides: where the fp32 and fp64
sums straddle a rounding boundary the stored values land one ulp apart, so
three additions can leave them three ulps apart, and a flip upstream (the
layer norms, the projections) can add one more through the branch that
reads it.  The residual stream holds values up to about 5, where one ulp is
2^-5 = 0.031, so an absolute 2e-2 would reject results that are right on
both sides."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import dit_block as db
from causal_attention_rtr_b200 import synth

from gpu_util import dev, host_f64
from test_gpu_cache import _raw_view

pytestmark = pytest.mark.gpu

NAMES = ("wqkv", "bqkv", "wo", "bo", "wq2", "bq2", "wo2", "bo2", "w1", "b1", "w2", "b2")


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _check(got, want, what):
    assert np.all(np.isfinite(got)), what
    rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    bound = np.maximum(2e-2, 4.0 * _bf16_ulp(want))
    worst = float(np.max(np.abs(got - want) / bound))
    print(f"{what}: rel_l2={rel:.3e} max_abs={float(np.max(np.abs(got - want))):.3e} worst/bound={worst:.3f}")
    assert rel <= 5e-3 and worst <= 1.0, f"{what}: rel_l2={rel:.3e} worst/bound={worst:.3f}"
    return rel


def _weights(rng, D, F, scale_x=1.0):
    shapes = {"wqkv": (D, 3 * D), "bqkv": (3 * D,), "wo": (D, D), "bo": (D,), "wq2": (D, D), "bq2": (D,),
              "wo2": (D, D), "bo2": (D,), "w1": (D, F), "b1": (F,), "w2": (F, D), "b2": (D,)}
    return {n: synth.normal(rng, s, 0.1 if n.startswith("b") else 1.0 / math.sqrt(s[0]), "bf16")
            for n, s in shapes.items()}


def _setup(H, d, gh, gw, R, W, appends, T, F, C, seed, room=0):
    rtr = _rtr()
    k = gh * gw
    D = H * d
    rng = np.random.default_rng(seed)
    c = rtr.rtr_kvcache_create_ex(1, H, d, k, R, W, room, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, R, W, "bf16", slots=W + room)
    if R:
        kr, vr = (synth.normal(rng, (R * k, H, d), 1.0, "bf16") for _ in range(2))
        rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
    for n in appends:
        kn, vn = (synth.normal(rng, (n * k, H, d), 1.0, "bf16") for _ in range(2))
        rtr.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), n)
        o.append(kn, vn, n)
    x = rtr.rtr_crossattn_create(1, H, d, max(T, 1), "bf16", 0)
    ox = oracle.CrossCache(H, d, max(T, 1), "bf16")
    kt, vt = (synth.normal(rng, (T, H, d), 1.0, "bf16") for _ in range(2))
    rtr.rtr_crossattn_set_text(x, 0, dev(kt), dev(vt), T)
    ox.set_text(kt, vt, T)
    w = _weights(rng, D, F)
    mod = synth.normal(rng, (6, D), 0.2, "bf16")
    hidden = synth.normal(rng, (C * k, D), 1.0, "bf16")
    return c, o, x, ox, w, mod, hidden


def _run(c, x, w, mod, hidden, C, gh, gw, t0, F, commit):
    rtr = _rtr()
    tw = {n: dev(a) for n, a in w.items()}
    tw["d_ffn"] = F
    th = dev(hidden)
    rtr.rtr_dit_block_forward(c, x, 0, tw, dev(mod), th, C, gh, gw, t0, commit)
    torch.cuda.synchronize()
    return th


CASES = [
    # H, d, grid_h, grid_w, R, W, appends, T, F, C, t0
    (2, 64, 3, 4, 1, 3, [1, 1], 7, 256, 2, 5),
    (2, 128, 10, 20, 1, 4, [2, 3], 40, 512, 2, 9),      # frames of 200 tokens: tiles straddle frames
    (3, 64, 8, 16, 0, 2, [1], 16, 384, 1, 3),           # no reference slot
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"H{c[0]}-d{c[1]}-k{c[2] * c[3]}-C{c[9]}")
@pytest.mark.parametrize("commit", [False, True])
def test_dit_block_parity(case, commit):
    H, d, gh, gw, R, W, appends, T, F, C, t0 = case
    rtr = _rtr()
    c, o, x, ox, w, mod, hidden = _setup(H, d, gh, gw, R, W, appends, T, F, C, seed=H * 100 + d + C)
    try:
        th = _run(c, x, w, mod, hidden, C, gh, gw, t0, F, commit)
        want = db.dit_block(hidden, mod, w, o, ox, C, gh, gw, t0)
        _check(host_f64(th).reshape(want["out"].shape), want["out"], str(case))
        slots, ref_valid, g, count = rtr.rtr_kvcache_get_index_map(c, 0, W)
        if commit:
            # the chunk's rotated keys and values are now the newest frames
            assert g == sum(appends) + C and count == min(W, sum(appends) + C)
            k = gh * gw
            rows = (R + W) * k
            kp, vp = rtr.rtr_kvcache_device_ptrs(c, 0)
            for ptr, bits in ((kp, want["k"]), (vp, want["v"])):
                buf = _raw_view(ptr, H * rows * d * 2).view(torch.bfloat16).view(H, rows, d)
                for i in range(C):
                    s = (sum(appends) + i) % W
                    got = buf[:, (R + s) * k:(R + s + 1) * k].float().cpu().numpy().astype(np.float64)
                    ref = oracle.decode(bits[i * k:(i + 1) * k], "bf16").transpose(1, 0, 2)
                    _check(got, ref, f"committed frame {i}")
        else:
            assert g == sum(appends)
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"H{c[0]}-d{c[1]}-k{c[2] * c[3]}-C{c[9]}")
def test_dit_block_packed_weights_bit_identical(case):
    """The block with weights packed once (rtr_dit_pack_weights) gives the
    same bits as with the row-major weights: each output element is the same
    K-ordered fp32 accumulation of the same products, whether one CTA or a
    CTA pair computes its tile and however the operands travel.  Both match
    the oracle."""
    H, d, gh, gw, R, W, appends, T, F, C, t0 = case
    rtr = _rtr()
    runs = []
    for packed in (False, True):
        c, o, x, ox, w, mod, hidden = _setup(H, d, gh, gw, R, W, appends, T, F, C, seed=H * 100 + d + C + 7)
        try:
            tw = {n: dev(a) for n, a in w.items()}
            tw["d_ffn"] = F
            th = dev(hidden)
            if packed:
                pw = rtr.rtr_dit_pack_weights(tw, H * d, 0)
                try:
                    rtr.rtr_dit_block_forward_packed(c, x, 0, pw, dev(mod), th, C, gh, gw, t0, False)
                    torch.cuda.synchronize()
                finally:
                    rtr.rtr_dit_packed_destroy(pw)
            else:
                rtr.rtr_dit_block_forward(c, x, 0, tw, dev(mod), th, C, gh, gw, t0, False)
                torch.cuda.synchronize()
            runs.append(th)
            want = db.dit_block(hidden, mod, w, o, ox, C, gh, gw, t0)
            _check(host_f64(th).reshape(want["out"].shape), want["out"], f"{case} packed={packed}")
            assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
        finally:
            rtr.rtr_kvcache_destroy(c)
            rtr.rtr_crossattn_destroy(x)
    assert torch.equal(runs[0].view(torch.int16), runs[1].view(torch.int16))


def test_dit_block_fused_commit_equals_append():
    """A cache with commit room writes the chunk from the attention launch;
    the block's output and the committed bytes equal the append path's."""
    rtr = _rtr()
    H, d, gh, gw, R, W, T, F, C = 2, 128, 10, 20, 1, 3, 12, 256, 2
    a = _setup(H, d, gh, gw, R, W, [1, 2], T, F, C, seed=77, room=C)
    b = _setup(H, d, gh, gw, R, W, [1, 2], T, F, C, seed=77, room=0)
    try:
        ha = _run(a[0], a[2], a[4], a[5], a[6], C, gh, gw, 4, F, True)
        hb = _run(b[0], b[2], b[4], b[5], b[6], C, gh, gw, 4, F, True)
        assert torch.equal(ha.view(torch.int16), hb.view(torch.int16))
        k = gh * gw
        for (pa, pb) in zip(rtr.rtr_kvcache_device_ptrs(a[0], 0), rtr.rtr_kvcache_device_ptrs(b[0], 0)):
            sa = rtr.rtr_kvcache_get_index_map(a[0], 0, W + C)[0]
            sb = rtr.rtr_kvcache_get_index_map(b[0], 0, W)[0]
            ra, rb = (R + W + C) * k, (R + W) * k
            ta = _raw_view(pa, H * ra * d * 2).view(torch.int16).view(H, ra, d)
            tb = _raw_view(pb, H * rb * d * 2).view(torch.int16).view(H, rb, d)
            for f in (3, 4):                                  # the two committed frames
                ia, ib = sa.index(f), sb.index(f)
                assert torch.equal(ta[:, (R + ia) * k:(R + ia + 1) * k], tb[:, (R + ib) * k:(R + ib + 1) * k])
    finally:
        for t in (a, b):
            rtr.rtr_kvcache_destroy(t[0])
            rtr.rtr_crossattn_destroy(t[2])


def test_dit_block_rejects_bad_arguments():
    rtr = _rtr()
    H, d, gh, gw = 2, 64, 3, 4
    c, o, x, ox, w, mod, hidden = _setup(H, d, gh, gw, 1, 3, [1], 5, 256, 1, seed=3)
    x2 = rtr.rtr_crossattn_create(1, H, d, 8, "bf16", 0)      # no text set
    try:
        tw = {n: dev(a) for n, a in w.items()}
        tw["d_ffn"] = 256
        th = dev(hidden)
        tm = dev(mod)
        for args, want in [((c, x, 0, tw, tm, th, 1, 4, 4, 0), rtr.RTR_E_INVAL),     # grid != k
                           ((c, x, 1, tw, tm, th, 1, 3, 4, 0), rtr.RTR_E_INVAL),     # no such layer
                           ((c, x2, 0, tw, tm, th, 1, 3, 4, 0), rtr.RTR_E_STATE),    # text not set
                           ((c, x, 0, dict(tw, d_ffn=100), tm, th, 1, 3, 4, 0), rtr.RTR_E_INVAL)]:
            with pytest.raises(rtr.RtrError) as e:
                rtr.rtr_dit_block_forward(*args)
            assert e.value.status == want
        assert rtr.rtr_kvcache_get_index_map(c, 0, 3)[2] == 1
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)
        rtr.rtr_crossattn_destroy(x2)


def test_full_wan13_block_sampled():
    """A Wan-1.3B-shaped block (12 heads, d 128, 30 x 52 tokens per frame,
    chunk of 3 frames against 1 reference + 21 window frames, 512 text
    tokens, feed-forward 8960): sampled rows against the oracle."""
    H, d, gh, gw, R, W, T, F, C = 12, 128, 30, 52, 1, 21, 512, 8960, 3
    rtr = _rtr()
    c, o, x, ox, w, mod, hidden = _setup(H, d, gh, gw, R, W, [3] * 7, T, F, C, seed=1313)
    try:
        th = _run(c, x, w, mod, hidden, C, gh, gw, 22, F, False)
        rows = np.array(sorted({0, 1, 1559, 1560, 3119, 3120, 4679}
                               | set(np.random.default_rng(9).integers(0, C * gh * gw, 9).tolist())))
        want = db.dit_block(hidden, mod, w, o, ox, C, gh, gw, 22, rows=rows)
        _check(host_f64(th).reshape(C * gh * gw, H * d)[rows], want["out"], "sampled rows")
        # the same block with packed weights: bit-identical
        tw = {n: dev(a) for n, a in w.items()}
        tw["d_ffn"] = F
        pw = rtr.rtr_dit_pack_weights(tw, H * d, 0)
        try:
            th2 = dev(hidden)
            rtr.rtr_dit_block_forward_packed(c, x, 0, pw, dev(mod), th2, C, gh, gw, 22, False)
            torch.cuda.synchronize()
        finally:
            rtr.rtr_dit_packed_destroy(pw)
        assert torch.equal(th.view(torch.int16), th2.view(torch.int16))
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    finally:
        rtr.rtr_kvcache_destroy(c)
        rtr.rtr_crossattn_destroy(x)
