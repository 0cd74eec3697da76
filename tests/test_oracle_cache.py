"""Pins of the oracle's cache state machine (reference-preserving rolling KV
cache) against hand-written sequences, closed forms and the invariants the
pages state.

Source: papernotes.org note "DiT as Real-Time Rerenderer", Method > Key
Designs 4 (rolling cache, oldest frames evicted, reference anchored in a
resident slot, switch keeps the most recent frame) and Key Designs 1 (the
reference is one latent frame in front of the first frame).
"""
import os

import numpy as np
import pytest

import oracle
from causal_attention_rtr_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_script(name):
    ops = []
    for line in open(os.path.join(GOLDEN, name)):
        if not line.strip() or line.startswith("#"):
            continue
        op, slots, ref, g = [p.strip() for p in line.split("|")]
        kind, arg = op.split()
        ops.append((kind, int(arg), [int(x) for x in slots.split()], int(ref), int(g)))
    return ops


def frame_data(f, k, H, d):
    """A recognisable frame: every element encodes the frame index."""
    return np.full((k, H, d), f % 60000 + 1, np.uint16)


def run_script(cache_cls, name="eviction_W4.txt"):
    k, H, d = 2, 1, 2
    c = cache_cls(H, d, k, 1, 4, "bf16")
    nxt = 0
    for kind, arg, slots, ref, g in read_script(name):
        if kind == "set_ref":
            c.set_reference(np.full((k, H, d), 7, np.uint16), np.full((k, H, d), 9, np.uint16))
        elif kind == "clear_ref":
            c.clear_reference()
        elif kind == "retain":
            c.retain_last(arg)
        elif kind == "append":
            ks = np.concatenate([frame_data(nxt + i, k, H, d) for i in range(arg)])
            c.append(ks, ks, arg)
            nxt += arg
        yield c, (slots, ref, g)


def test_golden_eviction_script():
    for c, (slots, ref, g) in run_script(oracle.ReferenceCache):
        assert c.index_map() == (slots, ref, g)
        # the data in each valid slot is the frame the index map names
        for s, f in enumerate(slots):
            if f >= 0:
                assert np.all(c.slots_k[s] == f % 60000 + 1)


@pytest.mark.parametrize("W", [1, 2, 3, 5, 21])
def test_closed_form_eviction(W):
    """After g appends and no trims the map is {f mod W -> f, f in [g-min(g,W), g)}."""
    rng = np.random.default_rng(W)
    c = oracle.ReferenceCache(1, 2, 1, 1, W, "f32")
    g = 0
    for _ in range(60):
        n = int(rng.integers(1, W + 1))
        c.append(np.zeros((n, 1, 2), np.float32), np.zeros((n, 1, 2), np.float32), n)
        g += n
        want = [-1] * W
        for f in range(g - min(g, W), g):
            want[f % W] = f
        assert c.index_map() == (want, 0, g)


def test_reference_survives_any_eviction():
    """The reference bytes equal the last set_reference input and stay valid
    through 10^4 appended frames and random retain / set sequences."""
    H, d, k, W = 2, 4, 3, 5
    rng = np.random.default_rng(11)
    c = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    ref_k = synth.normal(rng, (k, H, d), 1.0, "bf16")
    ref_v = synth.normal(rng, (k, H, d), 1.0, "bf16")
    c.set_reference(ref_k, ref_v)
    total = 0
    while total < 10_000:
        op = rng.integers(0, 10)
        if op == 0:
            c.retain_last(int(rng.integers(0, 3)))
        elif op == 1:
            ref_k = synth.normal(rng, (k, H, d), 1.0, "bf16")
            ref_v = synth.normal(rng, (k, H, d), 1.0, "bf16")
            c.set_reference(ref_k, ref_v)
        else:
            n = int(rng.integers(1, W + 1))
            x = synth.normal(rng, (n * k, H, d), 1.0, "bf16")
            c.append(x, x, n)
            total += n
        assert c.ref_valid
        assert np.array_equal(c.ref_k, ref_k) and np.array_equal(c.ref_v, ref_v)
        K, V = c.logical_kv()
        assert np.array_equal(K[: k], ref_k) and np.array_equal(V[: k], ref_v)


class NaiveRing(oracle.ReferenceCache):
    """Negative control: the reference treated as an ordinary frame of a
    rolling window of W+1 frames (the failure mode the pages describe: the
    reference is evicted as soon as the cache fills)."""

    def set_reference(self, k_ref, v_ref):
        self.ring = [(np.asarray(k_ref).copy(), np.asarray(v_ref).copy(), "ref")]

    def append(self, k_new, v_new, n_frames):
        k_new = np.asarray(k_new).reshape(n_frames, self.k, self.H, self.d)
        for i in range(n_frames):
            self.ring.append((k_new[i], k_new[i], "frame"))
        self.ring = self.ring[-(self.W + 1):]

    def has_reference(self):
        return any(tag == "ref" for _, _, tag in self.ring)


def test_negative_control_naive_ring_loses_reference():
    W, k = 4, 2
    naive = NaiveRing(1, 2, k, 1, W, "bf16")
    naive.set_reference(np.ones((k, 1, 2), np.uint16), np.ones((k, 1, 2), np.uint16))
    anchored = oracle.ReferenceCache(1, 2, k, 1, W, "bf16")
    anchored.set_reference(np.ones((k, 1, 2), np.uint16), np.ones((k, 1, 2), np.uint16))
    for f in range(W + 1):
        x = np.zeros((k, 1, 2), np.uint16)
        naive.append(x, x, 1)
        anchored.append(x, x, 1)
    assert not naive.has_reference()        # evicted after W+1 frames
    assert anchored.ref_valid               # still anchored


def test_stream_equals_prefill_without_eviction():
    """With W >= frames streamed, each chunk's streaming attention equals the
    corresponding rows of the block-causal prefill over [ref | all frames]."""
    H, d, k, F, C = 2, 16, 5, 7, 1
    rng = np.random.default_rng(21)
    for ref in (True, False):
        c = oracle.ReferenceCache(H, d, k, 1, 8, "bf16")
        seq_k, seq_v, seq_q = [], [], []
        if ref:
            rk = synth.normal(rng, (k, H, d), 1.0, "bf16")
            rv = synth.normal(rng, (k, H, d), 1.0, "bf16")
            c.set_reference(rk, rv)
            seq_k.append(rk); seq_v.append(rv); seq_q.append(np.zeros_like(rk))
        outs = []
        for f in range(F):
            q = synth.normal(rng, (C * k, H, d), 1.0, "bf16")
            kc = synth.normal(rng, (C * k, H, d), 1.0, "bf16")
            vc = synth.normal(rng, (C * k, H, d), 1.0, "bf16")
            outs.append(c.stream_attention(q, kc, vc, C))
            c.append(kc, vc, C)
            seq_q.append(q); seq_k.append(kc); seq_v.append(vc)
        Q, K, V = (oracle.decode(np.concatenate(s), "bf16") for s in (seq_q, seq_k, seq_v))
        pre = oracle.prefill(Q, K, V, k)
        off = k if ref else 0
        got = np.concatenate(outs)
        assert np.allclose(got, pre[off:], rtol=1e-12, atol=1e-13)


def test_stream_chunk_is_frame_causal():
    """Within a multi-frame chunk, chunk frame c sees chunk frames <= c only:
    perturbing frame c+1's K/V leaves frame c's rows bit-identical."""
    H, d, k, C = 2, 8, 4, 3
    w = synth.Workload("t", "bf16", 1, H, d, k, 1, 3, C, 1.0, 9)
    x = synth.stream_layer_inputs(w)
    c = oracle.ReferenceCache(H, d, k, 1, 3, "bf16")
    c.set_reference(x.ref_k, x.ref_v)
    for fk, fv in zip(x.window_k, x.window_v):
        c.append(fk, fv, 1)
    base = c.stream_attention(x.q, x.k_cur, x.v_cur, C)
    for f in range(1, C):
        k2 = x.k_cur.copy(); v2 = x.v_cur.copy()
        k2[f * k:] ^= np.uint16(0x0040)
        v2[f * k:] ^= np.uint16(0x0040)
        out = c.stream_attention(x.q, k2, v2, C)
        assert np.array_equal(out[: f * k], base[: f * k])
        assert not np.array_equal(out[f * k:], base[f * k:])


def test_window_order_is_oldest_first():
    c = oracle.ReferenceCache(1, 1, 1, 1, 3, "f32")
    for f in range(5):
        c.append(np.full((1, 1, 1), f, np.float32), np.full((1, 1, 1), f, np.float32), 1)
    K, _ = c.logical_kv()                       # no reference set
    assert K[:, 0, 0].tolist() == [2.0, 3.0, 4.0]
    assert c.chunk_first_frame() == 3


def test_cross_cache_reset_and_set():
    rng = np.random.default_rng(3)
    x = oracle.CrossCache(2, 8, 16, "bf16")
    with pytest.raises(RuntimeError):
        x.attention(synth.normal(rng, (4, 2, 8), 1.0, "bf16"))
    kt = synth.normal(rng, (10, 2, 8), 1.0, "bf16")
    vt = synth.normal(rng, (10, 2, 8), 1.0, "bf16")
    x.set_text(kt, vt, 10)
    q = synth.normal(rng, (4, 2, 8), 1.0, "bf16")
    out = x.attention(q)
    Q, K, V = (oracle.decode(a, "bf16") for a in (q, kt, vt))
    # unmasked: equals the dense softmax over all 10 text keys
    from scipy.special import softmax
    for h in range(2):
        want = softmax(Q[:, h] @ K[:, h].T / np.sqrt(8), axis=1) @ V[:, h]
        assert np.allclose(out[:, h], want, rtol=1e-12, atol=1e-13)
    x.reset()
    with pytest.raises(RuntimeError):
        x.attention(q)


@pytest.mark.parametrize("W,extra", [(1, 1), (3, 2), (5, 3), (21, 3)])
def test_closed_form_eviction_with_spare_slots(W, extra):
    """With S = W + extra physical slots and no trims, the map is
    {f mod S -> f, f in [g-min(g,W), g)}: W frames held, S slots addressed."""
    S = W + extra
    rng = np.random.default_rng(100 + W)
    c = oracle.ReferenceCache(1, 2, 1, 1, W, "f32", slots=S)
    g = 0
    for _ in range(60):
        n = int(rng.integers(1, W + 1))
        c.append(np.zeros((n, 1, 2), np.float32), np.zeros((n, 1, 2), np.float32), n)
        g += n
        want = [-1] * S
        for f in range(g - min(g, W), g):
            want[f % S] = f
        assert c.index_map() == (want, 0, g)


def test_spare_slots_change_nothing_but_placement():
    """Two caches fed the same random operations, one with S = W and one with
    S = W + 3 slots, hold the same logical sequence and give bit-identical
    attention; every held frame sits at f mod S in its own cache."""
    H, d, k, W, C = 2, 8, 3, 4, 2
    rng = np.random.default_rng(77)
    a = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    b = oracle.ReferenceCache(H, d, k, 1, W, "bf16", slots=W + 3)
    frames = {}
    g = 0
    for step in range(40):
        op = int(rng.integers(0, 6))
        if op == 0:
            rk, rv = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
            a.set_reference(rk, rv); b.set_reference(rk, rv)
        elif op == 1:
            r = int(rng.integers(0, 3))
            a.retain_last(r); b.retain_last(r)
        else:
            n = int(rng.integers(1, W + 1))
            x, y = (synth.normal(rng, (n * k, H, d), 1.0, "bf16") for _ in range(2))
            a.append(x, y, n); b.append(x, y, n)
            for i in range(n):
                frames[g + i] = x[i * k:(i + 1) * k]
            g += n
        Ka, Va = a.logical_kv()
        Kb, Vb = b.logical_kv()
        assert np.array_equal(Ka, Kb) and np.array_equal(Va, Vb)
        assert a.window_frames() == b.window_frames()
        for f in b.window_frames():
            assert np.array_equal(b.slots_k[f % (W + 3)], frames[f])
        if step % 8 == 7:
            q, kc, vc = (synth.normal(rng, (C * k, H, d), 1.0, "bf16") for _ in range(3))
            assert np.array_equal(a.stream_attention(q, kc, vc, C), b.stream_attention(q, kc, vc, C))


def test_spare_slots_must_cover_window():
    with pytest.raises(ValueError):
        oracle.ReferenceCache(1, 2, 1, 1, 4, "f32", slots=3)
