"""Pins of the DiT-block oracle (oracle/dit_block.py) against library
routines, closed forms and an independent torch composition of each branch
(papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
Architecture and Key Designs 1, 2, 4; RoFormer eq. 13-15 for the rotary
form).  CPU only."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import dit_block as db
from causal_attention_rtr_b200 import synth


# ------------------------------------------------------------------ primitives
def test_round_bf16_hand_values_and_torch():
    # bf16 keeps 8 significant bits: the ulp at 1 is 2^-7; ties go to even
    assert db.round_bf16(1 + 2 ** -8) == 1.0
    assert db.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    assert db.round_bf16(-1 - 2 ** -7) == -1 - 2 ** -7
    assert db.round_bf16(0.0) == 0.0
    x = np.random.default_rng(0).standard_normal(20000).astype(np.float32) * 3
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(db.round_bf16(x.astype(np.float64)), want)
    assert np.array_equal(oracle.decode(db.bf16_bits(want), "bf16"), want)


def test_layer_norm_and_gelu_against_torch():
    x = np.random.default_rng(1).standard_normal((7, 96)) * 2 + 0.5
    t = torch.from_numpy(x)
    assert np.allclose(db.layer_norm(x), F.layer_norm(t, (96,), eps=1e-6).numpy(), atol=1e-12)
    assert np.allclose(db.gelu_tanh(x), F.gelu(t, approximate="tanh").numpy(), atol=1e-12)
    assert db.gelu_tanh(0.0) == 0.0 and abs(db.gelu_tanh(10.0) - 10.0) < 1e-12


def test_rope_hand_case():
    """d = 6: one channel pair per part, frequency 1, so each pair turns by
    its position in radians."""
    assert db.rope_parts(6) == (2, 2, 2)
    x = np.array([1.0, 0.0, 0.0, 1.0, 2.0, 0.0]).reshape(1, 1, 6)
    got = db.rope3d(x, np.array([1]), np.array([2]), np.array([0]))[0, 0]
    want = [math.cos(1), math.sin(1), -math.sin(2), math.cos(2), 2.0, 0.0]
    assert np.allclose(got, want, atol=1e-15)
    assert db.rope_parts(128) == (44, 42, 42) and db.rope_parts(64) == (24, 20, 20)


def _rope_complex(x, t, y, xc, base=10000.0):
    """The same rotation written as complex multiplication of channel pairs."""
    x = np.asarray(x, np.float64)
    out = x.copy()
    c0 = 0
    d = x.shape[-1]
    p = 2 * (d // 6)
    for size, pos in zip((d - 2 * p, p, p), (t, y, xc)):
        z = x[..., c0:c0 + size:2] + 1j * x[..., c0 + 1:c0 + size:2]
        theta = base ** (-np.arange(0, size, 2) / size)
        z = z * np.exp(1j * np.asarray(pos, np.float64)[:, None, None] * theta)
        out[..., c0:c0 + size:2] = z.real
        out[..., c0 + 1:c0 + size:2] = z.imag
        c0 += size
    return out


def test_rope_complex_form_norm_and_relative_position():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((5, 3, 128))
    k = rng.standard_normal((5, 3, 128))
    t, y, xc = rng.integers(0, 40, 5), rng.integers(0, 30, 5), rng.integers(0, 52, 5)
    rq = db.rope3d(q, t, y, xc)
    assert np.allclose(rq, _rope_complex(q, t, y, xc), atol=1e-12)
    assert np.allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), atol=1e-12)
    assert np.array_equal(db.rope3d(q, 0 * t, 0 * y, 0 * xc), q)
    # <R(p) q, R(p') k> depends only on p - p'
    a = np.einsum("nhd,nhd->nh", db.rope3d(q, t, y, xc), db.rope3d(k, t + 3, y + 1, xc + 7))
    b = np.einsum("nhd,nhd->nh", db.rope3d(q, t + 11, y + 5, xc + 2), db.rope3d(k, t + 14, y + 6, xc + 9))
    assert np.allclose(a, b, atol=1e-10)


def test_token_positions():
    t, y, x = db.token_positions(2, 3, 4, 10)
    assert list(t) == [10] * 12 + [11] * 12
    assert list(y[:12]) == [0] * 4 + [1] * 4 + [2] * 4
    assert list(x[:12]) == [0, 1, 2, 3] * 3


# ------------------------------------------------------------------ the block
H, D_HEAD, GH, GW, C, R, W, T, FFN = 2, 64, 3, 4, 2, 1, 3, 7, 256
K = GH * GW
DM = H * D_HEAD


def _setup(seed, zero=(), gates_off=False, cross_off=False):
    rng = np.random.default_rng(seed)
    cache = oracle.ReferenceCache(H, D_HEAD, K, R, W, "bf16")
    kr, vr = (synth.normal(rng, (R * K, H, D_HEAD), 1.0, "bf16") for _ in range(2))
    cache.set_reference(kr, vr)
    for _ in range(2):
        kn, vn = (synth.normal(rng, (K, H, D_HEAD), 1.0, "bf16") for _ in range(2))
        cache.append(kn, vn, 1)
    xc = oracle.CrossCache(H, D_HEAD, 16, "bf16")
    kt, vt = (synth.normal(rng, (T, H, D_HEAD), 1.0, "bf16") for _ in range(2))
    xc.set_text(kt, vt, T)
    shapes = {"wqkv": (DM, 3 * DM), "bqkv": (3 * DM,), "wo": (DM, DM), "bo": (DM,), "wq2": (DM, DM),
              "bq2": (DM,), "wo2": (DM, DM), "bo2": (DM,), "w1": (DM, FFN), "b1": (FFN,), "w2": (FFN, DM),
              "b2": (DM,)}
    w = {}
    for name, shp in shapes.items():
        sc = 0.1 if name.startswith("b") else 1.0 / math.sqrt(shp[0])
        w[name] = synth.normal(rng, shp, sc, "bf16")
        if name in zero:
            w[name][...] = 0
    mod = synth.normal(rng, (6, DM), 0.2, "bf16")
    if gates_off:
        mod[2] = 0
        mod[5] = 0
    if cross_off:
        w["wo2"][...] = 0
        w["bo2"][...] = 0
    x = synth.normal(rng, (C * K, DM), 1.0, "bf16")
    return x, mod, w, cache, xc


def _run(x, mod, w, cache, xc, t0=5):
    return db.dit_block(x, mod, w, cache, xc, C, GH, GW, t0)


def test_block_zero_weights_is_identity():
    x, mod, w, cache, xc = _setup(3, zero=tuple(["wqkv", "bqkv", "wo", "bo", "wq2", "bq2", "wo2", "bo2", "w1",
                                                 "b1", "w2", "b2"]))
    r = _run(x, mod, w, cache, xc)
    assert np.array_equal(r["out"], oracle.decode(x, "bf16"))
    assert not oracle.decode(r["k"], "bf16").any() and not oracle.decode(r["v"], "bf16").any()


def test_block_closed_gates_and_cross_is_identity():
    x, mod, w, cache, xc = _setup(4, gates_off=True, cross_off=True)
    assert np.array_equal(_run(x, mod, w, cache, xc)["out"], oracle.decode(x, "bf16"))


def _rb(t):
    return t.to(torch.bfloat16).to(torch.float64)


def _torch_block(x, mod, w, cache, xc, t0=5, with_keys=False):
    """The block composed from torch routines (layer_norm, gelu, fp64 matmul,
    scaled_dot_product_attention with an explicit mask) and the complex-form
    rotary encoding, with the same bf16 storage points."""
    X = torch.from_numpy(oracle.decode(x, "bf16"))
    M = torch.from_numpy(oracle.decode(mod, "bf16"))
    Wt = {n: torch.from_numpy(oracle.decode(a, "bf16")) for n, a in w.items()}
    n = X.shape[0]
    ln = lambda z: F.layer_norm(z, (DM,), eps=1e-6)
    h = _rb(ln(X) * (1 + M[1]) + M[0])
    qkv = h @ Wt["wqkv"] + Wt["bqkv"]
    q, k, v = (qkv[:, i * DM:(i + 1) * DM].reshape(n, H, D_HEAD) for i in range(3))
    i = np.arange(n)
    t, yy, xx = t0 + i // K, (i % K) // GW, i % GW
    q = _rb(torch.from_numpy(_rope_complex(q.numpy(), t, yy, xx)))
    k = _rb(torch.from_numpy(_rope_complex(k.numpy(), t, yy, xx)))
    v = _rb(v)
    Kc, Vc = (torch.from_numpy(oracle.decode(a, "bf16")) for a in cache.logical_kv())
    keys, vals = torch.cat([Kc, k]), torch.cat([Vc, v])
    nc = Kc.shape[0]
    j = torch.arange(nc + n)
    vis = (j[None, :] < nc) | (((j[None, :] - nc) // K) <= (torch.arange(n)[:, None] // K))
    mask = torch.zeros(n, nc + n, dtype=torch.float64).masked_fill(~vis, float("-inf"))
    o = F.scaled_dot_product_attention(q.transpose(0, 1), keys.transpose(0, 1), vals.transpose(0, 1),
                                       attn_mask=mask).transpose(0, 1)
    o = _rb(o).reshape(n, DM)
    x1 = _rb(X + M[2] * (o @ Wt["wo"] + Wt["bo"]))
    q2 = _rb(_rb(ln(x1)) @ Wt["wq2"] + Wt["bq2"]).reshape(n, H, D_HEAD)
    kt = torch.from_numpy(oracle.decode(xc.k[:xc.n_text], "bf16"))
    vt = torch.from_numpy(oracle.decode(xc.v[:xc.n_text], "bf16"))
    o2 = F.scaled_dot_product_attention(q2.transpose(0, 1), kt.transpose(0, 1), vt.transpose(0, 1))
    o2 = _rb(o2.transpose(0, 1)).reshape(n, DM)
    x2 = _rb(x1 + (o2 @ Wt["wo2"] + Wt["bo2"]))
    h3 = _rb(ln(x2) * (1 + M[4]) + M[3])
    f = _rb(F.gelu(h3 @ Wt["w1"] + Wt["b1"], approximate="tanh"))
    out = _rb(x2 + M[5] * (f @ Wt["w2"] + Wt["b2"])).numpy()
    return (out, k.numpy()) if with_keys else out


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("seed", [5, 6])
def test_block_against_torch_composition(seed):
    x, mod, w, cache, xc = _setup(seed)
    got = _run(x, mod, w, cache, xc)["out"]
    want = _torch_block(x, mod, w, cache, xc)
    # the two differ only where fp64 summation order flips a bf16 rounding
    assert _rel(got, want) < 1e-3
    assert np.mean(got == want) > 0.97


def test_block_branches_against_torch_composition():
    """Each branch alone: self attention (FFN gate and cross output off),
    cross attention (gates off), feed-forward (self gate and cross off)."""
    for kw in ({"cross_off": True}, {"gates_off": True}):
        x, mod, w, cache, xc = _setup(7, **kw)
        if "cross_off" in kw:
            mod[5] = 0
        got, want = _run(x, mod, w, cache, xc)["out"], _torch_block(x, mod, w, cache, xc)
        assert _rel(got, want) < 1e-3
        assert not np.array_equal(got, oracle.decode(x, "bf16"))
    x, mod, w, cache, xc = _setup(8, cross_off=True)
    mod[2] = 0
    got, want = _run(x, mod, w, cache, xc)["out"], _torch_block(x, mod, w, cache, xc)
    assert _rel(got, want) < 1e-3


def test_block_key_value_outputs_are_the_rotated_projections():
    x, mod, w, cache, xc = _setup(9)
    r = _run(x, mod, w, cache, xc, t0=4)
    X = oracle.decode(x, "bf16")
    M = oracle.decode(mod, "bf16")
    h = db.round_bf16(db.layer_norm(X) * (1 + M[1]) + M[0])
    qkv = h @ oracle.decode(w["wqkv"], "bf16") + oracle.decode(w["bqkv"], "bf16")
    n = X.shape[0]
    i = np.arange(n)
    k = _rope_complex(qkv[:, DM:2 * DM].reshape(n, H, D_HEAD), 4 + i // K, (i % K) // GW, i % GW)
    assert np.array_equal(oracle.decode(r["k"], "bf16"), db.round_bf16(k))
    assert np.array_equal(oracle.decode(r["v"], "bf16"), db.round_bf16(qkv[:, 2 * DM:].reshape(n, H, D_HEAD)))


@pytest.mark.parametrize("slip", ["grid_transposed", "no_one_plus_scale", "time_off_by_one", "no_rope",
                                  "gate_ignored"])
def test_planted_block_mistakes_fail_a_pin(slip, monkeypatch):
    """A plausible mistake in the block oracle fails the torch-composition
    pin, on the output or on the rotated keys."""
    real_rope, real_pos, real_ln, real_dit = db.rope3d, db.token_positions, db.layer_norm, db.dit_block
    if slip == "grid_transposed":
        monkeypatch.setattr(db, "token_positions",
                            lambda nf, gh, gw, t0: (lambda t, y, x: (t, x, y))(*real_pos(nf, gh, gw, t0)))
    elif slip == "no_one_plus_scale":
        # LN(x) * scale + shift instead of LN(x) * (1 + scale) + shift, emulated
        # by halving the normalised input of the two modulated norms
        calls = {"n": 0}

        def ln_slip(x, eps=db.EPS):
            calls["n"] += 1
            return real_ln(x, eps) * (0.5 if calls["n"] in (1, 3) else 1.0)
        monkeypatch.setattr(db, "layer_norm", ln_slip)
    elif slip == "time_off_by_one":
        monkeypatch.setattr(db, "rope3d", lambda x, t, y, xc, base=db.ROPE_BASE: real_rope(x, t + 1, y, xc, base))
    elif slip == "no_rope":
        monkeypatch.setattr(db, "rope3d", lambda x, t, y, xc, base=db.ROPE_BASE: np.asarray(x, np.float64))
    elif slip == "gate_ignored":
        def dit_slip(x, mod, w, cache, xc, *a, **k):
            m = mod.copy()
            m[2] = db.bf16_bits(np.ones(DM))
            return real_dit(x, m, w, cache, xc, *a, **k)
        monkeypatch.setattr(db, "dit_block", dit_slip)
    x, mod, w, cache, xc = _setup(10)
    r = db.dit_block(x, mod, w, cache, xc, C, GH, GW, 5)
    want, want_k = _torch_block(x, mod, w, cache, xc, with_keys=True)
    got_k = oracle.decode(r["k"], "bf16")
    assert _rel(r["out"], want) > 1e-2 or _rel(got_k, want_k) > 1e-2


def test_block_sampled_rows_equal_the_full_block():
    x, mod, w, cache, xc = _setup(11)
    full = _run(x, mod, w, cache, xc)
    rows = np.array([0, 5, 11, 12, 23])
    part = db.dit_block(x, mod, w, cache, xc, C, GH, GW, 5, rows=rows)
    assert np.array_equal(part["out"], full["out"][rows])
    assert np.array_equal(part["k"], full["k"]) and np.array_equal(part["v"], full["v"])
