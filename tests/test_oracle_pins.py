"""Pins of the fp64 oracle's attention against things other than itself.

Each pin checks the oracle against what the pages or the mathematics fix:
hand-written fixtures, a dense explicit-mask brute force, PyTorch's own
scaled_dot_product_attention in its textbook special cases, closed forms and
invariants.  ``test_planted_mistakes_are_caught`` shows that plausible slips
in an attention routine (a flipped mask comparison, a missing scale, a
transposed operand, a dropped term) each fail at least one of these pins.

Source of the definition: papernotes.org note "DiT as Real-Time
Rerenderer", Method > Key Designs 2 (attention/mask equation).
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from causal_attention_rtr_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_matrix(name):
    rows = [l.split() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]
    return np.array([[float(x) for x in r] for r in rows])


def _rand(seed, n, H, d):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((n, H, d)) for _ in range(3)]


def brute_force(q, k, v, kpf, scale=None):
    """Dense reference: explicit n x n additive mask with -inf entries, then a
    row softmax from scipy, then one matrix product per head."""
    n, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    i = np.arange(n)[:, None]
    j = np.arange(k.shape[0])[None, :]
    M = np.where((j // kpf) <= (i // kpf), 0.0, -np.inf)
    out = np.empty_like(q)
    for h in range(H):
        S = q[:, h, :] @ k[:, h, :].T * scale + M
        out[:, h, :] = scipy.special.softmax(S, axis=1) @ v[:, h, :]
    return out


# --------------------------------------------------------------------------
# Pins written as functions of an attention routine with the oracle's
# signature, so the same checks can be run on planted mistakes.

def pin_golden_masks(attn):
    """Uniform keys make the softmax flat over the visible set, so each output
    equals the mean of the visible values; with one-hot values the output row
    is the visible row of the hand-written mask divided by its count."""
    for name, kpf in (("mask_k2_n7.txt", 2), ("mask_k3_n8.txt", 3)):
        vis = _read_matrix(name)
        n = vis.shape[0]
        q = np.ones((n, 1, 4))
        k = np.ones((n, 1, 4))
        v = np.eye(n)[:, None, :]                      # value j = e_j, d = n
        out = attn(np.pad(q, ((0, 0), (0, 0), (0, n - 4))), np.arange(n),
                   np.pad(k, ((0, 0), (0, 0), (0, n - 4))), v, kpf, True, None)
        want = vis / vis.sum(axis=1, keepdims=True)
        if not np.allclose(out[:, 0, :], want, rtol=0, atol=1e-14):
            return False
    return True


def pin_two_key_closed_form(attn):
    rows = _read_matrix("two_key_closed_form.txt")
    q = rows[:, 0].reshape(2, 1, 1)
    k = rows[:, 1].reshape(2, 1, 1)
    v = rows[:, 2].reshape(2, 1, 1)
    out = attn(q, rows[:, 3].astype(np.int64), k, v, 1, True, 1.0)
    return np.allclose(out[:, 0, 0], rows[:, 4], rtol=0, atol=1e-13)


def pin_brute_force(attn):
    for seed, (kpf, frames, H, d) in enumerate([(1, 9, 2, 8), (2, 6, 1, 16), (3, 5, 3, 8),
                                                 (16, 4, 2, 32), (5, 12, 1, 4), (7, 3, 2, 8)]):
        n = kpf * frames - (1 if kpf > 1 else 0)        # ragged last frame
        q, k, v = _rand(100 + seed, n, H, d)
        out = attn(q, np.arange(n), k, v, kpf, True, None)
        ref = brute_force(q, k, v, kpf)
        if not np.allclose(out, ref, rtol=1e-12, atol=1e-12):
            return False
    return True


def pin_torch_sdpa(attn):
    """k = 1 is token-causal attention; k >= n is full bidirectional attention
    (the teacher's case).  PyTorch's SDPA (fp64, CPU) computes both."""
    for seed, (n, H, d) in enumerate([(13, 2, 16), (33, 3, 8), (8, 1, 64)]):
        q, k, v = _rand(200 + seed, n, H, d)
        tq, tk, tv = (torch.from_numpy(x).permute(1, 0, 2) for x in (q, k, v))
        causal = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
        full = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=False)
        o1 = attn(q, np.arange(n), k, v, 1, True, None)
        o2 = attn(q, np.arange(n), k, v, n, True, None)
        o3 = attn(q, np.arange(n), k, v, 1, False, None)
        if not (np.allclose(o1, causal.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
                and np.allclose(o2, full.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
                and np.allclose(o3, full.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)):
            return False
    return True


def pin_single_visible_key(attn):
    """With k = 1 the first query sees exactly one key, so its output is that
    value row, exactly."""
    q, k, v = _rand(300, 10, 3, 16)
    out = attn(q, np.arange(10), k, v, 1, True, None)
    return np.array_equal(out[0], v[0])


def pin_convexity(attn):
    q, k, v = _rand(301, 40, 2, 8)
    q *= 4.0
    kpf = 6
    out = attn(q, np.arange(40), k, v, kpf, True, None)
    for i in range(40):
        vis = v[: (i // kpf + 1) * kpf]
        if np.any(out[i] < vis.min(axis=0) - 1e-12) or np.any(out[i] > vis.max(axis=0) + 1e-12):
            return False
    return True


def pin_no_future_frame(attn):
    """Changing K/V of later frames leaves every earlier row bit-identical."""
    kpf, frames = 4, 6
    n = kpf * frames
    q, k, v = _rand(302, n, 2, 8)
    base = attn(q, np.arange(n), k, v, kpf, True, None)
    for f in range(1, frames):
        k2, v2 = k.copy(), v.copy()
        k2[f * kpf:] += 10.0
        v2[f * kpf:] -= 7.0
        out = attn(q, np.arange(n), k2, v2, kpf, True, None)
        if not np.array_equal(out[: f * kpf], base[: f * kpf]):
            return False
        if np.array_equal(out[f * kpf:], base[f * kpf:]):
            return False          # later rows must see the change
    return True


PINS = [pin_golden_masks, pin_two_key_closed_form, pin_brute_force, pin_torch_sdpa,
        pin_single_visible_key, pin_convexity, pin_no_future_frame]


def oracle_attn(q, q_pos, k, v, kpf, causal, scale):
    return oracle.attention(q, q_pos, k, v, kpf, causal, scale)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    assert pin(oracle_attn)


def test_visible_matches_golden():
    for name, kpf in (("mask_k2_n7.txt", 2), ("mask_k3_n8.txt", 3)):
        vis = _read_matrix(name)
        n = vis.shape[0]
        got = np.array([[oracle.visible(i, j, kpf) for j in range(n)] for i in range(n)])
        assert np.array_equal(got, vis.astype(bool))


# --------------------------------------------------------------------------
# Planted mistakes (on the CPU): each is a plausible slip in an attention
# routine; at least one pin must reject each.

def _mutant(kind):
    def attn(q, q_pos, k, v, kpf, causal, scale):
        q = np.asarray(q, float); k = np.asarray(k, float); v = np.asarray(v, float)
        n, H, d = q.shape
        sc = 1.0 / math.sqrt(d) if scale is None else scale
        if kind == "no_scale":
            sc = 1.0
        q_pos = np.asarray(q_pos)
        j = np.arange(k.shape[0])
        out = np.zeros_like(q)
        for r in range(n):
            if not causal:
                vis = np.ones_like(j, bool)
            elif kind == "strict_mask":
                vis = (j // kpf) < (q_pos[r] // kpf)
            elif kind == "token_mask":
                vis = j <= q_pos[r]
            else:
                vis = (j // kpf) <= (q_pos[r] // kpf)
            if kind == "unmasked":
                vis = np.ones_like(j, bool)
            for h in range(H):
                kk, vv = k[:, h, :], v[:, h, :]
                if kind == "transposed_heads":
                    kk, vv = k[:, (h + 1) % H, :], v[:, (h + 1) % H, :]
                s = kk @ q[r, h] * sc
                s = np.where(vis, s, -np.inf)
                p = np.exp(s - s[vis].max()) if vis.any() else np.zeros_like(s)
                if kind == "no_normalise":
                    out[r, h] = p @ vv
                elif kind == "drop_last_key":
                    p = p.copy(); last = np.nonzero(vis)[0][-1]; p[last] = 0
                    out[r, h] = p @ vv / max(p.sum(), 1e-300)
                else:
                    out[r, h] = p @ vv / max(p.sum(), 1e-300)
        return out
    return attn


@pytest.mark.parametrize("kind", ["no_scale", "strict_mask", "token_mask", "unmasked",
                                  "transposed_heads", "no_normalise", "drop_last_key"])
def test_planted_mistakes_are_caught(kind):
    mutant = _mutant(kind)
    failed = [p.__name__ for p in PINS if not p(mutant)]
    assert failed, f"no pin catches the planted mistake {kind!r}"


def test_unplanted_mutant_passes_pins():
    """The mutant harness itself, with no mistake planted, passes every pin
    (so the failures above come from the planted slips)."""
    clean = _mutant("none")
    assert all(p(clean) for p in PINS)


def test_prefill_rows_subset():
    q, k, v = synth.random_qkv(5, 30, 2, 16, "bf16")
    Q, K, V = (oracle.decode(x, "bf16") for x in (q, k, v))
    full = oracle.prefill(Q, K, V, 4)
    rows = np.array([0, 3, 7, 29])
    part = oracle.prefill(Q, K, V, 4, rows=rows)
    assert np.array_equal(part, full[rows])


def test_decode_bf16_exact():
    x = np.array([1.0, -2.5, 3.140625, 65504.0, 1e-30], np.float32)
    bits = synth.f32_to_bf16_bits(x)
    got = oracle.decode(bits, "bf16")
    # 1.0, -2.5 and 3.140625 are exact in bf16; 65504 rounds to 65536 (ties
    # to even at 8 mantissa bits); the tiny value keeps its exponent.
    assert got[0] == 1.0 and got[1] == -2.5 and got[2] == 3.140625
    assert got[3] == 65536.0
    assert abs(got[4] - 1e-30) / 1e-30 < 2 ** -8
