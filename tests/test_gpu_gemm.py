"""GPU parity of the DiT block's tensor-core projections with their fused
epilogues (rtr_dit_linear, rtr_dit_qkv_rope) against the block oracle's own
steps (oracle/dit_block.py: fp64 products of the same bf16 operands, the
bias / GELU / gated residual / 3D rotary encoding in fp64, one rounding to
bf16; papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
Architecture).

Tolerance, per element: one bf16 unit in the last place of the result plus
the error bound of the fp32 accumulation.  Both sides round the same
quantity once to bf16, the GPU from an fp32 sum of K exact bf16 products
and the oracle from fp64.  Whatever the order and rounding mode, an fp32
sum of K terms is within K * 2^-23 * sum_k |a_k w_k| of the exact sum
(the standard recursive-summation bound with truncating additions, here
taken for any order); the bias adds |b| to the sum of magnitudes.  That
absolute error passes through the epilogue (times at most 1.13 for GELU's
slope, |gate| for the gated residual, and into both members of a rotary
pair), and the epilogue's own fp32 operations add a few fp32 units of its
result.  Where the result is far smaller than the terms that made it
(cancellation in the sum, GELU of a strongly negative input) the bound is
that absolute error, many bf16 ulps of the small result; elsewhere it is
about one ulp.  As checks of the whole matrix, under 1 % of the elements
may differ from the oracle at all (a wrong layout, tile or race changes
nearly every element of the tiles it touches) and the relative L2 error
must stay below 1e-3 (one-ulp differences on a small fraction of the
elements give about 1e-4)."""
import numpy as np
import pytest
import torch

from oracle import dit_block as db
from oracle.attention import decode
from causal_attention_rtr_b200 import synth

from gpu_util import dev, host_f64

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def _ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def acc_error(A, Wt, B, k):
    """Bound of the fp32 accumulation error of A @ Wt + B, per element."""
    return k * 2.0 ** -23 * (np.abs(A) @ np.abs(Wt) + np.abs(B))


def assert_parity(got, want, err_abs, what):
    """|got - want| <= one bf16 ulp + err_abs + a few fp32 units, every
    element; under 1 % of the elements different at all."""
    assert np.all(np.isfinite(got)), what
    mag = np.maximum(np.abs(got), np.abs(want))
    bound = _ulp(mag) + err_abs + 8 * 2.0 ** -24 * mag
    excess = np.abs(got - want) / bound
    worst = float(np.max(excess))
    frac_diff = float(np.mean(got != want))
    i = np.unravel_index(int(np.argmax(excess)), excess.shape)
    detail = f"worst at {i}: got {got[i]!r} want {want[i]!r} bound {bound[i]:.3e}"
    print(f"{what}: worst/bound={worst:.3f} differing={frac_diff:.2e} ({detail})")
    rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    print(f"{what}: rel_l2={rel:.3e}")
    assert worst <= 1.0, f"{what}: {detail}"
    assert frac_diff < 0.01, f"{what}: {frac_diff:.2%} of the elements differ"
    assert rel <= 1e-3, f"{what}: rel_l2={rel:.3e}"
    return worst, frac_diff


def _operands(rng, m, n, k, x_scale=1.0):
    a = synth.normal(rng, (m, k), x_scale, "bf16")
    w = synth.normal(rng, (k, n), 1.0 / np.sqrt(k), "bf16")
    b = synth.normal(rng, (n,), 0.1, "bf16")
    return a, w, b


LINEAR_CASES = [
    # m, n, k, epilogue
    (300, 200, 72, "bias"),              # ragged m, n (not a multiple of 64) and k
    (1, 64, 8, "bias"),                  # one row, one short K block
    (4680, 8960, 1536, "gelu"),          # the Wan-1.3B feed-forward input projection
    (1000, 1536, 8960, "gated_residual"),   # long K: the feed-forward output projection
    (777, 1536, 1536, "gated_residual_nogate"),
    (4680, 1536, 1536, "bias"),          # the cross-attention query projection
    (4800, 3072, 512, "bias"),           # 256-row tiles whose last has a partial second sub-tile
    (4800, 4600, 1024, "bias"),          # CTA-pair tiles: the last row tile's second CTA holds 64 rows,
                                         # the last column tile's second CTA a partial weight box
]


@pytest.mark.parametrize("m,n,k,epi", LINEAR_CASES, ids=lambda c: str(c))
def test_dit_linear_parity(m, n, k, epi):
    rtr = _rtr()
    rng = np.random.default_rng(m + n + k)
    a, w, b = _operands(rng, m, n, k)
    A, Wt, B = decode(a, "bf16"), decode(w, "bf16"), decode(b, "bf16")
    C = A @ Wt + B
    E = acc_error(A, Wt, B, k)
    gate = None
    if epi.startswith("gated_residual"):
        x = synth.normal(rng, (m, n), 1.0, "bf16")
        X = decode(x, "bf16")
        if epi == "gated_residual":
            gate = synth.normal(rng, (n,), 0.5, "bf16")
            G = decode(gate, "bf16")
            want = db.round_bf16(X + G * C)
            E = E * np.abs(G) + 4 * 2.0 ** -24 * (np.abs(X) + np.abs(G * C))
        else:
            want = db.round_bf16(X + C)
            E = E + 4 * 2.0 ** -24 * (np.abs(X) + np.abs(C))
        out = dev(x)
        code = "gated_residual"
    elif epi == "gelu":
        want = db.round_bf16(db.gelu_tanh(C))
        E = 1.13 * E + 2.0 ** -20 * np.abs(C)
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        code = "gelu"
    else:
        want = db.round_bf16(C)
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        code = "bias"
    rtr.rtr_dit_linear(dev(a), dev(w), m, n, k, code, dev(b), None if gate is None else dev(gate), out)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    assert_parity(host_f64(out), want, E, f"{epi} m={m} n={n} k={k}")


QKV_CASES = [
    # heads, head_dim, grid_h, grid_w, frames, t0
    (12, 128, 30, 52, 3, 22),            # the Wan-1.3B chunk: 4680 tokens, D = 1536
    (3, 64, 5, 10, 5, 3),                # head_dim 64, 250 tokens (ragged last tile)
    (2, 128, 1, 7, 1, 0),                # 7 tokens, position 0
]


@pytest.mark.parametrize("H,d,gh,gw,C,t0", QKV_CASES, ids=lambda c: str(c))
def test_dit_qkv_rope_parity(H, d, gh, gw, C, t0):
    rtr = _rtr()
    D, k = H * d, gh * gw
    m = C * k
    rng = np.random.default_rng(H * d + m)
    a, w, b = _operands(rng, m, 3 * D, D)
    A, Wt, B = decode(a, "bf16"), decode(w, "bf16"), decode(b, "bf16")
    qkv = A @ Wt + B
    E = acc_error(A, Wt, B, D)
    t, yy, xx = db.token_positions(C, gh, gw, t0)

    def pair_err(e3):
        """A rotary pair mixes both members' errors; the fp32 angle adds a
        few fp32 units of the pair's magnitude."""
        e = e3.reshape(m, H, d // 2, 2).sum(axis=-1, keepdims=True)
        return np.broadcast_to(e, (m, H, d // 2, 2)).reshape(m, H, d)

    want, errs = [], []
    for part in range(3):
        v = qkv[:, part * D:(part + 1) * D].reshape(m, H, d)
        e = E[:, part * D:(part + 1) * D].reshape(m, H, d)
        if part < 2:
            mag = np.abs(v).reshape(m, H, d // 2, 2).sum(axis=-1, keepdims=True)
            mag = np.broadcast_to(mag, (m, H, d // 2, 2)).reshape(m, H, d)
            want.append(db.round_bf16(db.rope3d(v, t, yy, xx)))
            errs.append(pair_err(e) + 2.0 ** -20 * mag)
        else:
            want.append(db.round_bf16(v))
            errs.append(e)
    q, kk, v = (torch.empty((m, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    rtr.rtr_dit_qkv_rope(dev(a), dev(w), dev(b), m, D, H, d, k, gw, t0, q, kk, v)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    for name, got, ref, err in zip("qkv", (q, kk, v), want, errs):
        assert_parity(host_f64(got), ref, err, f"{name} H={H} d={d} m={m}")


def test_cases_cover_both_tilings():
    """The cases above reach both kernels: tiles of one CTA, and 256 x 256
    tiles shared by a CTA pair (as the Wan-1.3B feed-forward input and QKV
    projections are)."""
    rtr = _rtr()
    plans = {}
    for m, n, k, epi in LINEAR_CASES:
        code = "gated_residual" if epi.startswith("gated_residual") else epi
        plans[(m, n, k, epi)] = rtr.rtr_dit_linear_tile(m, n, k, code)
    for H, d, gh, gw, C, t0 in QKV_CASES:
        D = H * d
        plans[("qkv", H, d, C * gh * gw)] = rtr.rtr_dit_linear_tile(C * gh * gw, 3 * D, D, "bias", qkv_rope=True)
    for key, plan in plans.items():
        print(key, plan)
    pairs = [key for key, plan in plans.items() if plan[2] == 1]
    singles = [key for key, plan in plans.items() if plan[2] == 0]
    assert (4680, 8960, 1536, "gelu") in pairs and ("qkv", 12, 128, 4680) in pairs
    assert (4800, 4600, 1024, "bias") in pairs
    assert len(singles) >= 4
    for key in pairs:
        assert plans[key][:2] == (256, 256) and plans[key][3] % 2 == 0


def test_dit_linear_repeat_is_bit_identical():
    """Each output element is produced once by one CTA from a fixed K order:
    two calls give the same bits."""
    rtr = _rtr()
    m, n, k = 2000, 1536, 1536
    a, w, b = (dev(x) for x in _operands(np.random.default_rng(4), m, n, k))
    o1, o2 = (torch.empty((m, n), dtype=torch.bfloat16, device="cuda") for _ in range(2))
    rtr.rtr_dit_linear(a, w, m, n, k, "bias", b, None, o1)
    rtr.rtr_dit_linear(a, w, m, n, k, "bias", b, None, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
