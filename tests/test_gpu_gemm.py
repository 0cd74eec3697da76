"""GPU parity of the DiT block's tensor-core projections with their fused
epilogues (rtr_dit_linear, rtr_dit_qkv_rope) against the block oracle's own
steps (oracle/dit_block.py: fp64 products of the same bf16 operands, the
bias / GELU / gated residual / 3D rotary encoding in fp64, one rounding to
bf16; papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
Architecture).

Tolerance: both sides round the same quantity once to bf16, the GPU from an
fp32 accumulation and the oracle from fp64.  The two unrounded values differ
by far less than a bf16 unit in the last place (fp32 sums over at most 8960
exact bf16 products, fp32 sin / cos of angles below 100 rad), so the rounded
results are equal or, where the two straddle a rounding boundary, one bf16
ulp apart: every element must be within one ulp of the oracle."""
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


def assert_within_one_ulp(got, want, what):
    assert np.all(np.isfinite(got)), what
    bound = _ulp(np.maximum(np.abs(got), np.abs(want)))
    worst = float(np.max(np.abs(got - want) / bound))
    frac_diff = float(np.mean(got != want))
    assert worst <= 1.0, f"{what}: worst |diff| / ulp = {worst:.3f}"
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
]


@pytest.mark.parametrize("m,n,k,epi", LINEAR_CASES, ids=lambda c: str(c))
def test_dit_linear_parity(m, n, k, epi):
    rtr = _rtr()
    rng = np.random.default_rng(m + n + k)
    a, w, b = _operands(rng, m, n, k)
    A, Wt, B = decode(a, "bf16"), decode(w, "bf16"), decode(b, "bf16")
    C = A @ Wt + B
    gate = None
    if epi.startswith("gated_residual"):
        x = synth.normal(rng, (m, n), 1.0, "bf16")
        X = decode(x, "bf16")
        if epi == "gated_residual":
            gate = synth.normal(rng, (n,), 0.5, "bf16")
            want = db.round_bf16(X + decode(gate, "bf16") * C)
        else:
            want = db.round_bf16(X + C)
        out = dev(x)
        code = "gated_residual"
    elif epi == "gelu":
        want = db.round_bf16(db.gelu_tanh(C))
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        code = "gelu"
    else:
        want = db.round_bf16(C)
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        code = "bias"
    rtr.rtr_dit_linear(dev(a), dev(w), m, n, k, code, dev(b), None if gate is None else dev(gate), out)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    worst, frac = assert_within_one_ulp(host_f64(out), want, f"{epi} m={m} n={n} k={k}")
    print(f"{epi} m={m} n={n} k={k}: worst/ulp={worst:.3f} differing={frac:.2e}")


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
    qkv = decode(a, "bf16") @ decode(w, "bf16") + decode(b, "bf16")
    t, yy, xx = db.token_positions(C, gh, gw, t0)
    want = [db.round_bf16(db.rope3d(qkv[:, :D].reshape(m, H, d), t, yy, xx)),
            db.round_bf16(db.rope3d(qkv[:, D:2 * D].reshape(m, H, d), t, yy, xx)),
            db.round_bf16(qkv[:, 2 * D:].reshape(m, H, d))]
    q, kk, v = (torch.empty((m, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    rtr.rtr_dit_qkv_rope(dev(a), dev(w), dev(b), m, D, H, d, k, gw, t0, q, kk, v)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    for name, got, ref in zip("qkv", (q, kk, v), want):
        worst, frac = assert_within_one_ulp(host_f64(got), ref, f"{name} H={H} d={d} m={m}")
        print(f"qkv {name} H={H} d={d} m={m}: worst/ulp={worst:.3f} differing={frac:.2e}")


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
