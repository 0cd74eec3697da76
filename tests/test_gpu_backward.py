"""GPU parity of the block-causal attention backward (dQ, dK, dV) and of the
forward's row log-sum-exp, against the fp64 oracle on identical bf16 input
bits (papernotes.org note "DiT as Real-Time Rerenderer", Method > Key
Designs 2: the attention and its mask; Key Designs 3: training runs
gradient descent through it).

Tolerance of the gradients, per tensor: the attention's own bounds, max
|gpu - oracle| <= 2e-2 and relative L2 error <= 5e-3 (gpu_util.assert_close).
P and dS enter the tensor cores as bf16 (relative rounding 2^-9 each), the
forward's output O is bf16 (it enters Delta = rowsum(dO * O)), and the
results are rounded once to bf16 (2^-9); with fp32 accumulation these
independent roundings give a relative L2 error near 2.4e-3 and elements
within about 1e-3 of the oracle at the gradients' scale here (|dV| <= 0.4).
The row log-sum-exp (fp32, natural log) must be within 2e-3 absolute."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu

LSE_ABS = 2e-3


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


def assert_grad_close(got, want, what):
    """A gradient against the oracle at the attention's bounds."""
    return assert_close(got, want, what)


def run_gpu(q, k, v, do, n, H, d, kpf):
    """Forward with row LSE, then the backward, all through the C ABI."""
    rtr = _rtr()
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    out = torch.empty_like(tq)
    lse = torch.empty((H, n), dtype=torch.float32, device="cuda")
    rtr.rtr_attn_block_causal_prefill_lse(tq, tk, tv, n, H, d, kpf, "bf16", out, lse)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tq), torch.empty_like(tq)
    rtr.rtr_attn_block_causal_backward(tq, tk, tv, out, tdo, lse, n, H, d, kpf, "bf16", dq, dk, dv)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    return out, lse, dq, dk, dv


def bf16_inputs(n, H, d, seed):
    rng = np.random.default_rng(seed)
    q, k, v = (synth.normal(rng, (n, H, d), 0.5, "bf16") for _ in range(3))
    do = synth.normal(rng, (n, H, d), 1.0, "bf16")
    return q, k, v, do


CASES = [
    # n, H, d, k
    (300, 2, 128, 50),     # ragged last tile, frames inside tiles
    (256, 2, 128, 128),    # tile-aligned frames
    (1000, 2, 128, 160),   # several tiles, frames straddle tiles
    (700, 3, 64, 90),      # head_dim 64
    (17, 1, 128, 5),       # one partial tile
    (200, 1, 128, 1),      # k = 1: token-causal
    (200, 2, 128, 300),    # k >= n: bidirectional
]


@pytest.mark.parametrize("n,H,d,kpf", CASES, ids=lambda c: str(c))
def test_backward_parity(n, H, d, kpf):
    q, k, v, do = bf16_inputs(n, H, d, n + kpf)
    out, lse, dq, dk, dv = run_gpu(q, k, v, do, n, H, d, kpf)
    Q, K, V, dO = (oracle.decode(a, "bf16") for a in (q, k, v, do))
    assert_close(host_f64(out), oracle.prefill(Q, K, V, kpf), "forward output")
    want_lse = oracle.prefill_lse(Q, K, kpf)                       # [n, H]
    assert np.max(np.abs(lse.cpu().numpy().T.astype(np.float64) - want_lse)) <= LSE_ABS
    wq, wk, wv = oracle.prefill_backward(Q, K, V, dO, kpf)
    assert_grad_close(host_f64(dq), wq, "dQ")
    assert_grad_close(host_f64(dk), wk, "dK")
    assert_grad_close(host_f64(dv), wv, "dV")


def test_backward_zero_tokens_is_noop():
    rtr = _rtr()
    x = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    rtr.rtr_attn_block_causal_backward(x, x, x, x, x, lse, 0, 1, 128, 4, "bf16", x, x, x)


def test_backward_rejects_fp32():
    rtr = _rtr()
    x = torch.zeros((16, 1, 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(rtr.RtrError) as e:
        rtr.rtr_attn_block_causal_backward(x, x, x, x, x, lse, 16, 1, 64, 4, "f32", x, x, x)
    assert e.value.status == rtr.RTR_E_UNSUPPORTED


def test_full_prefill_backward_sampled():
    """The 22-frame prefill (34,320 tokens, 12 heads, k = 1560): dQ on sampled
    query rows and dK, dV on sampled key rows of two heads against the
    oracle; over all heads, sum_j dV_j = sum_i dO_i and sum_j dK_j = 0 (the
    softmax-Jacobian invariants) within bf16 rounding."""
    w = synth.PREFILL_22
    n, H, d, kpf = w.chunk_frames * w.k, w.heads, w.head_dim, w.k
    q, k, v, do = bf16_inputs(n, H, d, w.seed)
    out, lse, dq, dk, dv = run_gpu(q, k, v, do, n, H, d, kpf)
    heads = [0, 7]
    Q, K, V, dO = (oracle.decode(a[:, heads], "bf16") for a in (q, k, v, do))
    qrows = np.array(sorted({0, 1, 127, 128, 1559, 1560, 17000, 34319}
                            | set(np.random.default_rng(1).integers(0, n, 8).tolist())))
    krows = np.array(sorted({0, 127, 1559, 1560, 20000, 32760, 34319}
                            | set(np.random.default_rng(2).integers(0, n, 5).tolist())))
    wq = oracle.prefill_backward_query_rows(Q, K, V, dO, kpf, qrows)
    wk, wv = oracle.prefill_backward_key_rows(Q, K, V, dO, kpf, krows)
    assert_grad_close(host_f64(dq)[qrows][:, heads], wq, "dQ rows")
    assert_grad_close(host_f64(dk)[krows][:, heads], wk, "dK rows")
    assert_grad_close(host_f64(dv)[krows][:, heads], wv, "dV rows")
    gdv = dv.float().sum(dim=0).cpu().numpy()
    gdo = torch.from_numpy(oracle.decode(do, "bf16")).sum(dim=0).numpy()
    assert np.linalg.norm(gdv - gdo) <= 2e-2 * np.linalg.norm(gdo)
    gdk = dk.float().sum(dim=0).cpu().numpy()
    assert np.linalg.norm(gdk) <= 2e-2 * np.linalg.norm(dk.float().abs().sum(dim=0).cpu().numpy())


def test_backward_custom_scale():
    """A softmax scale other than 1/sqrt(d) reaches both the forward's row
    log-sum-exp and every gradient (dQ and dK carry it, dV through P)."""
    rtr = _rtr()
    n, H, d, kpf, scale = 333, 2, 128, 70, 0.05
    q, k, v, do = bf16_inputs(n, H, d, 99)
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    out = torch.empty_like(tq)
    lse = torch.empty((H, n), dtype=torch.float32, device="cuda")
    rtr.rtr_attn_block_causal_prefill_lse(tq, tk, tv, n, H, d, kpf, "bf16", out, lse, scale)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tq), torch.empty_like(tq)
    rtr.rtr_attn_block_causal_backward(tq, tk, tv, out, tdo, lse, n, H, d, kpf, "bf16", dq, dk, dv, scale)
    torch.cuda.synchronize()
    Q, K, V, dO = (oracle.decode(a, "bf16") for a in (q, k, v, do))
    assert np.max(np.abs(lse.cpu().numpy().T - oracle.prefill_lse(Q, K, kpf, scale=scale))) <= LSE_ABS
    wq, wk, wv = oracle.prefill_backward(Q, K, V, dO, kpf, scale=scale)
    assert_grad_close(host_f64(dq), wq, "dQ")
    assert_grad_close(host_f64(dk), wk, "dK")
    assert_grad_close(host_f64(dv), wv, "dV")


def test_backward_is_deterministic():
    """Every output tile is written once by one CTA (no atomics): two calls
    give bit-identical gradients."""
    rtr = _rtr()
    n, H, d, kpf = 500, 2, 128, 100
    q, k, v, do = bf16_inputs(n, H, d, 7)
    a = run_gpu(q, k, v, do, n, H, d, kpf)
    b = run_gpu(q, k, v, do, n, H, d, kpf)
    for x, y in zip(a[2:], b[2:]):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
