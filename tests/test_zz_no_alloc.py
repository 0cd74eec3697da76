"""GPU: rtr_attn_block_causal_prefill_noalloc, the prefill for callers that
cannot let a library allocate device memory (its scratch is a static device
array), through the C ABI.

Each case makes two calls in a row with different inputs and checks both
against the fp64 oracle at the attention tolerance, and bit for bit against
rtr_attn_block_causal_prefill on the same inputs: both entry points plan and
launch the same kernels, so a stale partial result left in the shared array
by the first call, or a merge that reads the wrong part, shows as a
difference.  The first shape splits attention units across SMs, so the
static scratch is written and read; head_dim 64 and the fp32 path (which
needs no scratch) are covered too.  A separate test checks that a call allocates
nothing (device free memory is unchanged across it) and that bad arguments
are rejected.

This file is collected last and works both alone in a fresh process and
after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


def _rtr():
    from causal_attention_rtr_b200 import rtr
    return rtr


CASES = [
    # n, H, d, k, dtype, oracle rows (None: all)
    (3000, 4, 128, 300, "bf16", None),       # fewer units than SMs: the long ones split over CTAs
    (10000, 8, 128, 1560, "bf16", 48),       # two full rounds, then whole remainder units; sampled rows
    (2000, 3, 64, 250, "bf16", None),        # head_dim 64
    (600, 2, 64, 100, "f32", None),          # fp32 storage: the CUDA-core kernel, no scratch
]


@pytest.mark.parametrize("n,H,d,kpf,dt,sample", CASES, ids=lambda c: str(c))
def test_noalloc_prefill_parity(n, H, d, kpf, dt, sample):
    rtr = _rtr()
    scale_in = 0.5 if dt == "bf16" else 1.0
    for call in range(2):
        q, kk, v = synth.random_qkv(1000 * call + n + d, n, H, d, dt, scale_in)
        Q, K, V = dev(q), dev(kk), dev(v)
        got = torch.empty_like(Q)
        want = torch.empty_like(Q)
        rtr.rtr_attn_block_causal_prefill_noalloc(Q, K, V, n, H, d, kpf, dt, got)
        rtr.rtr_attn_block_causal_prefill(Q, K, V, n, H, d, kpf, dt, want)
        torch.cuda.synchronize()
        assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
        # the allocating entry point, bit for bit
        assert torch.equal(got.view(torch.int16) if dt == "bf16" else got.view(torch.int32),
                           want.view(torch.int16) if dt == "bf16" else want.view(torch.int32)), f"call {call}"
        # the oracle, at the attention tolerance
        rows = None
        if sample:
            rng = np.random.default_rng(call)
            rows = np.array(sorted({0, 1, kpf - 1, kpf, n - 1} | set(rng.integers(0, n, sample).tolist())))
        ref = oracle.prefill(*(oracle.decode(x, dt) for x in (q, kk, v)), kpf, rows=rows)
        g = host_f64(got)
        assert_close(g if rows is None else g[rows], ref, f"noalloc {dt} call {call}")


def test_noalloc_prefill_allocates_nothing():
    """Device free memory is unchanged across a call (after a first call on
    the same shapes has loaded the kernels), and again across a second one."""
    rtr = _rtr()
    n, H, d, kpf = 6000, 6, 128, 800
    q, kk, v = synth.random_qkv(17, n, H, d, "bf16", 0.5)
    Q, K, V = dev(q), dev(kk), dev(v)
    out = torch.empty_like(Q)
    rtr.rtr_attn_block_causal_prefill_noalloc(Q, K, V, n, H, d, kpf, "bf16", out)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        rtr.rtr_attn_block_causal_prefill_noalloc(Q, K, V, n, H, d, kpf, "bf16", out)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK


def test_noalloc_prefill_rejects_bad_arguments():
    rtr = _rtr()
    x = torch.zeros((64, 2, 128), dtype=torch.bfloat16, device="cuda")
    ptr = x.data_ptr()
    for args in [(ptr, ptr, ptr, 64, 2, 96, 16, 0, ptr, 0.0, 0, None),       # head_dim not 64 / 128
                 (ptr, ptr, ptr, 64, 0, 128, 16, 0, ptr, 0.0, 0, None),      # no heads
                 (ptr, ptr, ptr, 64, 2, 128, 0, 0, ptr, 0.0, 0, None),       # k_per_frame
                 (ptr + 2, ptr, ptr, 64, 2, 128, 16, 0, ptr, 0.0, 0, None),  # q not 16-byte aligned
                 (ptr, ptr, ptr, 64, 2, 128, 16, 5, ptr, 0.0, 0, None)]:     # element type
        assert rtr.raw_status("rtr_attn_block_causal_prefill_noalloc", *args) == rtr.RTR_E_INVAL, args
    assert rtr.raw_status("rtr_attn_block_causal_prefill_noalloc", ptr, ptr, ptr, 0, 2, 128, 16, 0, ptr, 0.0, 0,
                          None) == rtr.RTR_OK                                # no tokens: nothing to do
