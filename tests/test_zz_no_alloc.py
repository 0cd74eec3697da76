"""GPU: rtr_attn_block_causal_prefill_noalloc, the prefill variant for
callers that cannot allocate device memory (its scratch is a static device
array), returns what rtr_attn_block_causal_prefill returns, within the
attention tolerance, on two calls in a row through the C ABI.

The shapes split attention units across SMs, so the static scratch is
written and read; the second call uses new inputs, so a stale partial result
left by the first call would show.  This file is collected last and works
both alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,H,k", [(3000, 4, 300),       # fewer units than SMs: every unit split
                                   (10000, 8, 1560)])    # full rounds plus a split remainder
def test_noalloc_prefill_matches_allocating_prefill(n, H, k):
    from causal_attention_rtr_b200 import rtr
    d = 128
    for call in range(2):
        q, kk, v = synth.random_qkv(1000 * call + n, n, H, d, "bf16", 0.5)
        Q, K, V = dev(q), dev(kk), dev(v)
        want = torch.empty((n, H, d), dtype=torch.bfloat16, device="cuda")
        got = torch.empty_like(want)
        rtr.rtr_attn_block_causal_prefill(Q, K, V, n, H, d, k, "bf16", want)
        rtr.rtr_attn_block_causal_prefill_noalloc(Q, K, V, n, H, d, k, "bf16", got)
        torch.cuda.synchronize()
        assert_close(host_f64(got), host_f64(want), f"noalloc call {call}")
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
