"""GPU: the CTA-pair variant of the tensor-core attention (tcgen05
cta_group::2: one MMA covers 256 query rows on two SMs, each SM holding half
of every key / value tile) gives the same results as the oracle.  It is
selected by the cta_group argument of the _ex entry points; the default
single-CTA kernel was measured faster, so this path is kept covered here."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,H,k", [(700, 2, 100), (1300, 3, 1), (2600, 2, 600)])
def test_cta_pair_prefill_parity(n, H, k):
    from causal_attention_rtr_b200 import rtr
    d = 128
    q, kk, v = synth.random_qkv(n + 7 * k, n, H, d, "bf16")
    out = torch.empty((n, H, d), dtype=torch.bfloat16, device="cuda")
    rtr.rtr_attn_block_causal_prefill_ex(dev(q), dev(kk), dev(v), n, H, d, k, "bf16", out, cta_group=2)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    want = oracle.prefill(*(oracle.decode(x, "bf16") for x in (q, kk, v)), k)
    assert_close(host_f64(out), want, f"pair prefill n={n} k={k}")


def test_cta_pair_stream_parity():
    from causal_attention_rtr_b200 import rtr
    H, d, k, W, C = 4, 128, 300, 4, 2
    rng = np.random.default_rng(8)
    c = rtr.rtr_kvcache_create(1, H, d, k, 1, W, "bf16", 0)
    o = oracle.ReferenceCache(H, d, k, 1, W, "bf16")
    try:
        kr, vr = (synth.normal(rng, (k, H, d), 1.0, "bf16") for _ in range(2))
        rtr.rtr_kvcache_set_reference(c, 0, dev(kr), dev(vr))
        o.set_reference(kr, vr)
        for _ in range(3):
            kn, vn = (synth.normal(rng, (2 * k, H, d), 1.0, "bf16") for _ in range(2))
            rtr.rtr_kvcache_append_frame(c, 0, dev(kn), dev(vn), 2)
            o.append(kn, vn, 2)
        q, kc, vc = (synth.normal(rng, (C * k, H, d), 1.0, "bf16") for _ in range(3))
        out = torch.empty((C * k, H, d), dtype=torch.bfloat16, device="cuda")
        rtr.rtr_attn_frame_causal_ex(c, 0, dev(q), dev(kc), dev(vc), C, out, cta_group=2)
        torch.cuda.synchronize()
        assert_close(host_f64(out), o.stream_attention(q, kc, vc, C), "pair stream")
    finally:
        rtr.rtr_kvcache_destroy(c)
