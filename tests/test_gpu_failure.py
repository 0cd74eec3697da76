"""GPU: failure detection without a GPU fault.  Every mbarrier wait in the
tensor-core attention kernel is bounded; when a launch's inputs never arrive
(the test hook makes the producer issue no loads) the waits expire after about
a second, the kernel frees its tensor memory and returns, and the host reads
RTR_E_TIMEOUT from the latched device status.  The context stays usable: the
next launch is correct."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_rtr_b200 import synth

from gpu_util import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_recoverable():
    from causal_attention_rtr_b200 import rtr
    n, H, d, k = 600, 2, 128, 100
    q, kk, v = synth.random_qkv(42, n, H, d, "bf16")
    Q, K, V = dev(q), dev(kk), dev(v)
    out = torch.empty((n, H, d), dtype=torch.bfloat16, device="cuda")
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    rtr.rtr_test_inject_wait_timeout(0, 1)
    rtr.rtr_attn_block_causal_prefill(Q, K, V, n, H, d, k, "bf16", out)
    assert rtr.rtr_get_device_status(0) == rtr.RTR_E_TIMEOUT
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK          # read clears it
    rtr.rtr_attn_block_causal_prefill(Q, K, V, n, H, d, k, "bf16", out)
    torch.cuda.synchronize()
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
    want = oracle.prefill(*(oracle.decode(x, "bf16") for x in (q, kk, v)), k)
    assert_close(host_f64(out), want, "after timeout")
