"""GPU: the library's per-stream scratch buffers stay bounded.  Calls on many
short-lived streams keep at most 8 buffers per device (the least recently
used is freed), rtr_release_workspaces frees them on request, and calls
after a release allocate again and give the same results."""
import pytest
import torch

from causal_attention_rtr_b200 import synth

from gpu_util import dev

pytestmark = pytest.mark.gpu


def test_stream_workspaces_are_capped_and_released():
    from causal_attention_rtr_b200 import rtr
    n, H, d, k = 3000, 4, 128, 300          # fewer units than SMs: split units use the scratch
    q, kk, v = (dev(x) for x in synth.random_qkv(5, n, H, d, "bf16", 0.5))
    want = torch.empty_like(q)
    rtr.rtr_attn_block_causal_prefill(q, kk, v, n, H, d, k, "bf16", want)
    torch.cuda.synchronize()
    outs = []
    for _ in range(12):                     # twelve streams, each used once and dropped
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        out = torch.empty_like(q)
        rtr.rtr_attn_block_causal_prefill(q, kk, v, n, H, d, k, "bf16", out, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        outs.append(out)
    torch.cuda.synchronize()
    for out in outs:
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    held = rtr.rtr_release_workspaces(0)
    assert 1 <= held <= 8
    assert rtr.rtr_release_workspaces(0) == 0
    again = torch.empty_like(q)
    rtr.rtr_attn_block_causal_prefill(q, kk, v, n, H, d, k, "bf16", again)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), want.view(torch.int16))
    assert rtr.rtr_get_device_status(0) == rtr.RTR_OK
