"""CPU checks of the C-ABI library: it builds, loads without a GPU, exports
every function ``include/rtr.h`` declares, the Python binding covers exactly
those names, and argument validation answers before any device work."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rtr.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rtr_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from causal_attention_rtr_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("rtr_kvcache_create", "rtr_kvcache_set_reference", "rtr_kvcache_append_frame",
                     "rtr_attn_frame_causal", "rtr_attn_block_causal_prefill", "rtr_crossattn_set_text",
                     "rtr_crossattn_reset"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    handle, path = lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        getattr(handle, n)


def test_binding_matches_header(lib):
    from causal_attention_rtr_b200 import rtr
    assert sorted(rtr.EXPORTED) == declared_functions()
    for n in rtr.EXPORTED:
        assert callable(getattr(rtr, n))


def test_status_strings(lib):
    from causal_attention_rtr_b200 import rtr
    assert rtr.rtr_status_string(rtr.RTR_OK) == "RTR_OK"
    assert "invalid" in rtr.rtr_status_string(rtr.RTR_E_INVAL)
    assert "sm_100a" in rtr.rtr_build_info()


def test_validation_before_device_work(lib):
    """Bad shapes are rejected on the host, so these answer without a GPU."""
    from causal_attention_rtr_b200 import rtr
    h = ctypes.c_void_p()
    bad = [
        (0, 2, 128, 16, 1, 4, 0, 0),      # layers
        (1, 0, 128, 16, 1, 4, 0, 0),      # heads
        (1, 2, 96, 16, 1, 4, 0, 0),       # head_dim not 64/128
        (1, 2, 128, 0, 1, 4, 0, 0),       # k
        (1, 2, 128, 16, -1, 4, 0, 0),     # ref_frames
        (1, 2, 128, 16, 1, 0, 0, 0),      # window_frames
        (1, 2, 128, 16, 1, 4, 7, 0),      # dtype
        (1, 2, 128, 16, 1, 4, 0, -1),     # device
    ]
    for args in bad:
        st = rtr.raw_status("rtr_kvcache_create", *args, ctypes.byref(h))
        assert st == rtr.RTR_E_INVAL, args
        assert h.value is None
    assert rtr.raw_status("rtr_kvcache_create", 1, 2, 128, 16, 1, 4, 0, 0, None) == rtr.RTR_E_INVAL
    # commit room: 0 <= commit_frames <= window_frames
    for commit in (-1, 5):
        st = rtr.raw_status("rtr_kvcache_create_ex", 1, 2, 128, 16, 1, 4, commit, 0, 0, ctypes.byref(h))
        assert st == rtr.RTR_E_INVAL, commit
        assert h.value is None
    assert rtr.raw_status("rtr_attn_frame_causal_commit", None, 0, None, None, None, 1, None, 0.0,
                          None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_attn_block_causal_prefill_cache", None, 0, None, None, None, 1, 1, None, 0.0,
                          None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_block_forward", None, None, 0, None, None, None, 1, 1, 1, 0, 0,
                          None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_kvcache_set_index_map", None, 0, 0, 0, 0) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_kvcache_check_guards", None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_crossattn_check_guards", None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_test_fail_allocs", -1, 0) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_test_fail_allocs", 0, 0) == rtr.RTR_OK
    # null handles
    assert rtr.raw_status("rtr_kvcache_append_frame", None, 0, None, None, 1, None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_attn_frame_causal", None, 0, None, None, None, 1, None, 0.0, None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_kvcache_retain_last", None, 0, 1) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_crossattn_reset", None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_attn_cross", None, 0, None, 1, None, 0.0, None) == rtr.RTR_E_INVAL
    # prefill: bad shapes, and n_tokens == 0 is a no-op
    assert rtr.raw_status("rtr_attn_block_causal_prefill", None, None, None, 10, 2, 100, 4, 0, None, 0.0, 0,
                          None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_attn_block_causal_prefill", None, None, None, 0, 2, 128, 4, 0, None, 0.0, 0,
                          None) == rtr.RTR_OK
    assert rtr.raw_status("rtr_attn_block_causal_prefill", 16, 16, 16, 10, 2, 128, 0, 0, 16, 0.0, 0,
                          None) == rtr.RTR_E_INVAL


def test_explicit_cta_group_and_workspace_validation(lib):
    """The MMA form is an explicit argument (1 or 2); anything else is
    rejected before any device work, as is a negative device for the
    scratch release."""
    from causal_attention_rtr_b200 import rtr
    for cg in (0, 3, -1):
        assert rtr.raw_status("rtr_attn_block_causal_prefill_ex", 16, 16, 16, 10, 2, 128, 4, 0, 16, 0.0, cg, 0,
                              None) == rtr.RTR_E_INVAL, cg
        assert rtr.raw_status("rtr_attn_frame_causal_ex", None, 0, None, None, None, 1, None, 0.0, cg,
                              None) == rtr.RTR_E_INVAL, cg
    assert rtr.raw_status("rtr_attn_block_causal_prefill_ex", None, None, None, 0, 2, 128, 4, 0, None, 0.0, 2, 0,
                          None) == rtr.RTR_OK
    assert rtr.raw_status("rtr_release_workspaces", -1, None) == rtr.RTR_E_INVAL


def test_dit_projection_validation(lib):
    """The fused projections check shapes, epilogue and alignment on the
    host (no GPU needed)."""
    from causal_attention_rtr_b200 import rtr
    p = 256
    bad_linear = [
        (p, p, 10, 12, 64, 0, p, None, p, 0, None),     # n not a multiple of 8
        (p, p, 10, 64, 4, 0, p, None, p, 0, None),      # k < 8
        (p, p, -1, 64, 64, 0, p, None, p, 0, None),     # m < 0
        (p, p, 10, 64, 64, 7, p, None, p, 0, None),     # no such epilogue
        (p, p, 10, 64, 64, 0, p, p, p, 0, None),        # gate with the plain bias epilogue
        (p + 2, p, 10, 64, 64, 0, p, None, p, 0, None), # a not 16-byte aligned
        (p, p, 10, 64, 64, 0, p, None, p, -1, None),    # device
    ]
    for args in bad_linear:
        assert rtr.raw_status("rtr_dit_linear", *args) == rtr.RTR_E_INVAL, args
    assert rtr.raw_status("rtr_dit_linear", p, p, 0, 64, 64, 2, p, p, p, 0, None) == rtr.RTR_OK
    bad_qkv = [
        (p, p, p, 10, 64, 2, 96, 16, 4, 0, p, p, p, 0, None),    # head_dim
        (p, p, p, 10, 60, 2, 64, 16, 4, 0, p, p, p, 0, None),    # d_in not a multiple of 8
        (p, p, p, 10, 64, 2, 64, 0, 4, 0, p, p, p, 0, None),     # k_per_frame
        (p, p, p, 10, 64, 2, 64, 16, 0, 0, p, p, p, 0, None),    # grid_w
        (p, p, p, 10, 64, 2, 64, 16, 4, -1, p, p, p, 0, None),   # t0
        (p, p, p, 10, 64, 2, 64, 16, 4, 0, p + 8, p, p, 0, None),  # q not 16-byte aligned
    ]
    for args in bad_qkv:
        assert rtr.raw_status("rtr_dit_qkv_rope", *args) == rtr.RTR_E_INVAL, args
    assert rtr.raw_status("rtr_dit_qkv_rope", p, p, p, 0, 64, 2, 64, 16, 4, 0, p, p, p, 0, None) == rtr.RTR_OK


def test_dit_packed_validation(lib):
    """Packing checks its shape and pointers on the host (no GPU needed)."""
    import ctypes as ct
    from causal_attention_rtr_b200 import rtr
    w = rtr.DitWeights(*([256] * 12), 512)
    h = ct.c_void_p()
    for d_model in (0, 96, 100):
        assert rtr.raw_status("rtr_dit_pack_weights", ct.byref(w), d_model, 0, None, ct.byref(h)) == rtr.RTR_E_INVAL
        assert h.value is None
    w_bad_ffn = rtr.DitWeights(*([256] * 12), 200)            # d_ffn not a multiple of 64
    assert rtr.raw_status("rtr_dit_pack_weights", ct.byref(w_bad_ffn), 128, 0, None, ct.byref(h)) == rtr.RTR_E_INVAL
    w_misaligned = rtr.DitWeights(*([256] * 11 + [258]), 512)
    assert rtr.raw_status("rtr_dit_pack_weights", ct.byref(w_misaligned), 128, 0, None,
                          ct.byref(h)) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_pack_weights", ct.byref(w), 128, -1, None, ct.byref(h)) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_pack_weights", ct.byref(w), 128, 0, None, None) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_block_forward_packed", None, None, 0, None, None, None, 1, 1, 1, 0, 0,
                          None) == rtr.RTR_E_INVAL
    rtr.rtr_dit_packed_destroy(None)                          # no-op


def test_dit_linear_tile_plan_on_host(lib):
    """The projection's tile planner answers without a GPU: without a device
    it plans for 148 SMs and single-CTA tiles (no CTA pairs, whose residency
    it cannot query); shapes and pointers are checked first."""
    import ctypes as ct
    import torch
    from causal_attention_rtr_b200 import rtr
    if torch.cuda.is_available():
        pytest.skip("a device is present: the plan is the device's (tests/test_gpu_gemm.py)")
    for m, n, k, epi, qkv in [(4680, 8960, 1536, "gelu", False), (4680, 1536, 8960, "gated_residual", False),
                              (4680, 4608, 1536, "bias", True), (7, 64, 8, "bias", False)]:
        rows, cols, pair, ctas = rtr.rtr_dit_linear_tile(m, n, k, epi, qkv)
        assert pair == 0 and rows in (128, 256) and cols in (128, 192, 256)
        tiles = -(-m // rows) * -(-n // cols)
        assert ctas == min(tiles, 148), (m, n, k, rows, cols, ctas)
    r = [ct.c_int() for _ in range(4)]
    refs = [ct.byref(x) for x in r]
    assert rtr.raw_status("rtr_dit_linear_tile", 0, 64, 64, 0, 0, 0, *refs) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_linear_tile", 64, 64, 64, 7, 0, 0, *refs) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_linear_tile", 64, 64, 64, 0, 0, -1, *refs) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_linear_tile", 64, 64, 64, 0, 0, 0, refs[0], refs[1], None, refs[3]) == rtr.RTR_E_INVAL


# The six projections of a Wan-1.3B-shaped block on its 3-frame chunk
# (4680 tokens, D = 1536, FFN 8960): name, m, n, k, epilogue, qkv_rope.
WAN13_PROJECTIONS = [("qkv", 4680, 4608, 1536, "bias", True), ("out", 4680, 1536, 1536, "gated_residual", False),
                     ("cross_q", 4680, 1536, 1536, "bias", False),
                     ("cross_out", 4680, 1536, 1536, "gated_residual", False),
                     ("ffn_in", 4680, 8960, 1536, "gelu", False), ("ffn_out", 4680, 1536, 8960, "gated_residual", False)]


def test_projection_planner_for_a_b200(lib):
    """The planner's choices for a B200 (148 SMs, 74 resident CTA pairs), as
    measured on the Wan-1.3B block: with packed weights every projection
    takes 256 x 256 CTA-pair tiles; with row-major weights (8 KB boxes, more
    TMA instructions) the 1,536-wide ones keep 256 x 256 tiles of one CTA.
    Without pairs the planner never picks one; a pair launch takes an even
    number of CTAs, never more than the SMs."""
    from causal_attention_rtr_b200 import rtr
    for name, m, n, k, epi, qkv in WAN13_PROJECTIONS:
        assert rtr.rtr_dit_plan_tile(m, n, k, epi, qkv, True) == (256, 256, 1, 148), name
        plan = rtr.rtr_dit_plan_tile(m, n, k, epi, qkv, False)
        want_pair = name in ("qkv", "ffn_in")
        assert plan[2] == int(want_pair), (name, plan)
        if not want_pair:
            assert plan == (256, 256, 0, 114), (name, plan)
        for packed in (True, False):
            rows, cols, pair, ctas = rtr.rtr_dit_plan_tile(m, n, k, epi, qkv, packed, 148, 0)
            assert pair == 0 and ctas <= 148, (name, packed)
    for m, n, k in [(7, 64, 8), (300, 200, 72), (20000, 8960, 1536), (1560, 5120, 5120)]:
        for packed in (True, False):
            rows, cols, pair, ctas = rtr.rtr_dit_plan_tile(m, n, k, "bias", False, packed, 148, 74)
            tiles = -(-m // rows) * -(-n // cols)
            assert ctas <= 148 and (not pair or (ctas % 2 == 0 and rows == 256 and cols == 256))
            assert ctas == min(tiles, 74 if pair else 148) * (2 if pair else 1)


def test_projection_planner_validation(lib):
    import ctypes as ct
    from causal_attention_rtr_b200 import rtr
    r = [ct.c_int() for _ in range(4)]
    refs = [ct.byref(x) for x in r]
    for args in [(0, 64, 64, 0, 0, 0, 148, 74), (64, 64, 64, 0, 0, 0, 0, 0), (64, 64, 64, 0, 0, 0, 148, 75),
                 (64, 64, 64, 0, 0, 0, 148, -1), (64, 64, 64, 3, 0, 0, 148, 74)]:
        assert rtr.raw_status("rtr_dit_plan_tile", *args, *refs) == rtr.RTR_E_INVAL, args
    assert rtr.raw_status("rtr_dit_plan_tile", 64, 64, 64, 0, 0, 0, 148, 74, refs[0], None, refs[2],
                          refs[3]) == rtr.RTR_E_INVAL
    assert rtr.raw_status("rtr_dit_plan_tile", 64, 64, 64, 0, 0, 0, 148, 74, *refs) == rtr.RTR_OK
