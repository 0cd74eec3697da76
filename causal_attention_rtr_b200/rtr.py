"""ctypes binding of librtr (``include/rtr.h``): one Python function per C
entry point, same names and argument order.  Argument marshalling only --
every step of the path runs in librtr's kernels.  Device buffers may be given
as torch tensors (their ``data_ptr()`` is passed) or as integers; streams as
``torch.cuda.Stream`` objects, raw handles or ``None`` (legacy default
stream).

Importing this module loads ``librtr.so`` and raises ``ImportError`` if it has
not been built: there is no fallback.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# RTR_LIBRARY selects another build of the same library (e.g. one compiled
# with different tuning macros); the default is the in-tree build.
LIB_PATH = os.environ.get("RTR_LIBRARY", os.path.join(_HERE, "librtr.so"))

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "librtr.so is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
        "or `python causal_attention_rtr_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

RTR_OK, RTR_E_INVAL, RTR_E_NOMEM, RTR_E_STATE, RTR_E_CUDA, RTR_E_TIMEOUT, RTR_E_UNSUPPORTED = range(7)
RTR_BF16, RTR_F32 = 0, 1
RTR_EPI_BIAS, RTR_EPI_BIAS_GELU, RTR_EPI_GATED_RESIDUAL = 0, 1, 2

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

class DitWeights(ctypes.Structure):
    """rtr_dit_weights of include/rtr.h: device pointers of one block's bf16
    weights ([in][out] row-major) and biases, and the feed-forward width."""
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("wqkv", "bqkv", "wo", "bo", "wq2", "bq2", "wo2", "bo2", "w1", "b1", "w2", "b2")] + \
               [("d_ffn", ctypes.c_int)]


# (name, restype, argtypes) for every symbol of include/rtr.h
_SIGNATURES = [
    ("rtr_status_string", ctypes.c_char_p, [_i]),
    ("rtr_build_info", ctypes.c_char_p, []),
    ("rtr_kvcache_create", _i, [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    ("rtr_kvcache_create_ex", _i, [_i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    ("rtr_kvcache_destroy", None, [_vp]),
    ("rtr_kvcache_set_reference", _i, [_vp, _i, _vp, _vp, _vp]),
    ("rtr_kvcache_clear_reference", _i, [_vp, _i]),
    ("rtr_kvcache_append_frame", _i, [_vp, _i, _vp, _vp, _i, _vp]),
    ("rtr_kvcache_retain_last", _i, [_vp, _i, _i]),
    ("rtr_kvcache_get_index_map", _i, [_vp, _i, ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int32)]),
    ("rtr_kvcache_device_ptrs", _i, [_vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    ("rtr_kvcache_set_index_map", _i, [_vp, _i, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]),
    ("rtr_kvcache_check_guards", _i, [_vp]),
    ("rtr_crossattn_check_guards", _i, [_vp]),
    ("rtr_test_fail_allocs", _i, [_i, _i]),
    ("rtr_attn_frame_causal", _i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _f, _vp]),
    ("rtr_attn_frame_causal_ex", _i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _f, _i, _vp]),
    ("rtr_attn_frame_causal_f32out", _i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _f, _vp]),
    ("rtr_attn_frame_causal_commit", _i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _f, _vp]),
    ("rtr_attn_block_causal_prefill", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _i, _vp]),
    ("rtr_attn_block_causal_prefill_ex", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _i, _i, _vp]),
    ("rtr_attn_block_causal_prefill_noalloc", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _i, _vp]),
    ("rtr_attn_block_causal_prefill_lse", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _f, _i, _vp]),
    ("rtr_dit_block_forward", _i, [_vp, _vp, _i, ctypes.POINTER(DitWeights), _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    ("rtr_attn_block_causal_prefill_cache", _i, [_vp, _i, _vp, _vp, _vp, _i, _i, _vp, _f, _vp]),
    ("rtr_dit_pack_weights", _i, [ctypes.POINTER(DitWeights), _i, _i, _vp, ctypes.POINTER(_vp)]),
    ("rtr_dit_packed_destroy", None, [_vp]),
    ("rtr_dit_block_forward_packed", _i, [_vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    ("rtr_dit_linear", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp]),
    ("rtr_dit_qkv_rope", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp]),
    ("rtr_dit_linear_tile", _i, [_i, _i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                                 ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    ("rtr_dit_plan_tile", _i, [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                               ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    ("rtr_attn_block_causal_backward", _i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _f,
                                            _i, _vp]),
    ("rtr_crossattn_create", _i, [_i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    ("rtr_crossattn_destroy", None, [_vp]),
    ("rtr_crossattn_set_text", _i, [_vp, _i, _vp, _vp, _i, _vp]),
    ("rtr_crossattn_reset", _i, [_vp]),
    ("rtr_attn_cross", _i, [_vp, _i, _vp, _i, _vp, _f, _vp]),
    ("rtr_get_device_status", _i, [_i, _vp]),
    ("rtr_test_inject_wait_timeout", _i, [_i, _i]),
    ("rtr_kernel_launches", ctypes.c_ulonglong, []),
    ("rtr_release_workspaces", _i, [_i, ctypes.POINTER(_i)]),
]

for _name, _res, _args in _SIGNATURES:
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = [s[0] for s in _SIGNATURES]


class RtrError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {rtr_status_string(status)}")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, ctypes.c_void_p):
        return x.value
    raise TypeError(f"cannot pass {type(x).__name__} as a device pointer")


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    raise TypeError("stream must be None, an int handle or a torch.cuda.Stream")


def _check(st, where):
    if st != RTR_OK:
        raise RtrError(st, where)
    return st


def _dtype(dt):
    if dt in ("bf16", RTR_BF16):
        return RTR_BF16
    if dt in ("f32", RTR_F32):
        return RTR_F32
    raise ValueError("dtype must be 'bf16' or 'f32'")


# ---------------------------------------------------------------- raw calls
def rtr_status_string(status):
    return _lib.rtr_status_string(int(status)).decode()


def rtr_build_info():
    return _lib.rtr_build_info().decode()


def rtr_kvcache_create(layers, heads, head_dim, k, ref_frames, window_frames, dt, device):
    h = _vp()
    _check(_lib.rtr_kvcache_create(layers, heads, head_dim, k, ref_frames, window_frames, _dtype(dt),
                                   device, ctypes.byref(h)), "rtr_kvcache_create")
    return h.value


def rtr_kvcache_create_ex(layers, heads, head_dim, k, ref_frames, window_frames, commit_frames, dt, device):
    h = _vp()
    _check(_lib.rtr_kvcache_create_ex(layers, heads, head_dim, k, ref_frames, window_frames, commit_frames,
                                      _dtype(dt), device, ctypes.byref(h)), "rtr_kvcache_create_ex")
    return h.value


def rtr_kvcache_destroy(c):
    _lib.rtr_kvcache_destroy(c)


def rtr_kvcache_set_reference(c, layer, k_ref, v_ref, stream=None):
    return _check(_lib.rtr_kvcache_set_reference(c, layer, _ptr(k_ref), _ptr(v_ref), _stream(stream)),
                  "rtr_kvcache_set_reference")


def rtr_kvcache_clear_reference(c, layer=-1):
    return _check(_lib.rtr_kvcache_clear_reference(c, layer), "rtr_kvcache_clear_reference")


def rtr_kvcache_append_frame(c, layer, k_new, v_new, n_frames, stream=None):
    return _check(_lib.rtr_kvcache_append_frame(c, layer, _ptr(k_new), _ptr(v_new), n_frames,
                                                _stream(stream)), "rtr_kvcache_append_frame")


def rtr_kvcache_retain_last(c, layer, n_frames):
    return _check(_lib.rtr_kvcache_retain_last(c, layer, n_frames), "rtr_kvcache_retain_last")


def rtr_kvcache_get_index_map(c, layer, n_slots):
    """Returns (slot_frame list, ref_valid, frames_appended, count).  n_slots:
    the cache's physical window slots (window_frames + commit_frames)."""
    slots = (ctypes.c_int32 * n_slots)()
    ref = ctypes.c_int32()
    g = ctypes.c_int64()
    cnt = ctypes.c_int32()
    _check(_lib.rtr_kvcache_get_index_map(c, layer, slots, ctypes.byref(ref), ctypes.byref(g),
                                          ctypes.byref(cnt)), "rtr_kvcache_get_index_map")
    return list(slots), ref.value, g.value, cnt.value


def rtr_kvcache_set_index_map(c, layer, frames_appended, count, ref_valid):
    return _check(_lib.rtr_kvcache_set_index_map(c, layer, int(frames_appended), int(count), int(ref_valid)),
                  "rtr_kvcache_set_index_map")


def rtr_kvcache_check_guards(c):
    return _check(_lib.rtr_kvcache_check_guards(c), "rtr_kvcache_check_guards")


def rtr_crossattn_check_guards(x):
    return _check(_lib.rtr_crossattn_check_guards(x), "rtr_crossattn_check_guards")


def rtr_test_fail_allocs(after, n):
    return _check(_lib.rtr_test_fail_allocs(int(after), int(n)), "rtr_test_fail_allocs")


def rtr_kvcache_device_ptrs(c, layer):
    k, v = _vp(), _vp()
    _check(_lib.rtr_kvcache_device_ptrs(c, layer, ctypes.byref(k), ctypes.byref(v)), "rtr_kvcache_device_ptrs")
    return k.value, v.value


def rtr_attn_frame_causal(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale=0.0, stream=None):
    return _check(_lib.rtr_attn_frame_causal(c, layer, _ptr(q), _ptr(k_cur), _ptr(v_cur), n_cur_frames,
                                             _ptr(out), float(scale), _stream(stream)), "rtr_attn_frame_causal")


def rtr_attn_frame_causal_ex(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale=0.0, cta_group=1, stream=None):
    return _check(_lib.rtr_attn_frame_causal_ex(c, layer, _ptr(q), _ptr(k_cur), _ptr(v_cur), n_cur_frames,
                                                _ptr(out), float(scale), cta_group, _stream(stream)),
                  "rtr_attn_frame_causal_ex")


def rtr_attn_frame_causal_f32out(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale=0.0, stream=None):
    """rtr_attn_frame_causal with an fp32 output tensor (the rows before the
    bf16 rounding)."""
    return _check(_lib.rtr_attn_frame_causal_f32out(c, layer, _ptr(q), _ptr(k_cur), _ptr(v_cur), n_cur_frames,
                                                    _ptr(out), float(scale), _stream(stream)),
                  "rtr_attn_frame_causal_f32out")


def rtr_attn_frame_causal_commit(c, layer, q, k_cur, v_cur, n_cur_frames, out, scale=0.0, stream=None):
    return _check(_lib.rtr_attn_frame_causal_commit(c, layer, _ptr(q), _ptr(k_cur), _ptr(v_cur), n_cur_frames,
                                                    _ptr(out), float(scale), _stream(stream)),
                  "rtr_attn_frame_causal_commit")


def rtr_attn_block_causal_prefill_lse(q, k, v, n_tokens, heads, head_dim, k_per_frame, dt, out, lse, scale=0.0,
                                      device=0, stream=None):
    return _check(_lib.rtr_attn_block_causal_prefill_lse(_ptr(q), _ptr(k), _ptr(v), n_tokens, heads, head_dim,
                                                         k_per_frame, _dtype(dt), _ptr(out), _ptr(lse),
                                                         float(scale), device, _stream(stream)),
                  "rtr_attn_block_causal_prefill_lse")


def rtr_attn_block_causal_prefill_cache(c, layer, q, k, v, n_frames, with_reference, out, scale=0.0, stream=None):
    return _check(_lib.rtr_attn_block_causal_prefill_cache(c, layer, _ptr(q), _ptr(k), _ptr(v), n_frames,
                                                           1 if with_reference else 0, _ptr(out), float(scale),
                                                           _stream(stream)),
                  "rtr_attn_block_causal_prefill_cache")


def dit_weights(weights, d_ffn):
    """DitWeights from a mapping of the twelve names to device buffers."""
    return DitWeights(*[_ptr(weights[f[0]]) for f in DitWeights._fields_[:-1]], int(d_ffn))


def rtr_dit_block_forward(c, x, layer, weights, modulation, hidden, n_cur_frames, grid_h, grid_w, t0, commit=False,
                          stream=None):
    """``weights``: a DitWeights, or a mapping of its twelve names to device
    buffers plus "d_ffn"."""
    w = weights if isinstance(weights, DitWeights) else dit_weights(weights, weights["d_ffn"])
    return _check(_lib.rtr_dit_block_forward(c, x, layer, ctypes.byref(w), _ptr(modulation), _ptr(hidden),
                                             n_cur_frames, grid_h, grid_w, t0, 1 if commit else 0,
                                             _stream(stream)),
                  "rtr_dit_block_forward")


def rtr_dit_pack_weights(weights, d_model, device=0, stream=None):
    """Pack a block's weights once (see include/rtr.h); returns the handle."""
    w = weights if isinstance(weights, DitWeights) else dit_weights(weights, weights["d_ffn"])
    h = _vp()
    _check(_lib.rtr_dit_pack_weights(ctypes.byref(w), d_model, device, _stream(stream), ctypes.byref(h)),
           "rtr_dit_pack_weights")
    return h.value


def rtr_dit_packed_destroy(pw):
    _lib.rtr_dit_packed_destroy(pw)


def rtr_dit_block_forward_packed(c, x, layer, pw, modulation, hidden, n_cur_frames, grid_h, grid_w, t0, commit=False,
                                 stream=None):
    return _check(_lib.rtr_dit_block_forward_packed(c, x, layer, pw, _ptr(modulation), _ptr(hidden), n_cur_frames,
                                                    grid_h, grid_w, t0, int(bool(commit)), _stream(stream)),
                  "rtr_dit_block_forward_packed")


def _epilogue(epilogue):
    return int({"bias": RTR_EPI_BIAS, "gelu": RTR_EPI_BIAS_GELU,
                "gated_residual": RTR_EPI_GATED_RESIDUAL}.get(epilogue, epilogue))


def rtr_dit_linear(a, w, m, n, k, epilogue, bias, gate, out, device=0, stream=None):
    """out = epilogue(a w + bias) on the tensor cores (see include/rtr.h)."""
    return _check(_lib.rtr_dit_linear(_ptr(a), _ptr(w), m, n, k, _epilogue(epilogue), _ptr(bias), _ptr(gate),
                                      _ptr(out), device, _stream(stream)), "rtr_dit_linear")


def rtr_dit_qkv_rope(a, wqkv, bqkv, m, d_in, heads, head_dim, k_per_frame, grid_w, t0, q, k, v, device=0,
                     stream=None):
    """q, k, v = thirds of a wqkv + bqkv, q and k rotary-encoded (see include/rtr.h)."""
    return _check(_lib.rtr_dit_qkv_rope(_ptr(a), _ptr(wqkv), _ptr(bqkv), m, d_in, heads, head_dim, k_per_frame,
                                        grid_w, t0, _ptr(q), _ptr(k), _ptr(v), device, _stream(stream)),
                  "rtr_dit_qkv_rope")


def rtr_dit_linear_tile(m, n, k, epilogue, qkv_rope=False, device=0):
    """(rows, cols, cta_pair, ctas) of the tile the projection picks and its
    launch's CTAs (see include/rtr.h)."""
    rows, cols, pair, ctas = _i(), _i(), _i(), _i()
    _check(_lib.rtr_dit_linear_tile(m, n, k, _epilogue(epilogue), int(bool(qkv_rope)), device, ctypes.byref(rows),
                                    ctypes.byref(cols), ctypes.byref(pair), ctypes.byref(ctas)),
           "rtr_dit_linear_tile")
    return rows.value, cols.value, pair.value, ctas.value


def rtr_dit_plan_tile(m, n, k, epilogue, qkv_rope=False, w_packed=False, sms=148, pair_clusters=74):
    """(rows, cols, cta_pair, ctas) the projection planner picks for a
    hypothetical device (host arithmetic only; see include/rtr.h)."""
    rows, cols, pair, ctas = _i(), _i(), _i(), _i()
    _check(_lib.rtr_dit_plan_tile(m, n, k, _epilogue(epilogue), int(bool(qkv_rope)), int(bool(w_packed)), sms,
                                  pair_clusters, ctypes.byref(rows), ctypes.byref(cols), ctypes.byref(pair),
                                  ctypes.byref(ctas)), "rtr_dit_plan_tile")
    return rows.value, cols.value, pair.value, ctas.value


def rtr_attn_block_causal_backward(q, k, v, out, dout, lse, n_tokens, heads, head_dim, k_per_frame, dt, dq, dk, dv,
                                   scale=0.0, device=0, stream=None):
    return _check(_lib.rtr_attn_block_causal_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                                      n_tokens, heads, head_dim, k_per_frame, _dtype(dt), _ptr(dq),
                                                      _ptr(dk), _ptr(dv), float(scale), device, _stream(stream)),
                  "rtr_attn_block_causal_backward")


def rtr_attn_block_causal_prefill(q, k, v, n_tokens, heads, head_dim, k_per_frame, dt, out, scale=0.0,
                                  device=0, stream=None):
    return _check(_lib.rtr_attn_block_causal_prefill(_ptr(q), _ptr(k), _ptr(v), n_tokens, heads, head_dim,
                                                     k_per_frame, _dtype(dt), _ptr(out), float(scale),
                                                     device, _stream(stream)),
                  "rtr_attn_block_causal_prefill")


def rtr_attn_block_causal_prefill_ex(q, k, v, n_tokens, heads, head_dim, k_per_frame, dt, out, scale=0.0,
                                     cta_group=1, device=0, stream=None):
    return _check(_lib.rtr_attn_block_causal_prefill_ex(_ptr(q), _ptr(k), _ptr(v), n_tokens, heads, head_dim,
                                                        k_per_frame, _dtype(dt), _ptr(out), float(scale),
                                                        cta_group, device, _stream(stream)),
                  "rtr_attn_block_causal_prefill_ex")


def rtr_attn_block_causal_prefill_noalloc(q, k, v, n_tokens, heads, head_dim, k_per_frame, dt, out, scale=0.0,
                                          device=0, stream=None):
    """Same as rtr_attn_block_causal_prefill, with its scratch in the
    library's static device array instead of a buffer it allocates (for
    callers that cannot allocate device memory)."""
    return _check(_lib.rtr_attn_block_causal_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), n_tokens, heads,
                                                             head_dim, k_per_frame, _dtype(dt), _ptr(out),
                                                             float(scale), device, _stream(stream)),
                  "rtr_attn_block_causal_prefill_noalloc")


def rtr_crossattn_create(layers, heads, head_dim, max_text, dt, device):
    h = _vp()
    _check(_lib.rtr_crossattn_create(layers, heads, head_dim, max_text, _dtype(dt), device, ctypes.byref(h)),
           "rtr_crossattn_create")
    return h.value


def rtr_crossattn_destroy(x):
    _lib.rtr_crossattn_destroy(x)


def rtr_crossattn_set_text(x, layer, k_text, v_text, n_text, stream=None):
    return _check(_lib.rtr_crossattn_set_text(x, layer, _ptr(k_text), _ptr(v_text), n_text, _stream(stream)),
                  "rtr_crossattn_set_text")


def rtr_crossattn_reset(x):
    return _check(_lib.rtr_crossattn_reset(x), "rtr_crossattn_reset")


def rtr_attn_cross(x, layer, q, n_q, out, scale=0.0, stream=None):
    return _check(_lib.rtr_attn_cross(x, layer, _ptr(q), n_q, _ptr(out), float(scale), _stream(stream)),
                  "rtr_attn_cross")


def rtr_get_device_status(device=0, stream=None):
    """Latched device-side status (RTR_OK or RTR_E_TIMEOUT); clears it."""
    return _lib.rtr_get_device_status(device, _stream(stream))


def raw_status(fn_name, *args):
    """Call a C entry point and return its status without raising (tests of
    the error paths)."""
    return getattr(_lib, fn_name)(*args)


def rtr_test_inject_wait_timeout(device, launches):
    """Test hook: the next `launches` bf16 attention launches on `device`
    issue no loads, so their bounded waits expire and RTR_E_TIMEOUT is
    latched (see include/rtr.h)."""
    return _check(_lib.rtr_test_inject_wait_timeout(device, launches), "rtr_test_inject_wait_timeout")


def rtr_kernel_launches():
    """Kernels this library has launched since it was loaded."""
    return int(_lib.rtr_kernel_launches())


def rtr_release_workspaces(device=0):
    """Free the library's per-stream scratch buffers of `device`; returns
    how many it held."""
    n = _i(0)
    _check(_lib.rtr_release_workspaces(device, ctypes.byref(n)), "rtr_release_workspaces")
    return n.value
