"""Reference-preserving rolling KV cache and cross-attention cache, as plain
state machines over numpy arrays (test infrastructure; see package doc).

Source: "DiT as Real-Time Rerenderer" (papernotes note), Method > Key
Designs 4, and Key Designs 1 for the reference frame:

* Fixed-length caches are set up for the 3D attention and for the cross
  attention.  New frames are appended; once the cache is full the oldest
  frames are evicted.
* The reference tokens sit in a resident slot at the front that eviction never
  touches, so every later frame can still attend to them.
* On a switch of text prompt or reference image the cross-attention cache is
  reinitialised, the 3D cache keeps only the most recent frame, and a new
  reference image is anchored at the front.
* The reference latent counts as one latent frame placed before the first
  frame; TV2V carries no reference.

Readings where the pages are silent:
* the window W counts past frames only; the chunk being generated attends to
  [reference | window | chunk] and is appended afterwards;
* "keeps the most recent frame" is ``retain_last(1)``: the window shrinks to
  its newest frame;
* eviction is by whole latent frames, oldest first;
* without a reference (TV2V) the reference span is simply absent.

Physical placement (a layout choice of this library, not of the pages): the
window ring may have more physical slots than the W frames it holds
(``slots`` >= W).  Frame f lives in slot f mod slots; which frames are held,
and so the attention, does not depend on ``slots``.  The extra slots are
where a chunk can be written while the W frames it attends to stay intact.

Stored data are the caller's raw bits (uint16 bfloat16 patterns or float32),
copied exactly.  A slot holds the bytes last written to it; the bytes of an
invalid slot are unspecified and never compared.
"""
import numpy as np

from .attention import attention, decode


class ReferenceCache:
    """One layer of the 3D-attention cache.

    State: ``ref_valid``; ``g`` = frames appended since creation; ``count`` =
    frames currently held (<= W); ``slots_k/v[s]`` = data of the frame f with
    f mod S == s, S = ``slots`` physical slots (W unless given).  Slot s holds
    a valid frame f iff g - count <= f < g.  Every tensor is [tokens, H, d].
    """

    def __init__(self, heads, head_dim, k, ref_frames, window_frames, dtype, slots=None):
        slots = window_frames if slots is None else slots
        if min(heads, head_dim, k, window_frames) <= 0 or ref_frames < 0 or slots < window_frames:
            raise ValueError("bad cache shape")
        self.H, self.d, self.k = heads, head_dim, k
        self.R, self.W = ref_frames, window_frames
        self.S = slots
        self.dtype = dtype
        raw = np.uint16 if dtype == "bf16" else np.float32
        self._raw = raw
        self.ref_k = np.zeros((ref_frames * k, heads, head_dim), raw)
        self.ref_v = np.zeros_like(self.ref_k)
        self.slots_k = [np.zeros((k, heads, head_dim), raw) for _ in range(slots)]
        self.slots_v = [np.zeros((k, heads, head_dim), raw) for _ in range(slots)]
        self.ref_valid = False
        self.g = 0
        self.count = 0

    # -- updates -----------------------------------------------------------
    def set_reference(self, k_ref, v_ref):
        """Anchor (or overwrite in place) the reference slot; window untouched."""
        shape = (self.R * self.k, self.H, self.d)
        if self.R == 0:
            raise ValueError("cache was created without a reference slot")
        k_ref = np.asarray(k_ref, self._raw).reshape(shape)
        v_ref = np.asarray(v_ref, self._raw).reshape(shape)
        self.ref_k = k_ref.copy()
        self.ref_v = v_ref.copy()
        self.ref_valid = True

    def clear_reference(self):
        """TV2V: no reference condition, so the reference span is absent."""
        self.ref_valid = False

    def append(self, k_new, v_new, n_frames):
        """Append n frames: frame f goes to slot f mod S; once the window is
        full the oldest frames drop out of it (= eviction; with S == W the
        new frame overwrites the evicted one's slot)."""
        if not 1 <= n_frames <= self.W:
            raise ValueError("n_frames must be in [1, W]")
        k_new = np.asarray(k_new, self._raw).reshape(n_frames, self.k, self.H, self.d)
        v_new = np.asarray(v_new, self._raw).reshape(n_frames, self.k, self.H, self.d)
        for i in range(n_frames):
            f = self.g + i
            s = f % self.S
            self.slots_k[s] = k_new[i].copy()
            self.slots_v[s] = v_new[i].copy()
        self.g += n_frames
        self.count = min(self.W, self.count + n_frames)

    def retain_last(self, r):
        """Condition switch: keep only the r most recent frames (r = 1 on the
        page)."""
        if r < 0:
            raise ValueError("r must be >= 0")
        self.count = min(self.count, r)

    # -- views -------------------------------------------------------------
    def window_frames(self):
        """Global indices of the held frames, oldest first."""
        return list(range(self.g - self.count, self.g))

    def index_map(self):
        """(slot_frame[S] with -1 for empty, ref_valid, g)."""
        slot_frame = [-1] * self.S
        for f in self.window_frames():
            slot_frame[f % self.S] = f
        return slot_frame, int(self.ref_valid), self.g

    def logical_kv(self):
        """Raw K, V of the cached logical sequence [reference | window frames
        oldest -> newest], each [n, H, d]."""
        ks, vs = [], []
        if self.ref_valid:
            ks.append(self.ref_k)
            vs.append(self.ref_v)
        for f in self.window_frames():
            ks.append(self.slots_k[f % self.S])
            vs.append(self.slots_v[f % self.S])
        empty = np.zeros((0, self.H, self.d), self._raw)
        K = np.concatenate(ks, axis=0) if ks else empty
        V = np.concatenate(vs, axis=0) if vs else empty
        return K, V

    def chunk_first_frame(self):
        """Logical frame index of the first frame of the chunk being
        generated: R (if a reference is held) + count."""
        return (self.R if self.ref_valid else 0) + self.count

    def stream_attention(self, q, k_cur, v_cur, n_cur_frames, rows=None,
                         scale=None, nthreads=0):
        """Attention of the current chunk's queries against
        [reference | window | chunk] under the frame-causal mask.

        q, k_cur, v_cur: raw [n_cur*k, H, d].  Chunk row i sits at logical
        position chunk_first_frame()*k + i; cached keys come first in logical
        order, so every cached key is in an earlier frame than every query and
        chunk frames see chunk frames up to their own.  ``rows`` selects query
        rows.  Returns fp64 [len(rows), H, d].
        """
        Q, pos, K, V = self.stream_operands(q, k_cur, v_cur, n_cur_frames)
        rows = np.arange(Q.shape[0], dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
        return attention(Q[rows], pos[rows], K, V, self.k, True, scale, nthreads)

    def stream_operands(self, q, k_cur, v_cur, n_cur_frames):
        """The decoded operands of ``stream_attention``: queries [nc, H, d],
        their logical positions [nc], and the logical keys and values
        [reference | window | chunk], all fp64."""
        nc = n_cur_frames * self.k
        shape = (nc, self.H, self.d)
        q = np.asarray(q).reshape(shape)
        k_cur = np.asarray(k_cur).reshape(shape)
        v_cur = np.asarray(v_cur).reshape(shape)
        Kc, Vc = self.logical_kv()
        K = decode(np.concatenate([Kc, k_cur], axis=0), self.dtype)
        V = decode(np.concatenate([Vc, v_cur], axis=0), self.dtype)
        pos = self.chunk_first_frame() * self.k + np.arange(nc, dtype=np.int64)
        return decode(q, self.dtype), pos, K, V


class CrossCache:
    """One layer of the cross-attention (text) cache: fixed capacity
    ``max_text`` tokens, filled by ``set_text``, invalidated by ``reset``."""

    def __init__(self, heads, head_dim, max_text, dtype):
        self.H, self.d, self.max_text, self.dtype = heads, head_dim, max_text, dtype
        raw = np.uint16 if dtype == "bf16" else np.float32
        self._raw = raw
        self.k = np.zeros((max_text, heads, head_dim), raw)
        self.v = np.zeros_like(self.k)
        self.n_text = 0

    def set_text(self, k_text, v_text, n_text):
        if not 1 <= n_text <= self.max_text:
            raise ValueError("n_text must be in [1, max_text]")
        shape = (n_text, self.H, self.d)
        self.k[:n_text] = np.asarray(k_text, self._raw).reshape(shape)
        self.v[:n_text] = np.asarray(v_text, self._raw).reshape(shape)
        self.n_text = n_text

    def reset(self):
        self.n_text = 0

    def attention(self, q, rows=None, scale=None, nthreads=0):
        """Unmasked softmax attention of q [n, H, d] against the text keys."""
        if self.n_text == 0:
            raise RuntimeError("cross-attention cache is empty (reset)")
        q = np.asarray(q)
        rows = np.arange(q.shape[0], dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
        K = decode(self.k[:self.n_text], self.dtype)
        V = decode(self.v[:self.n_text], self.dtype)
        return attention(decode(q[rows], self.dtype), np.zeros(len(rows), np.int64),
                         K, V, 1, False, scale, nthreads)
