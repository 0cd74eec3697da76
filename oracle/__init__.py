"""fp64 CPU oracle for RTR-DiT's frame-causal attention and its
reference-preserving rolling KV cache.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with ``causal_attention_rtr_b200`` and does not
import it; the two meet only in the seeded input generators, which hold none
of the method's arithmetic.

Sources (all on the papernotes.org note "DiT as Real-Time Rerenderer:
Streaming Video Stylization with Autoregressive Diffusion Transformer"):

* Method > Key Designs 2 -- the attention equation
  softmax(QK^T/sqrt(d) + M)V with M_ij = 0 iff floor(j/k) <= floor(i/k).
* Method > Key Designs 4 -- the rolling KV cache with the reference tokens
  anchored in a resident slot at the front, the oldest frames evicted, the
  cross-attention cache reinitialised on a condition switch while the 3D cache
  keeps the most recent frame.
* Method > Key Designs 1 -- the reference latent is one extra latent frame in
  front of the first frame; TV2V has no reference (c = {empty, c_text}).
* Method > Key Designs 3 -- training (Self Forcing, DMD) runs gradient descent
  through the block-causal attention; ``backward.py`` holds its plain
  derivative.
* Method > Overall Architecture and Key Designs 1 -- the DiT block around the
  attention (``dit_block.py``: modulated layer norms, projections, 3D rotary
  encoding, cross attention to the text, feed-forward), with the readings the
  pages leave open stated there.

Every function here is the plain definition; see ``attention.py``,
``cache.py`` and ``backward.py``.  Parity pins live in ``tests/test_oracle_*.py``.
"""
from .attention import (attention, prefill, visible, decode, max_threads,
                        library_path)
from .cache import ReferenceCache, CrossCache
from .backward import (prefill_lse, prefill_backward, prefill_backward_key_rows,
                       prefill_backward_query_rows)
from . import dit_block

__all__ = ["attention", "prefill", "visible", "decode", "max_threads",
           "library_path", "ReferenceCache", "CrossCache", "prefill_lse",
           "prefill_backward", "prefill_backward_key_rows",
           "prefill_backward_query_rows", "dit_block"]
