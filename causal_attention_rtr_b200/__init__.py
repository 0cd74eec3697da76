"""B200-native (sm_100a) frame-causal attention with a reference-preserving
rolling KV cache, after RTR-DiT ("DiT as Real-Time Rerenderer: Streaming
Video Stylization with Autoregressive Diffusion Transformer").

The work runs in ``librtr.so`` (hand-written CUDA behind a C ABI declared in
``include/rtr.h``).  ``causal_attention_rtr_b200.rtr`` is a thin ctypes
binding with the same names; it only marshals arguments.  ``synth`` draws the
seeded synthetic inputs.
"""
__all__ = ["rtr", "synth"]


def __getattr__(name):
    # Lazy: importing the package does not load the CUDA library.
    if name in __all__:
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
