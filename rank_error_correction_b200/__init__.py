"""B200-native GlowQ corrected quantised linear layer.

The compute path lives in the CUDA library ``libglowq.so`` (built from
``csrc/``) behind the C ABI declared in ``include/glowq.h``; ``glowq`` is its
thin Python binding.  ``synth`` draws the seeded synthetic inputs.

Submodules are imported lazily so that importing the package needs neither a
GPU nor the built library.
"""
__all__ = ["glowq", "synth"]
__version__ = "0.1.0"
