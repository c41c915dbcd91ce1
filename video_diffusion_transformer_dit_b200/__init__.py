"""B200-native (sm_100a) Wan DiT denoising-step forward.

The product is ``libwandit.so`` (C ABI declared in ``include/wandit.h``); this
package holds its CUDA sources (``csrc/``), the build step, the thin ctypes
binding (``binding``), model presets (``configs``) and the seeded synthetic
input generator (``synth``).  Importing the package loads nothing; the binding
loads the library on first use and raises if it is missing.
"""
__all__ = ["configs", "synth", "binding"]
