"""Test infrastructure: the float64 CPU oracles of the Wan DiT forward
(``wan_oracle``) and of the Wan2.1 VAE decoder (``wan_vae``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` and ``--impl reference`` legs) may import this package.  The
product path (the CUDA library and its Python binding) never does.
"""
from . import wan_oracle, wan_vae  # noqa: F401
