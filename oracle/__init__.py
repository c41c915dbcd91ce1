"""Test infrastructure: the float64 CPU oracle of the Wan DiT forward.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` and ``--impl reference`` legs) may import this package.  The
product path (the CUDA library and its Python binding) never does.
"""
from . import wan_oracle  # noqa: F401
