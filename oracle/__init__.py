"""Plain CPU oracle for the SVDQuant W4A4 / AWQ W4A16 layers.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference arm of ``bench.py`` may import this package.  The
CUDA library never calls it and shares no code with it; the two meet only
through the seeded input generators in ``workloads/``.
"""
from . import awq, formats, svdq  # noqa: F401
