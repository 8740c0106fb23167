"""CPU oracle of the DiT-block denoising path: test infrastructure only.

Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg import it.
"""
from . import oracle  # noqa: F401
