"""fp64 CPU oracle of the LLaMA pre-norm decoder block.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs, never by the CUDA library.
"""

from . import block  # noqa: F401
