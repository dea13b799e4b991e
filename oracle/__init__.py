"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline /
reference arm may import this package.  The CUDA library and its binding
never import it, and it imports nothing from them.

Every function is pinned by ``tests/test_oracle.py`` (decode:
``tests/test_oracle_decode.py``) against invariants,
closed forms, finite differences, a float64 library routine and brute-force
loops; no function here is "parity unpinned".
"""
from .attention import *  # noqa: F401,F403
from .attention import __all__ as _attn_all
from .decode import *  # noqa: F401,F403
from .decode import __all__ as _decode_all

__all__ = list(_attn_all) + list(_decode_all)
