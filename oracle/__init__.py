"""CPU oracle for KVSlimmer asymmetric KV merging (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package. The product path never does.
"""
from .kvslimmer_oracle import *  # noqa: F401,F403
