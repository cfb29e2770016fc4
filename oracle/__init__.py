"""CPU oracle for the NSA / MoBA forward and decode (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this package; the library never does.
"""
from .nsa_oracle import *  # noqa: F401,F403
from .dsa_oracle import dsa_forward, indexer_scores, select_tokens  # noqa: F401
