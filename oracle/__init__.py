"""CPU oracle for the QSA decode step (test infrastructure, not the product).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference arms may import this package.
"""

from .qsa_oracle import *  # noqa: F401,F403
