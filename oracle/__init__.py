"""CPU oracle (test infrastructure only; see ``oracle.sgqa_oracle``).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does.
"""
from .sgqa_oracle import *  # noqa: F401,F403
