"""Test infrastructure: the CPU oracle for the rotate-then-quantize int4 codec.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  The product never does.
"""

from .kvq_oracle import *  # noqa: F401,F403
from .kvq_oracle import __all__  # noqa: F401
