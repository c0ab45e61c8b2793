"""CPU oracle for the Kascade hot path -- test infrastructure only.

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The product library never does.
"""
from .kascade_oracle import *  # noqa: F401,F403
from .kascade_oracle import __all__  # noqa: F401
