"""CPU oracle for the SageSLA attention forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py`` may
import this package. The product path never does.
"""
from .sagesla_oracle import *  # noqa: F401,F403
from . import norm_oracle  # noqa: F401,E402
from . import w8a8_oracle  # noqa: F401,E402
from . import sla_backward_oracle  # noqa: F401,E402
