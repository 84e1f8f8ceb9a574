"""CPU oracle for the Mustafar hot path.

Test infrastructure only: ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it.  The CUDA library never does.
"""
from .mustafar_oracle import *  # noqa: F401,F403
