"""CPU oracle for the GPTQ layer solver (test infrastructure only).

Only the test suite, the smoke check in ``__graft_entry__`` and the CPU
baseline leg of ``bench.py`` may import this package; the GPU library and its
Python binding never do.
"""
from .gptq_oracle import *  # noqa: F401,F403
from .gptq_oracle import __all__  # noqa: F401
