"""Plain fp64 CPU oracle for mean-corrected block-sparse causal prefill attention.

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  It shares no code with the
CUDA library and never imports it.
"""

from .fp2_oracle import *  # noqa: F401,F403
