"""B200 (sm_100a) library for FlashPrefill V2's mean-corrected block-sparse causal prefill attention.

The compute lives in libfp2.so (C ABI in include/fp2.h); ``fp2`` is its ctypes binding.
"""

from . import fp2  # noqa: F401
from .fp2 import (FP2Error, fp2_attend, fp2_discover, fp2_discover_static, fp2_get_device_status,  # noqa: F401
                  fp2_last_error,
                  fp2_pool, fp2_prefill, fp2_version, fp2_workspace_query, fp2_workspace_size, load_library,
                  make_params,
                  make_problem)
