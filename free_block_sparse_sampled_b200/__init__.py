"""SparsePR attention call on B200 (sm_100a): C ABI library + thin binding.

The library (libsparsepr.so, built from csrc/ by ``build.py``) implements the
whole call in CUDA; this package only marshals arguments.
"""

from .api import (HostPipeline, SparsePRConfig, alloc_workspace, apply, attention, call, device_status,  # noqa: F401
                  partition, probe_fit, probe_fit_static, route, validate, workspace_bytes)
from ._abi import EXPORTED, LIB_PATH, SparsePRError, lib  # noqa: F401
