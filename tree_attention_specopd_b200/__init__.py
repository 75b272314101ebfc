"""SpecOPD branch-scoring hot path for NVIDIA B200 (sm_100a).

The work runs in the CUDA kernels of ``libspecopd.so`` behind the C ABI of
``include/specopd.h``; ``api`` is the thin ctypes binding (same names).
"""

from . import api  # noqa: F401
from .api import (  # noqa: F401
    SpecopdError,
    specopd_e2e_tv,
    specopd_e2e_tv_lmhead,
    specopd_e2e_tv_lmhead_workspace_size,
    specopd_e2e_tv_workspace_size,
    specopd_get_device_status,
    specopd_rope_apply,
    specopd_tree_attn,
    specopd_tree_attn_workspace_size,
    specopd_tree_build,
)
