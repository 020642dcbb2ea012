"""B200 (sm_100a) implementation of HTTM's head-wise temporal token merging
around a VGGT-style global-attention layer, behind the C ABI of
``include/httm.h``.  Importing the package does not load the CUDA library;
the first call does, and fails loudly if it is missing."""
from .binding import (  # noqa: F401
    EXPORTS,
    HTTM_CONTIGUOUS,
    HTTM_DENSE,
    HTTM_HEAD_UNIFORM,
    HTTM_HEADWISE_TEMPORAL,
    HTTM_PARTITION,
    HttmError,
    TorchExchange,
    LayerConfig,
    Plan,
    debug_buffers,
    httm_forward,
    httm_forward_debug,
    httm_forward_reuse,
    httm_forward_sharded,
    httm_forward_with_plan,
    httm_get_device_status,
    httm_plan,
    httm_plan_partition,
    httm_reorder,
    httm_set_fused_unmerge,
    httm_set_wait_budget,
    load_library,
    workspace_view,
)
