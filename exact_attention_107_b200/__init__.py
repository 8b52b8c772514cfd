"""exact_attention_107_b200 -- exact, IO-aware tiled attention for NVIDIA B200 (sm_100a).

The compute lives in libfa.so (hand-written CUDA for sm_100a behind the C ABI
of include/fa.h); this package only marshals torch tensors into that ABI.
Importing the package does not load the library; the first call does, and it
fails loudly if libfa.so has not been built.
"""
from ._binding import (  # noqa: F401
    LIB_PATH,
    SYMBOLS,
    FAError,
    FlashAttention,
    HostStepPipeline,
    attention_backward,
    attention_forward,
    attention_fwd_bwd_from_host,
    default_scale,
    fa_bwd,
    fa_bwd_f16,
    fa_bwd_deterministic,
    fa_bwd_deterministic_workspace_size,
    fa_bwd_dkdv,
    fa_bwd_dkdvdq,
    fa_bwd_dq,
    fa_bwd_dq_finish,
    fa_bwd_noalloc,
    fa_bwd_preprocess,
    fa_bwd_workspace_size,
    fa_device_status,
    fa_fwd,
    fa_fwd_f16,
    fa_fwd_f32,
    fa_version,
    flash_attention,
    load_library,
    status_string,
    workspace_views,
)

from .shard import head_ranges, shard_view, sharded_attention, sharded_attention_devices  # noqa: F401,E402

__version__ = "2.0.0"
