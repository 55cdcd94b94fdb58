"""rolling_kv_cache_sa_b200: per-chunk block-causal attention over a rolling
(sink + sliding window) KV cache with 3D RoPE, as a C-ABI CUDA library for
B200 (libsa.so) and its thin Python binding.

The library is loaded lazily on first use and must exist: there is no
fallback implementation.
"""
from ._lib import SAError, lib  # noqa: F401
from .cache import (  # noqa: F401
    SACache, attention_flops, config_for, make_config, sa_abi_version, sa_append_attend,
    sa_append_attend_host, sa_append_attend_noalloc, sa_cache_copy_out, sa_cache_create, sa_cache_destroy, sa_cache_reset,
    sa_get_device_status, sa_plan_chunk, sa_profile_begin, sa_profile_end, sa_profile_launches, sa_refresh_delta,
    sa_rope_refresh, sa_stream_state, sa_wait_probe, sa_attend, sa_cache_set_sink_mode,
    sa_sink_update, sa_append_attend_host_async, sa_host_wait, sa_cache_set_fp8_scales,
    sa_cache_export, sa_cache_import, sa_cache_get_fp8_scales, sa_noalloc_device_status,
)
from .gdn import (GDNState, gdn_workspace, sa_gdn_chunk, sa_gdn_device_status,  # noqa: F401
                  sa_gdn_workspace_size)
