"""B200-native Kimi Delta Attention (KDA) mixer: chunked prefill and decode step.

The compute runs in ``libkda_b200.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/kda.h``); this package only marshals arguments to it.  The
binding is imported lazily so that ``workloads`` (input generation) is usable
without a GPU; every compute entry point raises if the CUDA library is missing.
"""
from __future__ import annotations

__all__ = ["kda_prefill", "kda_decode_step", "kda_prefill_workspace_size",
           "kda_status_string", "library_path", "KdaError", "kda_prefill_kernel_count",
           "kda_device_status", "kda_prefill_noalloc", "kda_prefill_checkpointed",
           "kda_checkpoint_count", "kda_decode_multi", "kda_prefill_segments",
           "kda_prefill_debug", "kda_decode_check_slots"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
