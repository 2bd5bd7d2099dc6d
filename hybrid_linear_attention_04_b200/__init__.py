"""KDA (Kimi Delta Attention) hot path for NVIDIA B200: libkda + its binding.

The computation lives in libkda.so (CUDA, sm_100a), built in-tree by
``hybrid_linear_attention_04_b200.build``; ``kda`` is the ctypes binding with
the C ABI's names (include/kda.h).
"""
from .kda import (KDAError, kda_check_device_status, kda_decode, kda_launch_count, kda_prefill,
                  kda_snapshot, kda_snapshot_plan, kda_status_string, kda_verify, lib)

__all__ = ["KDAError", "kda_check_device_status", "kda_decode", "kda_launch_count", "kda_prefill",
           "kda_snapshot", "kda_snapshot_plan", "kda_status_string", "kda_verify", "lib"]
