"""B200-native (sm_100a) Multi-head Latent Attention decode.

The public entry points are those of include/mla_decode.h, bound in
``mla_decode_attention_11_b200.binding``; the CUDA library is loaded on
first use (and built in-tree if missing).
"""
from .binding import (MlaError, alloc_workspace, load_library, mla_decode, mla_decode_check,  # noqa: F401
                         mla_decode_host, mla_decode_plan, mla_decode_plan_batch_invariant, mla_decode_run, mla_decode_run_noalloc, mha_decode_plan, mha_decode_run,
                         mla_decode_run_sinks, mla_decode_plan_fp8, mla_decode_run_fp8,
                         mla_decode_set_debug,
                         mla_decode_workspace_init, mla_plan, status_string)
