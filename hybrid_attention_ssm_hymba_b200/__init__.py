"""B200-native (sm_100a) forward (prefill) pass of Hymba's hybrid-head layer.

The product is the CUDA library ``libhymba.so`` behind the C ABI in
``include/hymba.h``; this package is its thin Python binding (``_abi``: same
names as the C entry points, argument marshalling only), the in-place build
step (``build``), host-side upload helpers (``host``) and the seeded synthetic
workloads (``synth``).  Importing the package does not load the library; the
first entry-point call does, and raises if it is missing.
"""
from ._abi import (ENTRY_POINTS, HYMBA_BF16, HYMBA_ERR_CUDA, HYMBA_ERR_INVALID_ARG,  # noqa: F401
                   HYMBA_ERR_TIMEOUT, HYMBA_ERR_UNSUPPORTED, HYMBA_ERR_WORKSPACE, HYMBA_F32,
                   HYMBA_KV_CONSUME, HYMBA_KV_OWN, HYMBA_KV_PRODUCE, HYMBA_OK, HymbaError, LIB_PATH,
                   check, hymba_attention, hymba_check_wait_timeout, hymba_decode_workspace_size,
                   hymba_layer_decode, hymba_layer_prefill, hymba_meta_prefix_size, hymba_meta_prefix,
                   hymba_layer_fwd_prefixed, hymba_branch_norm, hymba_cfg_t, hymba_gemm,
                   hymba_layer_fuses_dt_proj, hymba_layer_fwd, hymba_layer_fwd_events, hymba_layer_fwd_noalloc,
                   HYMBA_NOALLOC_SCRATCH_BYTES, hymba_rmsnorm, hymba_selective_scan, hymba_selective_scan_dtproj,
                   hymba_selective_scan_dtproj_workspace_size, hymba_stack_fwd,
                   hymba_stack_workspace_size, hymba_status_string, hymba_weights_t,
                   hymba_workspace_size, hymba_workspace_status, load, make_cfg, make_weights, STAGES)
