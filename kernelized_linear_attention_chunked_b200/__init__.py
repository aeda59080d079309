"""Causal kernelized linear attention (rank-one PSD feature phi(x) = x x^T) and
the LoLA self-recall-error sparse cache on NVIDIA B200 (sm_100a).

The computation lives in libkata.so (C ABI: include/kata.h); this package is
its thin Python binding plus the seeded synthetic input generators.
"""
from ._binding import (  # noqa: F401
    KATA_BF16,
    KATA_F32,
    FORMS,
    LIB_PATH,
    SIGNATURES,
    KataError,
    debug_build,
    decode_step,
    decode_step_feature,
    feature_dim,
    decode_step_host,
    hybrid_readout,
    launch_count,
    lib,
    lola_fused_applies,
    lola_prefill,
    lola_prefill_workspace_bytes,
    packed_dim,
    prefill,
    prefill_auto_form,
    prefill_feature,
    prefill_host,
    prefill_host_workspace_bytes,
    prefill_uses_tensor_cores,
    prefill_workspace_bytes,
    quadratic_max_tokens,
    sre_score_topk,
    state_prefix,
    sync_status,
    test_bounds_check,
    test_forced_timeout,
)
