"""B200-native hybrid-mixer decoding: the per-layer token-mixer step (FA, SWA, KDA, GDN) of a
supernet decoder whose placement vector picks one mixer per layer.

The compute lives in libhmd.so (hand-written sm_100a CUDA kernels behind the C ABI declared in
include/hmd.h); this package is its ctypes binding plus the seeded input generator and the
48-layer mixer-only stack driver.
"""
from ._lib import (BF16, BatchPlan, group_sequences, mixer_decode_step_batch, DEVERR_GATE, DEVERR_PAGE, DEVERR_SEQLEN, DEVERR_SLOT, DEVERR_TIMEOUT, F32, FA, GDN,
                   KDA, SWA, DecodeIO, HmdError, KVCache, StateCache, attn_decode,
                   attn_decode_static_ws, attn_prefill, attn_prefill_ext, attn_decode_workspace_size,
                   attn_verify,
                   attn_verify_workspace_size, delta_rule_decode, delta_rule_decode_act,
                   delta_rule_decode_chain,
                   delta_rule_decode_to, delta_rule_prefill_chunked_act,
                   delta_rule_prefill_chunked, delta_rule_prefill_chunked_ws,
                   delta_rule_prefill_workspace_size, hmd_device_errors, hmd_last_error,
                   hmd_status_string, hmd_test_arm_copy_skip, hmd_version, lib,
                   mixer_decode_step)

__all__ = ["BF16", "BatchPlan", "group_sequences", "mixer_decode_step_batch", "DEVERR_GATE", "DEVERR_PAGE", "DEVERR_SEQLEN", "DEVERR_SLOT", "DEVERR_TIMEOUT", "F32", "FA",
           "GDN", "KDA", "SWA", "DecodeIO", "HmdError", "KVCache", "StateCache", "attn_decode",
           "attn_decode_static_ws", "attn_decode_workspace_size", "attn_prefill", "attn_prefill_ext",
           "attn_verify",
           "attn_verify_workspace_size", "delta_rule_decode", "delta_rule_decode_act",
           "delta_rule_decode_chain",
           "delta_rule_decode_to", "delta_rule_prefill_chunked_act",
           "delta_rule_prefill_chunked", "delta_rule_prefill_chunked_ws",
           "delta_rule_prefill_workspace_size", "hmd_device_errors", "hmd_last_error",
           "hmd_status_string", "hmd_test_arm_copy_skip", "hmd_version", "lib",
           "mixer_decode_step"]
