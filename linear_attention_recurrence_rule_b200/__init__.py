"""Gated delta rule (Gated DeltaNet core) for NVIDIA B200, sm_100a.

The computation lives in the CUDA library built from ``csrc/`` (C ABI in
``include/gdn.h``); this package is its thin Python binding plus the seeded
synthetic input generator used by the tests and the benchmark.
"""
from .gdn import (GDN_BF16, GDN_F32, GDNError, gdn_chunk_prefill,  # noqa: F401
                  gdn_chunk_prefill_host, gdn_chunk_prefill_host_workspace_size, gdn_validate_cu_seqlens,
                  gdn_chunk_prefill_path, gdn_chunk_prefill_workspace_size, gdn_read_status, gdn_recurrent_step,
                  gdn_recurrent_verify, gdn_recurrent_verify_workspace_size, gdn_state_commit,
                  gdn_recurrent_commit_verify, gdn_recurrent_commit_verify_workspace_size,
                  gdn_state_commit_deltas, gdn_short_conv, gdn_output_gate, gdn_recurrent_step_layer,
                  gdn_chunk_prefill_layer, gdn_chunk_prefill_layer_workspace_size, CONV_SILU,
                  CONV_MAX_WIDTH, lib_path, load_library, status_string, PROLOGUE_NORM_Q, PROLOGUE_NORM_K,
                  PROLOGUE_GATE_LOGITS, PROLOGUE_ALL, ROW_DECAY)

__all__ = ["gdn_chunk_prefill", "gdn_recurrent_step", "gdn_recurrent_verify", "gdn_recurrent_verify_workspace_size", "gdn_state_commit",
           "gdn_recurrent_commit_verify", "gdn_recurrent_commit_verify_workspace_size",
           "gdn_state_commit_deltas", "gdn_chunk_prefill_workspace_size", "gdn_chunk_prefill_path",
           "gdn_chunk_prefill_host", "gdn_chunk_prefill_host_workspace_size", "gdn_validate_cu_seqlens",
           "gdn_read_status", "status_string", "load_library", "lib_path", "GDNError",
           "GDN_F32", "GDN_BF16", "PROLOGUE_NORM_Q", "PROLOGUE_NORM_K", "PROLOGUE_GATE_LOGITS",
           "PROLOGUE_ALL", "ROW_DECAY", "gdn_short_conv", "gdn_output_gate",
           "gdn_recurrent_step_layer", "gdn_chunk_prefill_layer",
           "gdn_chunk_prefill_layer_workspace_size", "CONV_SILU", "CONV_MAX_WIDTH"]
