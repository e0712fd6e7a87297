"""KDA (Kimi Delta Attention) prefill and decode on NVIDIA B200 (sm_100a).

The compute lives in libkda.so (CUDA, C ABI in include/kda.h); :mod:`.kda` is
its ctypes binding and :mod:`.workloads` draws seeded synthetic inputs.
"""
from .kda import (  # noqa: F401
    EXPORTS, KDA_DTYPE_BF16, KDA_DTYPE_F32, KDA_NOALLOC_SCRATCH_BYTES, KDA_ERR_BAD_SEQLENS, KDA_ERR_CUDA,
    KDA_ERR_INVALID_ARG, KDA_ERR_TIMEOUT, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_OK,
    KdaError, alloc_workspace, chunk_fwd, chunk_bwd, chunk_kda, ChunkKDA, decode_step,
    kda_chunk_fwd,
    kda_chunk_fwd_workspace_size, kda_chunk_gate_cumsum, kda_chunk_inter, kda_chunk_intra,
    kda_chunk_output, kda_chunk_fwd_noalloc, kda_chunk_split_chain, kda_chunk_split_intra,
    kda_chunk_split_workspace_size, kda_chunk_fwd_plan, kda_qkv_conv_norm, kda_qkv_conv_norm_step, kda_output_norm_gate,
    PLAN_NAMES, PLAN_CODES, plan_code, kda_chunk_fwd_with_plan, kda_chunk_fwd_plan_workspace_size,
    kda_gdn_chunk_fwd, kda_gdn_chunk_fwd_workspace_size, kda_gdn_decode_step,
    kda_chunk_bwd, kda_chunk_bwd_workspace_size, kda_gdn_chunk_bwd,
    kda_gdn_chunk_bwd_workspace_size, KDA_PLAN_SIMT,
    KDA_PLAN_SPLIT, KDA_PLAN_OVERLAP, kda_decode_step, kda_get_device_status, kda_num_chunks_upper_bound,
    load, status_string, kda_layer_decode_step, kda_test_overlap_flag_timeout,
    kda_layer_chunk_fwd, kda_layer_chunk_fwd_workspace_size, kda_chunk_state_maps,
    kda_fold_segment_states,
)
