"""SERQ W4A4 linear for NVIDIA B200 (sm_100a): Python binding of libserq.so.

Y ~= X^_q W^_q + X~_{s,q} Q(R) -- saliency-aware single-matrix low-rank error
reconstruction ("SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
Quantization"). The computation runs in the CUDA kernels of libserq.so;
this package only marshals arguments (see include/serq.h).
"""

from .serq import (  # noqa: F401
    QuantAct,
    SerqWeight,
    alloc_act,
    serq_act_buffer_sizes,
    serq_add,
    serq_attention_prefill,
    serq_calib_absmax,
    serq_debug_fail_next_allocations,
    serq_device_status,
    serq_fold_producer,
    serq_fold_quant_act,
    serq_linear,
    serq_linear_l2qer,
    serq_linear_small_m_noalloc,
    serq_linear_swiglu_quant,
    serq_prepare,
    serq_prepare_swiglu,
    serq_quant_act,
    serq_rope,
    serq_rmsnorm_quant_act,
    serq_swiglu_quant_act,
    serq_selftest_wait,
    serq_version,
    serq_weight_create_from_host,
    serq_weight_export,
    serq_weight_file_read,
    serq_weight_file_write,
    serq_weight_get_view,
    serq_weight_load,
    serq_weight_save,
)
from ._native import SerqError  # noqa: F401
