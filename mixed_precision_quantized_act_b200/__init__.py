"""MixLLM W4.4A8 linear layer for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libmixllm_b200.so`` (C ABI in
``include/mixllm.h``); this package is its thin Python binding plus the seeded
synthetic workloads used by the tests and the benchmark.
"""
from ._lib import (  # noqa: F401
    GROUP,
    MixLLMError,
    SMALL_M_MAX,
    PackedLinear,
    empty_packed,
    gemm_debug_partials,
    gemm_w4w8a8,
    channel_salience,
    channel_salience_into,
    gemm_w4w8a8_into,
    gemm_w4w8a8_plain_i2f_into,
    gemm_w4w8a8_small_m,
    gemm_w4w8a8_small_m_noalloc_into,
    gemm_w4w8a8_small_m_into,
    linear,
    linear_into,
    linear_small_m_into,
    linear_small_m_workspace,
    linear_workspace,
    load,
    pack_weights,
    pack_weights_host,
    packed_sizes,
    quantize_act,
    quantize_act_into,
    select_top_t,
    select_top_t_into,
    select_top_t_workspace,
    selftest_bounds,
    selftest_wait_timeout,
    checked_build,
    small_m_kernel,
    small_m_debug_partials,
    small_m_workspace,
    small_m_workspace_bytes,
    sync_status,
    version,
)
from .packfile import load_packed, save_packed  # noqa: F401
