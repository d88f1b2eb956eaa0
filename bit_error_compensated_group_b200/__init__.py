"""Echo 4-bit error-compensated all-reduce, simulated over P virtual ranks on
one B200 (sm_100a). The compute path is ``libecho_b200.so`` (C ABI in
``include/echo.h``); ``echo`` is its ctypes binding.

Importing the package does not load the CUDA library; the first call does,
and raises if the library is missing.
"""
from .echo import (  # noqa: F401
    ECHO_EINVAL, ECHO_ECUDA, ECHO_ENOSPACE, ECHO_ERANGE, ECHO_ETIMEOUT, ECHO_FLAG_RANGE, ECHO_FLAG_TIMEOUT,
    ECHO_MAX_CHUNKS, ECHO_MAX_RANKS, ECHO_NOALLOC_SCRATCH_BYTES, ECHO_OK, ECHO_QUANT_DIRECTED, ECHO_QUANT_INT_ZERO, ECHO_QUANT_NEAREST,
    EchoAllReduce, EchoError, EchoLayout, EchoRank, EchoRankLayout, ExchangePlan, column_window,
    echo_allreduce_sim, echo_allreduce_sim_host, echo_allreduce_sim_noalloc, echo_allreduce_sim_range,
    echo_background_traffic, echo_bf16_allreduce_sim,
    echo_check_watchdog, echo_free, echo_get_status, echo_get_wait_limit, echo_init_rank, echo_init_state,
    echo_inject_launch_failure, echo_phase_gather, echo_phase_quantize, echo_phase_reduce, echo_query_layout,
    echo_query_chunk, echo_query_rank_layout, echo_rank_decode, echo_rank_decode_chunk, echo_rank_quantize,
    echo_rank_quantize_chunk, echo_rank_reduce, echo_rank_reduce_chunk, echo_set_quantizer,
    echo_set_wait_limit, echo_state_bytes, echo_status_string, echo_workspace_bytes, exchange_all_gather,
    exchange_all_to_all, exchange_chunk, exchange_chunk_in_process, exchange_in_process, lib, run_chunked,
)
