"""DeepSeekMoE layer forward on NVIDIA B200 (sm_100a).

The compute lives in libdsmoe.so (hand-written CUDA kernels behind a C ABI,
declared in include/dsmoe.h); this package is its ctypes binding plus the
multi-GPU token-sharding helper.
"""
from .binding import *  # noqa: F401,F403
from .binding import (DSMoE, DsmoeCfg, DsmoeError, make_cfg, cfg_from, dsmoe_create, dsmoe_destroy,
                      dsmoe_forward, dsmoe_forward_host, dsmoe_balance_stats, dsmoe_get_status,
                      dsmoe_set_wait_limit, dsmoe_set_timing, dsmoe_stage_times, dsmoe_stage_name,
                      dsmoe_launch_count, dsmoe_check_config, dsmoe_workspace_bytes, dsmoe_abi_version,
                      dsmoe_status_string, dsmoe_last_error, stage_names, ABI_FUNCTIONS, LIB_PATH,
                      dsmoe_workspace_tensor, workspace_view, dsmoe_balance_losses,
                      dsmoe_sequence_balance, dsmoe_bias_update, dsmoe_route_noalloc)
