"""B200-native (sm_100a) MoE layer hot path: router top-k, dispatch layout, permute,
grouped SwiGLU experts on tcgen05 tensor cores, and the gate-weighted combine.

The compute lives in libmoe.so (C ABI in include/moe.h); this package is its Python
binding.  Importing it loads the library and fails loudly when it is missing.
"""
from .binding import (EXPORTED, Layout, MoEError, alloc_workspace, c_config, check_config,  # noqa: F401
                      combine, combine_staged, dispatch_layout, dispatch_layout_noalloc, eplb_assign,
                      eplb_place_weights, eplb_plan, eplb_workspace_bytes, expert_fc1, physical_config,
                      expert_fc2, grouped_ffn, layer_forward, layer_forward_overlapped, layout_workspace_bytes,
                      load, permute, permute_staged, route, routed_ffn, selftest_bounded_wait, shared_ffn, version,
                      workspace_bytes, quantize_fp8, permute_fp8, grouped_ffn_fp8, workspace_bytes_fp8,
                      layer_forward_fp8, capacity_drop, capacity_of, checks_enabled, checks_register,
                      layer_forward_chunked, workspace_bytes_chunked, quantize_mx, permute_mx,
                      grouped_ffn_mx, workspace_bytes_mx, layer_forward_mx)

from . import ep  # noqa: F401,E402  (expert parallelism across GPUs: moe_ep_*)

load()
