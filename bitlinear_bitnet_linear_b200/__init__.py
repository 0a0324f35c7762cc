"""BitNet b1.58 BitLinear hot path for NVIDIA B200 (sm_100a).

The compute lives in libbitnet.so (C ABI, include/bitnet.h); this package is
the thin Python binding over it plus the seeded synthetic workload
generators.  Importing the package does not load the library; the first call
does, and fails loudly if it is missing.
"""
from ._binding import (BF16, F32, PATH_AUTO, PATH_GEMV, PATH_TC, BitnetError, bitnet_get_error,  # noqa: F401
                       bitnet_linear, bitnet_linear_b1, bitnet_linear_grouped, bitnet_linear_q, bitnet_linear_relu2, bitnet_pack,
                       bitnet_pack_b1, bitnet_pack_t3, bitnet_quant_act, bitnet_quant_weights_b1, bitnet_unpack_b1,
                       bitnet_unpack_t3, bitnet_linear_t3, bitnet_t3_row_bytes,
                       bitnet_quant_act_relu2, bitnet_quant_weights,
                       bitnet_quant_weights_noalloc, bitnet_quant_weights_workspace_bytes, bitnet_set_wait_limit_us, bitnet_ternarise,
                       bitnet_unpack, bitnet_watchdog_selftest, bitnet_workspace_bytes, bitnet_workspace_init,
                       bitnet_debug_stream_plan,
                       lib, new_workspace, GroupedCall)
