"""AQUA (Attention via QUery mAgnitudes) online attention step for NVIDIA B200 (sm_100a).

The CUDA library libaqua_b200.so (C ABI in include/aqua.h) does all the work;
this package is its ctypes binding plus PyTorch-allocated cache buffers.
"""
from .abi import (  # noqa: F401
    AQUA_BF16, AQUA_F32, AQUA_OK, AquaError, aqua_cache, aqua_calibrate, aqua_calibrate_workspace_size,
    aqua_decode_attn, aqua_decode_attn_static, aqua_decode_attend, aqua_decode_select, aqua_decode_workspace_size, aqua_h2o_update, aqua_last_error, aqua_prefill_attn,
    aqua_prefill_workspace_size, aqua_project_keys, aqua_selftest_wait_timeout, aqua_status, aqua_version,
    load_library, LIB_PATH, EXPORTED,
)
from .cache import AquaCache  # noqa: F401
