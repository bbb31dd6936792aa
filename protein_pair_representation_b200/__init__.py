"""B200 (sm_100a) triangle multiplicative update.

The computation runs in the CUDA library built from ``csrc/`` (C ABI in
``include/trimul.h``); ``trimul`` is its Python binding.
"""
from .trimul import (  # noqa: F401
    BF16, F16, F32, INCOMING, OUTGOING, TriMulError, TriMulLayer, check_device_status, contract,
    contract_scale, intermediate_dtype, kernels_per_forward, library_path, load_library,
)
