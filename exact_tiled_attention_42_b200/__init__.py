"""Exact tiled softmax attention for B200 (sm_100a).

Python binding of the C ABI in ``include/fa.h``. The functions here only
marshal arguments (torch tensors -> device pointers, the current CUDA stream)
and raise on a non-zero status; every step of the computation runs in the
library's CUDA kernels. PyTorch provides device memory and streams only.
"""

from .api import (  # noqa: F401
    FAError,
    FA_OK,
    fa_fwd,
    fa_bwd,
    fa_bwd_noalloc,
    fa_fwd_varlen,
    fa_bwd_varlen,
    fa_bwd_varlen_workspace_size,
    fa_fwd_fp8,
    fa_fwd_mxfp8,
    fa_fp8_quantize,
    fa_fwd_fp8_quantized,
    fa_fwd_decode,
    fa_decode_workspace_size,
    fa_bwd_workspace_size,
    fa_fp8_workspace_size,
    fa_mxfp8_workspace_size,
    fa_status_string,
    fa_last_device_status,
)
