"""B200-native split-KV decode attention (Flash-Decoding) behind a C ABI.

The computation lives in libfdecode.so (CUDA, sm_100a; declared in
include/fd.h). This package is its thin binding (same entry-point names) plus
the workload table and the seeded input generator."""
from . import configs, context, inputs  # noqa: F401
from ._lib import (  # noqa: F401
    FdError, decode, decode_multi, decode_paged, decode_quant, decode_quant_paged, fd_combine, fd_decode, fd_decode_multi,
    fd_decode_paged, fd_decode_quant, fd_decode_splits, fd_merge_partials, fd_decode_static, fd_device_status, fd_plan,
    fd_plan_for_sms, fd_read_probe, fd_segments, fd_split, fd_strerror, fd_version, fd_workspace_bytes, fd_workspace_init, lib,
    prepare_decode, prepare_decode_multi, prepare_decode_paged, prepare_decode_quant, prepare_decode_quant_paged, quant_workspace_bytes,
    workspace_layout,
)
