"""kv_quantization_b200 -- B200-native rotated scalar quantization and QJL sketching.

The product is the C-ABI library ``librq.so`` (include/rq.h) built from
``csrc/`` for sm_100a; ``_lib`` is its ctypes binding (same function names),
``synth`` the seeded input recipes, ``build`` the nvcc build step.
"""
from ._lib import (  # noqa: F401
    RQ_BF16, RQ_CODES_INT8, RQ_CODES_PACKED, RQ_F16, RQError, lib, qjl_attention, qjl_attention_workspace_bytes,
    qjl_make_projection, qjl_score,
    qjl_score_noalloc, qjl_score_outlier, qjl_score_workspace_bytes, qjl_sketch, qjl_sketch_outlier,
    qjl_sketch_outlier_workspace_bytes, rq_beta_lloyd_max, rq_code_bytes, rq_dequantize, rq_dequantize_dense, rq_device_error, rq_last_launch, rq_lloyd_max, rq_make_rotation, rq_quantize_dense,
    rq_probe_bounded_wait, rq_quantize,
    rq_quantize_qjl, status_string,
)
