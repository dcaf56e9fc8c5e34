"""CPU oracle for the VQ + sparse linear layer (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
package.  It shares no code with the CUDA library.
"""
from .oracle import (  # noqa: F401
    build,
    f16_to_f64,
    bf16_to_f64,
    round_f16,
    body_f16,
    unpack,
    dequant_exact,
    dequant_f64,
    gemv_f64,
    vptq_compression_ratio,
    assign_exact,
    residual_assign_exact,
    sqdist_exact,
    OracleError,
)
