"""Plain fp64 CPU oracle for GPTQ's per-layer quantization pass.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
anything in this package: only the tests, the smoke check in the repository's
entry module and the CPU-baseline leg of the benchmark do. It shares no code
with the CUDA library and does not import it.

Every function follows the method as the source pages state it (citations are
in each docstring) with NumPy doing the dense linear algebra.  No blocking,
fusion or reordering is added beyond what the pages describe: the one blocked
structure (lazy 128-column blocks with a global trailing update) is the pages'
own.  GPTQ-2D (two-sided rounding) lives in ``oracle.gptq2d_oracle``.
"""
from .gptq_oracle import (  # noqa: F401
    hessian,
    accumulate_hessian,
    prepare,
    inverse_factor,
    inverse_factor_reversed,
    group_params,
    quantize_values,
    group_params_f32,
    quantize_values_f32,
    gptq_core,
    gptq_quantize,
    rtn_quantize,
    rtn_quantize_f32,
    gptq_layer,
    layer_output_error,
    pack_codes,
    unpack_codes,
    packed_words_per_row,
)
from . import gptq2d_oracle  # noqa: F401,E402
