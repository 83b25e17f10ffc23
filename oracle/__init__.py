"""fp64 CPU oracle for GPTQ layer quantization (test infrastructure only; see gptq_oracle)."""
from .gptq_oracle import (  # noqa: F401
    hessian_accumulate, hessian_finalize, hessian, damp, inverse_hessian_factor, quant_params,
    quantize, gptq_quantize, gptq_quantize_unbatched, rtn_quantize, layer_error, gptq_layer,
    check_shapes,
)
from .w4a16 import (  # noqa: F401
    pack_codes, unpack_codes, dequantize, w4a16_matmul, w4a16_abs_terms, group_of_column,
    pack_codes_3bit, unpack_codes_3bit,
)
from .rotation import (  # noqa: F401
    hadamard_block, rotation_matrix, rotate, rotate_abs_terms, weight_incoherence,
)
from .obq import obq_row, obq_quantize  # noqa: F401
