"""B200-native GPTQ layer quantization.

Two C-ABI calls do the work (``include/gptq.h``): ``gptq_accumulate_hessian``
(H += 2 X^T X on the tcgen05 tensor cores) and ``gptq_quantize_layer``
(damped inverse-Cholesky factor, quantize-and-compensate sweep, packing), plus
the factor / factored-sweep split for layers that share one Hessian.  This
package is the thin Python binding over ``lib/libgptq.so``.
"""

from .api import (  # noqa: F401
    GPTQError,
    QuantResult,
    accumulate_hessian,
    dequantize_weight,
    device_status,
    factor_hessian,
    factor_hessians,
    group_count,
    launch_count,
    quantize_layer,
    quantize_layer_factored,
    quantize_linears,
    quantized_linear,
    reorder_act_order,
)

__version__ = "0.1.0"
