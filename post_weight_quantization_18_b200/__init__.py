"""GPTQ layer-wise weight quantization on NVIDIA B200 (sm_100a).

The hot path runs in libgptq_b200.so (C ABI in include/gptq.h); this package is its ctypes
binding (`_lib`, same names as the C entry points) plus a small allocation helper (`layer`)
and the data-parallel driver over torch.distributed (`sharded`).
Importing it without the built library raises: there is no CPU fallback.
"""
from ._lib import (EXPORTED, GPTQ_BF16, GPTQ_F32, GPTQ_ORDER_DESC_ACT, GPTQ_ORDER_GIVEN,  # noqa: F401
                   GPTQ_ORDER_NATURAL, GPTQError, LIB_PATH, gptq_hessian_accumulate,
                   gptq_dequant_gemm, gptq_dequant_gemv, gptq_gemm_f32, gptq_pack, gptq_params, gptq_prepare_hinv, gptq_quantize_layer, gptq_quantize_pack_layer,
                   gptq_quantize_layer_noalloc, GPTQ_NOALLOC_SCRATCH_BYTES,
                   gptq_status_string, gptq_workspace_size, make_params, rtn_quantize, status_string)
from .layer import QuantizedLayer, check_status, hessian, prepare, quantize_layer, rtn  # noqa: F401
from . import sharded  # noqa: F401  (token-sharded H, one all-reduce, row-sharded sweep)
