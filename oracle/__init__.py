"""FP64 CPU oracle for GPTQ layer-wise quantization — TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this package.
The product path (the CUDA library and its Python binding) never imports, links or runs it,
and this package imports nothing from the product path.

It restates, plainly and slowly, what the source pages define:
  hessian   H = 2 X X^T (brute-force loops for tiny inputs, a library matmul otherwise)
  prepare   dead columns, relative damping, act-order permutation, and the upper Cholesky
            factor U of H^-1 by the pages' three steps (chol, cholesky_inverse, chol upper)
  sweep     the column sweep three ways: OBS with the recursive inverse-Hessian downdate,
            unblocked with rows of U, and blocked with lazy trailing updates; plus a
            least-squares brute force that shares none of the inverse-Hessian machinery
  quantizer uniform asymmetric / symmetric quantizer, group and per-row statistics, RTN
  pack      LSB-first bit packing of the codes, fp16 scales/zeros
  error     the layer objective ||W X - W_hat X||_F^2

Page titles cited in the docstrings (section names follow each title):
  [INT4-GPTQ]  "INT4 and GPTQ Quantization" (beta.fermi.ai wiki)
  [RA-GPTQ]    "GPTQ" (robotsatlas.com)
  [Q-INT8]     "Quantization (INT8, INT4, GPTQ)" (brentwoodlivery.com)
  [GPTQ-MATH]  "GPTQ: Mathematical Foundations, Optimal Brain Surgeon Inversion, and
               Second-Order Error Minimization in LLM Quantization" (llms.blog)

Floating point: FP64 throughout, except the quantizer used for RTN and for bit-exact parity of
quantize-given-scales, which the pages write as float32 tensor code and which therefore runs
in float32 with IEEE division and round-half-to-even.

Parity status of each function is stated in its docstring ("pinned by ..."). Functions with
no external pin say "parity unpinned".
"""
from . import error, gemv, hessian, pack, prepare, quantizer, sweep  # noqa: F401
from .layer import gptq_layer, rtn_layer  # noqa: F401
