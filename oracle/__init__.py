"""CPU oracle for the WUSH transform-then-quantize linear layer -- TEST INFRASTRUCTURE.

This package is the plain, slow, obviously-correct statement of what the CUDA
path computes. It is written in numpy, in fp64 wherever the pages leave the
precision open, and it shares no code with the CUDA library: it neither imports
``activation_quantization_b200`` nor is imported by it. Only the tests, the
smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
use it.

Pages it follows (cited by title and section in each function):
  * "WUSH news article" -- the Chinese news report on WUSH (ETH Zurich, ISTA,
    Red Hat AI): its paragraphs on the construction, the optimality claims, the
    layer-wise experiments and the deployment workflow.
  * "WUSH: Near-Optimal Adaptive Transforms for LLM Quantization" (AI Radio
    episode): "The gist", "Problem Setup and Goal" (the output loss).
  * "打破精度瓶颈：ITQ3_S如何重塑消费级GPU上的大语言模型推理效率" (the ITQ3_S
    article): section "核心技术：FWHT预旋转与TurboQuant的完美融合".

Where the pages are silent (the WUSH matrix formula, the MXFP4/NVFP4/INT4 scale
and rounding rules, normalisations, eigenvector signs), the plainest reading is
taken and stated in the function that uses it.

Parity status per function: every public function is pinned by a
``-m "not gpu"`` test against closed forms, library routines or brute force
(tests/test_oracle_*.py). None is "parity unpinned".
"""
from . import formats, transforms, calibrate, quant, gemm, itq3, loss  # noqa: F401
