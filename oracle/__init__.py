"""CPU oracle for the Hadamard incoherence hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import or run it.  It shares no code with the CUDA
library (``hadamard_incoherence_transforms_b200``); both sides take their
inputs from the separate ``synth`` generators only.

Everything here is plain and slow on purpose: dense Sylvester Hadamard
matrices and float64 matrix products for the transforms, a scalar fp32
round-to-nearest quantizer written element-wise with numpy float32
arithmetic, ``np.packbits`` for the code layout, a dense scatter-add plus a
matmul for the sparse adapter, and einsum over one mixed-radix digit at a time
for the butterfly stages.

Sources (page title, section):

* HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
  Quantization -- technical summary §1 (the randomized Hadamard transform is
  fast, O(d log d), exactly orthogonal), §2.1 (mixed-radix schedule of
  stride-based block-diagonal orthogonal stages), §2.2 (normalized Sylvester
  Hadamard as the fixed mixer; zero-initialised HARP recovers the RHT), §5
  (exact change of basis, two-sided processor); §2.2 also gives the learnable
  blocks Q(theta) G (Givens / Cayley) and §2.4 their int8 storage.
* QWHA: Quantization-Aware Walsh-Hadamard Adaptation for Parameter-Efficient
  Fine-Tuning on Large Language Models -- technical summary §2.1 (single
  transform adapter dW = F H^-1, F sparse from a value vector c and an index
  list E; WHT kernel of +-1 entries, add/subtract only; the two-transform form
  H'^-1 F H^-1), §2.2 (AdaAlloc budget split and per-channel top-k,
  least-squares Refinement), §4 (scatter operations).

Parity status of each function is stated in its module header.
"""
from . import hadamard, quant, butterfly, sparse, harp, qwha  # noqa: F401
