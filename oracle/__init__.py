"""Plain, slow CPU oracle for online fine-grained quantization and block-scaled GEMM.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code, tables or
constants generator with the CUDA library in ``fp4_precision_gemm_b200``; the only
module both sides consume is the seeded input generator ``workloads.py``, which holds
none of the method's arithmetic.

The oracle is written in NumPy from the definitions:

* ``formats``  E4M3 / E5M2 / E8M0 / E2M1 / BF16 codecs from their bit definitions
  (OCP 8-bit floating point spec for E4M3 and E5M2, OCP MX spec v1.0 for E8M0 and E2M1).
* ``philox``   Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
  Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), pinned by the generator's
  published known-answer vectors (``tests/golden/philox4x32_10_kat.txt``).
* ``rht``      the 16x16 random Hadamard transform used on gradient inputs.
* ``quant``    the quantizers: 1x128 tiles, 128x128 blocks, MX (32-element blocks,
  E8M0 scales), per-tensor current and delayed scaling (E4M3 or E5M2), NVFP4 (E2M1
  values, per-16 E4M3 scales, a per-tensor FP32 scale, optional RHT and stochastic
  rounding; 16x16 blocks for weights).
* ``gemm``     dequantization and the FP64 reference product with the tolerance check.

The pages the method comes from (cited by title in every module):

* "Accelerating FP8 training performance with the NVIDIA NeMo framework" (hyper.ai):
  the four NeMo scaling recipes, MXFP8 on DGX B200 (blocks of 32 values).
* "NVIDIA developed a method to train neural networks in 4-bit precision"
  (news.hamidun.com), section "How it works": NVFP4, 16x16 random Hadamard transforms
  on gradient inputs, stochastic rounding.
* "Can you explain the role of FP8 precision in DeepSeek-V3 training" (codingmall.com),
  sections "Fine-grained quantization" (1x128 activation tiles, 128x128 weight blocks),
  "Online quantization" (scales from the live amax), "Increased accumulation precision"
  (promotion of partial sums to FP32 at fixed intervals) and "Unified E4M3 format".

Functions whose result is pinned only by the written spec (no independent pin exists)
say "parity unpinned" in their docstring.  Pins live in ``tests/test_oracle_*.py``.
"""
