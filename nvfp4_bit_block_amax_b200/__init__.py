"""NVFP4 linear-layer hot path for B200 (sm_100a).

The product is the C-ABI library ``libnvfp4.so`` (declared in
``include/nvfp4.h``, built in-tree by ``build.py``): tensor amax -> FP32
global scale -> E4M3 block scales (16 along K, or 16x16 for weights) -> E2M1
codes (nearest-even, or stochastic rounding with Philox4x32-10 bits; an
optional 16-point random Hadamard transform for the weight-gradient
operands) -> block-scaled tcgen05 GEMM with FP32 accumulation; dequantize;
an MXFP4 variant.

Modules:
  nvfp4   ctypes binding with the C names (argument marshalling only) and a
          few torch helpers (quantize_1d, quantize_2d, quantize_dual, gemm,
          mxfp4_quantize, mxfp4_gemm, dequantize).  Raises if the library is
          not built: there is no fallback path.
  inputs  seeded synthetic inputs (bf16 bit arrays) shared by the tests and
          the benchmark; no quantization arithmetic lives there.
  build   nvcc build of libnvfp4.so for sm_100a.
"""
