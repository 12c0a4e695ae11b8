"""NVFP4 W4A4 linear layer for B200 (sm_100a).

Submodules:
  native      -- ctypes binding of libnvfp4w4a4.so (quantize, harmonize, the W4A4
                 linear and GEMM, the gate projection, fake-quant, FP8 quantize,
                 the re-quantizing harmonize, the RMSNorm-fused quantize)
  checkpoint  -- save/load of quantized weights and static FP8 KV scales
  workloads   -- seeded synthetic inputs shaped like the model's layers
  build       -- compiles the library in-tree with nvcc for sm_100a
"""
