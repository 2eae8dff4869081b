"""weight_quantized_expert_b200 -- a B200-native (sm_100a) MoE layer with group-quantised
experts: a C-ABI CUDA library (libfocr_moe.so, include/focr_moe.h) and a thin binding.

Submodules: ``api`` (the binding), ``synth`` (seeded synthetic inputs), ``build``
(nvcc build of the library).  Importing the package loads nothing; the library is
loaded on the first call through ``api``.
"""
