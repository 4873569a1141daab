"""B200-native SliM-LLM per-layer quantizer (sm_100a CUDA behind a C ABI).

Importing the package loads nothing; `from post_weight_quantization_hessian_b200 import slim`
binds the compiled library.
"""
