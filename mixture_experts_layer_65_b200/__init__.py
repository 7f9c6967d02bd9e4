"""DeepSeekMoE layer forward pass on B200 (sm_100a): hand-written CUDA kernels behind a C-ABI.

The compiled library is loaded on first use (``mixture_experts_layer_65_b200.layer``);
importing the package alone does not touch the GPU.
"""
