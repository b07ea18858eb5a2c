"""Lightning Attention forward (causal linear attention with SiLU features, block-wise,
fp32 state, RMSNorm * sigmoid(gate)) as a C-ABI CUDA library for B200 (sm_100a).

``lightning_attn`` is the ctypes binding of ``liblightning_attn.so``; ``build`` compiles
the library in-tree with nvcc.
"""
