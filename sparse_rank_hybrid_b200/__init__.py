"""B200-native forward pass of 3D-RoPE sparse + low-rank hybrid attention (RoLA / RoPeSLR).

The compute path is the C-ABI library `libslra.so` (hand-written CUDA for sm_100a) wrapped by
`sparse_rank_hybrid_b200.slra`; importing this package does not load it, so the seeded input
generator (`inputs`) and the workload table (`workloads`) work on machines without a GPU.
"""
