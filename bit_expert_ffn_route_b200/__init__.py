"""B200-native routed-MoE expert pass (router, top-k, expert-cache slot lookup,
quantised SwiGLU experts, combine).  The CUDA library is loaded lazily by
:mod:`bit_expert_ffn_route_b200.moe`; importing the package loads nothing."""
