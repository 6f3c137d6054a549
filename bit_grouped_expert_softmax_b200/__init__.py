"""B200-native routed int4 MoE layer (top-k softmax routing, shared expert, grouped SwiGLU)."""
