"""memory_bound_fk_b200: fused memory-bound operators (tanh-GELU, row softmax) for B200."""
