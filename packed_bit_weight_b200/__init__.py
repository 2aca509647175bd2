"""packed_bit_weight_b200: packed 4-bit weight GEMV/GEMM for B200 (sm_100a)."""
