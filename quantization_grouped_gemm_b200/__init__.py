"""B200-native FP8 quantisation and FP8 scaled grouped GEMM for MoE training."""
