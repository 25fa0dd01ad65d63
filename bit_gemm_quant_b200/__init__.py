"""B200-native group-wise INT4 weight quantization and W4A16 GEMV/GEMM."""
