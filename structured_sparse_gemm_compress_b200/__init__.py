"""B200-native N:M semi-structured sparse weight x dense activation GEMM."""
