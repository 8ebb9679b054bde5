"""B200-native fused dequantize + GEMV for GGML-style Q8_0 / Q4_K weights."""
