"""B200-native low-bit two-step quantized all-reduce (Flash Communication)."""
