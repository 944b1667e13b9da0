"""B200-native block-quantized dequant GEMV (placeholder, filled in with the binding)."""
