"""B200-native per-group low-bit weight quantization and quantized linear layers."""
