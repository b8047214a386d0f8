"""B200-native W8A8 / W4A8 activation-quantized linear (sm_100a CUDA behind a C ABI)."""
