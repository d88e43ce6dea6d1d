"""B200-native fused per-token normalisation cores of the Muse Spark Open decoder layer."""
