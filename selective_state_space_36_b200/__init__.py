"""B200-native selective state-space (S6) scan: C-ABI CUDA library + binding."""
