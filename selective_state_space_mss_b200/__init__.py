"""B200-native selective scan (S6): CUDA library + thin Python binding."""
