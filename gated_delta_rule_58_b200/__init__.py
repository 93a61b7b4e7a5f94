"""B200-native gated delta rule library (placeholder; binding added with the CUDA library)."""
