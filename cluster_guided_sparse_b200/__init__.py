"""B200-native centroid-guided sparse attention (SCOPE formulation)."""
