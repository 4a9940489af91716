"""B200-native LCSA (locality-constrained sparse attention) library binding."""
