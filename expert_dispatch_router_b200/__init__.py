"""B200-native forward pass of one Mixture-of-Experts FFN layer (see binding)."""
