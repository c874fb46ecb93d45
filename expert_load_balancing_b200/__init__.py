"""B200-native sigmoid MoE router with Exact Quantile Balancing."""
