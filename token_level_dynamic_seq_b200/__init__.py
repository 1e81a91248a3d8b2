"""B200-native token-level dynamic local-global attention (placeholder, binding follows)."""
