"""B200-native forward pass of one mixture-of-experts layer (placeholder; binding follows)."""
