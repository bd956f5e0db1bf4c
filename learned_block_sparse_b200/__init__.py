"""B200-native ETA block-sparse decode (placeholder until the binding lands)."""
