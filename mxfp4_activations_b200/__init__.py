"""B200-native KroQuant online activation quantizer (placeholder, filled below)."""
