"""B200-native ART run-time-terminated decode attention (placeholder; binding added below)."""
