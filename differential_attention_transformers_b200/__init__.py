"""B200-native differential attention forward (placeholder; binding follows)."""
