"""B200-native states-form KV-cache attention (package placeholder; binding follows)."""
