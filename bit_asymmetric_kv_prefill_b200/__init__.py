"""B200-native KIVI asymmetric 2-bit KV cache (placeholder; binding follows)."""
