"""B200-native DiT joint attention (placeholder; the binding is added with the C-ABI)."""
