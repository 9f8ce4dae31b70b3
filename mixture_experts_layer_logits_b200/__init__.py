"""B200-native MoE layer forward (placeholder; the binding is added with the C ABI)."""
