"""packed_variable_length_attn_b200 (placeholder; the binding lands with the C ABI)."""
