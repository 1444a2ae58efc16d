"""BitLinear W1.58·A8 matmul for B200 (placeholder while the binding is written)."""
