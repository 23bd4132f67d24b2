"""Sol-Attn block-sparse attention forward for B200 (sm_100a)."""
