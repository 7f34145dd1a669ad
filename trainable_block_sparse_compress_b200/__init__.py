"""InfLLM v2 block-sparse attention for B200 (sm_100a)."""
