"""winattn: fused window attention for vision transformers on B200 (sm_100a)."""
