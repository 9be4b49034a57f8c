"""GTR token-mixer forward pass for B200 (sm_100a)."""
