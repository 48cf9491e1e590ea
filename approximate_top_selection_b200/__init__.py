"""Two-stage bucketed approximate top-k on B200 (sm_100a)."""
