"""HSTU layer hot path for B200 (sm_100a)."""
