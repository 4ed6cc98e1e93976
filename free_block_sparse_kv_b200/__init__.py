"""Block-sparse attention with skipped-block compensation on NVIDIA B200 (sm_100a)."""
