"""Row-wise scaled 2:4 sparse FP8 linear for B200 (sm_100a)."""
