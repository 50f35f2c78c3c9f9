"""B200-native Mamba-2 SSD scan: chunked forward and decode step (sm_100a)."""
