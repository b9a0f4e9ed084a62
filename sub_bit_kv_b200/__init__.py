"""LoopVQ KV-cache codec and coded-cache decode attention for NVIDIA B200 (sm_100a)."""
