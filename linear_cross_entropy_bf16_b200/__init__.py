"""Fused linear cross-entropy forward for NVIDIA B200 (sm_100a)."""
