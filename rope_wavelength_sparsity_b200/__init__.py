"""Per-RoPE-wavelength windowed causal attention for NVIDIA B200 (sm_100a)."""
