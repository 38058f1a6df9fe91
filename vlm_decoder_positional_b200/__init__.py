"""Canvas M-RoPE for the Qwen3.5-hybrid decoder of MiniCPM-V-4.7-1B, on B200."""
