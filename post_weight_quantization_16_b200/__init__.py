"""GPTQ per-layer quantization solve on B200 (sm_100a)."""
