"""QLoRA NF4 quantized linear for NVIDIA B200 (sm_100a)."""
