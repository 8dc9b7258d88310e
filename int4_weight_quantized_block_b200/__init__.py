"""Packed-INT4 ConvRot quantized linear layer for B200 (sm_100a)."""
