"""Quantized KV-cache handoff and decode attention for B200 (placeholder)."""
