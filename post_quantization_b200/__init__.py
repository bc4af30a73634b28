"""KronQ per-layer quantization hot path for B200 (sm_100a)."""
