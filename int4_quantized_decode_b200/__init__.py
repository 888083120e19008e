"""libqgemv: B200-native weight-only quantized GEMV for LLM decode."""
