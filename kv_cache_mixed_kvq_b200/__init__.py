"""Key-priority mixed-precision KV-cache quantization and decode attention for B200."""
