"""B200-native fp8 MQA indexer (logits + top-k)."""
