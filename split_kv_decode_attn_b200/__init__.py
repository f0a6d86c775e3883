"""B200-native split-KV decode attention (Flash-Decoding)."""
