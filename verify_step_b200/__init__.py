"""B200-native speculative-decoding verify step (see include/sd_verify.h for the C ABI)."""
