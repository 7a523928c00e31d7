"""B200-native grouped-query attention: decode and causal prefill behind a C ABI."""
