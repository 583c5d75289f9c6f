"""B200-native decode attention over a paged KV cache (GQA, GTA, GLA/MLA)."""
