"""B200-native DSA sparse-attention step: lightning indexer -> top-k -> sparse MLA."""
