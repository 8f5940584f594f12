"""Blackwell-native (sm_100a) MLA decoding over a paged latent KV cache."""
