"""B200-native (sm_100a) Multi-head Latent Attention decode."""
