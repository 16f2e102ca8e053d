"""B200-native tile-sparse attention for video diffusion transformers."""
