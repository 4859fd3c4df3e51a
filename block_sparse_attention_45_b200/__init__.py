"""B200-native dynamic block-sparse attention for video diffusion transformers."""
