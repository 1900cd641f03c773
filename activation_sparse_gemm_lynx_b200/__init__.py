"""B200-native RT-Lynx online 2:4 activation-sparse linear layer (placeholder)."""
