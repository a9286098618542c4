"""Star Attention two-phase hot path, B200-native."""
