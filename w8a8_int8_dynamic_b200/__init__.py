"""B200-native W8A8 int8-dynamic linear layers (placeholder; the binding is added with the library)."""
