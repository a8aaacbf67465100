"""W4A16 for B200: placeholder, replaced by the binding below."""
