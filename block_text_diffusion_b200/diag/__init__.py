"""Performance diagnostics (not used by the library)."""
