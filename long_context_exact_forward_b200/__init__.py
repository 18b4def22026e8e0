"""Ring Attention exact forward on B200 (placeholder; the binding is added with the library)."""
