"""libgdr binding placeholder (filled in with the C-ABI binding)."""
