"""Placeholder; replaced by the ctypes binding once the library exists."""
