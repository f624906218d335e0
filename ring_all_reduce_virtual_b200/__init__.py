"""Ring all-reduce over N virtual ranks on one B200 (placeholder; the
binding to the CUDA library is added with the library)."""
