"""B200-native DSpark draft MLA attention (sm_100a CUDA kernels behind a C ABI)."""
