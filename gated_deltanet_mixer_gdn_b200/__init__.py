"""B200-native Gated DeltaNet token mixer (sm_100a CUDA kernels behind a C ABI)."""
