"""B200-native HSTU jagged layer: tcgen05/TMA CUDA kernels behind a C ABI (libhstu_b200.so)."""
