"""B200-native sequence/head-parallel attention: C-ABI CUDA library binding."""
