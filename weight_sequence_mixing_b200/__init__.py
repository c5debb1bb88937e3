"""B200 (sm_100a) TTT-layer forward pass: a C-ABI CUDA library and its Python binding."""
