"""B200-native weight-only ternary linear layer (W1.58A16): packing, the decode GEMV and
prefill GEMM on packed planes, and bit accounting, behind the C-ABI library libtern.so."""
