"""B200-native MoE layer forward (route -> dispatch -> SwiGLU grouped GEMM -> combine ->
load statistics) behind a C-ABI library; this package is its thin Python binding."""
