"""B200-native DeepSeek Sparse Attention (DSA) forward: lightning indexer,
per-row top-k and sparse MLA in MQA mode, as hand-written sm_100a CUDA kernels
behind the C ABI in include/dsa.h."""
