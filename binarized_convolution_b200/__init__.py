"""B200-native binary convolution (XNOR / AND / binaryWeights) behind a C-ABI library."""
