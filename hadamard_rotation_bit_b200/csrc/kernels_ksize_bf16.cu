// bf16-input instantiations of the K * 2^m rotation kernels.
#define HADQ_KSIZE_BF16 1
#include "kernels_ksize.cu"
