// Kernels for block size 256, bf16 values.
#define RQ_D 256
#define RQ_BF16 1
#include "rq_quant_inst.cuh"
