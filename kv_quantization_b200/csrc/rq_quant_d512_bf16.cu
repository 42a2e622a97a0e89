// Kernels for block size 512, bf16 values.
#define RQ_D 512
#define RQ_BF16 1
#include "rq_quant_inst.cuh"
