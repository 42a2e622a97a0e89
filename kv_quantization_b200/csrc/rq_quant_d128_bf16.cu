// Kernels for block size 128, bf16 values.
#define RQ_D 128
#define RQ_BF16 1
#include "rq_quant_inst.cuh"
