// Kernels for block size 64, bf16 values.
#define RQ_D 64
#define RQ_BF16 1
#include "rq_quant_inst.cuh"
