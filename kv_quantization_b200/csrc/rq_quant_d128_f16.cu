// Kernels for block size 128, f16 values.
#define RQ_D 128
#define RQ_BF16 0
#include "rq_quant_inst.cuh"
