// Kernels for block size 512, f16 values.
#define RQ_D 512
#define RQ_BF16 0
#include "rq_quant_inst.cuh"
