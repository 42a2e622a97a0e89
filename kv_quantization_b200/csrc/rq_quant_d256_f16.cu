// Kernels for block size 256, f16 values.
#define RQ_D 256
#define RQ_BF16 0
#include "rq_quant_inst.cuh"
