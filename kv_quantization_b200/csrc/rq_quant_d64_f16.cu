// Kernels for block size 64, f16 values.
#define RQ_D 64
#define RQ_BF16 0
#include "rq_quant_inst.cuh"
