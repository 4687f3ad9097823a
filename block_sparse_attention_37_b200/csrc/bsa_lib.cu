// Single translation unit of libbsa.so: the kernels share the device error
// word, so they are compiled as one module.
#include "api.cu"
#include "forward.cu"
#include "score.cu"
#include "mask.cu"
#include "permute.cu"
#include "select.cu"
#include "select_static.cu"
#include "quant.cu"
#include "plan.cu"
#include "schedule.cu"
