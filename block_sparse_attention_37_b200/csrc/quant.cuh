// Parameters of the e4m3 quantisation kernels (quant.cu).
#pragma once

#include "common.cuh"

namespace bsa {

struct QuantParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  uint8_t* q8;   // [BH, N, 128]
  uint8_t* k8;   // [BH, N, 128]
  uint8_t* v8t;  // [BH, 128, Nt]
  float* sq;     // [BH, nS]
  float* sk;
  float* sv;
  long long BH;
  int N, Nt, nS;
};

cudaError_t launch_quant_fp8(const QuantParams& p, cudaStream_t stream);

}  // namespace bsa
