// Parameters of the tile permutation kernels (permute.cu).
#pragma once

#include "common.cuh"

namespace bsa {

struct PermuteParams {
  int n_tensors;
  long long BH;
  int d;
  int n_raster;  // n_text + prod(grid)
  int n_tiled;   // text_span + n_tiles * vol
  const __nv_bfloat16* in[4];
  __nv_bfloat16* out[4];
  GnaDev g;
};

cudaError_t launch_permute(bool forward, const PermuteParams& p, int num_sms, cudaStream_t stream);

}  // namespace bsa
