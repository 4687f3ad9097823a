// Parameters of the block-list builder (mask.cu).
#pragma once

#include "common.cuh"

namespace bsa {

struct MaskParams {
  int kind;  // BSA_MASK_ARROW / BSA_MASK_GNA
  int B, H, nQB, nKB, ntb;
  const int32_t* head_mode;
  const int32_t* window;
  int32_t* cnt;
  int32_t* idx;
  uint8_t* flag;
  uint8_t* bitmap;
  int max_k;
  GnaDev g;
};

cudaError_t launch_build_mask(const MaskParams& p, cudaStream_t stream);

}  // namespace bsa
