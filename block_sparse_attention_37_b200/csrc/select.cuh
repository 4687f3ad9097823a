// Parameters of the pooling and selection kernels (select.cu).
#pragma once

#include "common.cuh"

namespace bsa {

struct PoolParams {
  int B, H, N, block_q, block_k, nQB, nKB;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  float* qbar;  // [B,H,nQB,d]
  float* kbar;  // [B,H,nKB,d]
};

struct SelectParams {
  int method;
  int B, H, N, block_q, block_k, nQB, nKB;
  int ntbq, ntbk, keep_text;
  int n_groups;
  bsa_key_group groups[4];
  const float* qbar;
  const float* kbar;
  // FULL_SCORE: block sums of softmax, [B*H*nQB*parts][nKB]; the `parts`
  // rows of a query block add up to its row of A' (one per 128-row query
  // tile of the block; a ragged last block has fewer, its others unread)
  const float* apool;
  int parts, nQT;
  int32_t* cnt;
  int32_t* idx;
  uint8_t* flag;
  uint8_t* bitmap;
  int max_k;
};

cudaError_t launch_block_pool(int d, const PoolParams& p, cudaStream_t stream);
cudaError_t launch_select(int d, const SelectParams& p, cudaStream_t stream);

}  // namespace bsa
