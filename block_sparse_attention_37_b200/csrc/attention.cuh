// Parameters and launchers of the tcgen05 attention kernels (forward.cu, score.cu).
#pragma once

#include "common.cuh"

namespace bsa {

enum { KIND_LSE = 1, KIND_POOL = 2, KIND_TLSE = 3 };

// 64-key segments per sequence the per-CTA schedule can hold: N <= 131072.
constexpr int kMaxSeg = 2048;

struct AttnParams {
  int B, H, N;
  int block_q, block_k, n_text;
  int nQB, nKB, nQT, nSeg;
  // block list (SPARSE heads)
  const int32_t* cnt;
  const int32_t* idx;
  const uint8_t* flag;
  int max_k;
  const int32_t* head_mode;  // [H] (forward only)
  const float* cache_in;     // [B,H,N,d] fp32, SKIP heads
  float* cache_out;          // [B,H,N,d] fp32 or null
  const float* bias;         // [H,nQB,nKB] fp32 or null (natural-log units)
  float scale_log2;          // scale * log2(e)
  __nv_bfloat16* O;          // [B,H,N,d]
  float* lse;                // [B,H,N] log2-domain row LSE (LSE out, POOL in)
  float* apool;              // [B,H,nQB,nKB] block sums of softmax (POOL out)
  // TLSE: per 128-row query tile (CTA c of the launch) a [T][128] slab of
  // per-tile row LSEs, T = ceil(N/128); the launch covers the query blocks
  // u0, u0 + 1, ... in (b, h, I) order, block_q / 128 CTAs per block
  float* tlse;
  long long u0;
  int has_gna;
  GnaDev g;
  // failure detection: the limit of every pipeline wait, and a tile whose K
  // the producer withholds (-1: none) so that a test can make a wait run out
  uint64_t wait_limit_ns;
  int withhold_tile;
  // e4m3 forward: dequantisation scales per 64-token block, [B*H, nSeg]
  const float* sq;
  const float* sk;
  const float* sv;
};

// The forward: two 128-row query tiles per CTA (forward.cu); grid = B*H*ceil(N/256).
cudaError_t launch_forward(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const CUtensorMap& o, const AttnParams& p, int grid, cudaStream_t stream);

// The e4m3 forward (d = 128): Q and K codes [B*H, N, 128] bytes, V codes
// transposed [B*H, 128, N rounded up to 16] bytes, scales in p.sq/sk/sv.
cudaError_t launch_forward_fp8(const CUtensorMap& q8, const CUtensorMap& k8, const CUtensorMap& v8t,
                               const CUtensorMap& o, const AttnParams& p, int grid, cudaStream_t stream);

// The score passes of the full-score selection (score.cu). KIND_LSE and
// KIND_POOL: grid = B*H*ceil(N/128). KIND_TLSE: grid = (query blocks in the
// chunk) * block_q / 128.
cudaError_t launch_score(int d, int kind, const CUtensorMap& q, const CUtensorMap& k, const AttnParams& p,
                         int grid, cudaStream_t stream);

}  // namespace bsa
