// Content-driven block selection.
//  * block_pool_kernel: mean of every 64/128/256-token block of Q and K in
//    fp32 (lmnt.cn BSA post, section 2.2, mean-pooled block vectors). HBM
//    bound: 16-byte coalesced loads, eight blocks of loads in flight per CTA.
//  * select_kernel: per (b, h, query block) row, the score of every KV block
//    (pooled dot product, or the SparseD avg-pooled softmax mass from the
//    attention kernel's POOL pass), then an exact rank-and-cut per key group
//    (descending score, ties to the lower index) and an ascending block list.
#include "select.cuh"

namespace bsa {

// grid: (nB, B*H, 2 tensors); block 256. out[t][bh][I][:] = mean of block I.
template <int D>
__global__ void __launch_bounds__(256) block_pool_kernel(PoolParams p) {
  constexpr int CH = D / 8;           // 16-byte chunks per row
  constexpr int RPI = 256 / CH;       // rows per iteration
  __shared__ float red[RPI][D + 1];
  const int I = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int bs = which ? p.block_k : p.block_q;
  const int nb = which ? p.nKB : p.nQB;
  if (I >= nb) return;
  const __nv_bfloat16* src = (which ? p.K : p.Q) + ((size_t)bh * p.N) * D;
  float* dst = (which ? p.kbar : p.qbar) + ((size_t)bh * nb + I) * D;
  const int r0 = I * bs;
  const int rows = min(bs, p.N - r0);
  const int c = threadIdx.x % CH, rr = threadIdx.x / CH;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int base = 0; base < rows; base += RPI * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = base + u * RPI + rr;
      if (r < rows)
        v[u] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(r0 + r) * D) + c);
      else
        v[u] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        acc[2 * j] += f.x;
        acc[2 * j + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[rr][c * 8 + j] = acc[j];
  __syncthreads();
  for (int col = threadIdx.x; col < D; col += 256) {
    float s = 0.f;
#pragma unroll 4
    for (int q = 0; q < RPI; ++q) s += red[q][col];
    dst[col] = s / (float)rows;
  }
}

__device__ __forceinline__ float sanitize(float x) { return (x == x) ? x : -__int_as_float(0x7f800000); }

// One CTA per (b, h, query block). Block 256 threads.
template <int D>
__global__ void __launch_bounds__(256) select_kernel(SelectParams p) {
  extern __shared__ float sc[];  // [nKB] scores
  __shared__ int warp_tot[8];
  uint8_t* keep = reinterpret_cast<uint8_t*>(sc + p.nKB);
  const int I = blockIdx.x % p.nQB;
  const int bh = blockIdx.x / p.nQB;
  const size_t row = (size_t)bh * p.nQB + I;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (p.method == BSA_SELECT_POOLED_QK) {
    // One warp per key block: the lanes read the pooled key row together
    // (D / 32 consecutive floats each, one coalesced row per load) and
    // reduce the dot product with shuffles.
    constexpr int PL = D / 32;  // floats per lane
    float qr[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) qr[i] = p.qbar[row * D + lane * PL + i];
    const float* kb = p.kbar + (size_t)bh * p.nKB * D;
    // eight key rows per warp in flight at a time (their loads are
    // independent), then the eight reductions
    constexpr int R = 8;
    for (int J0 = warp; J0 < p.nKB; J0 += 8 * R) {
      float kv[R][PL];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int J = J0 + 8 * r;
        const float* kr = kb + (size_t)(J < p.nKB ? J : 0) * D + lane * PL;
        if constexpr (PL == 4) {
          const float4 k4 = __ldg(reinterpret_cast<const float4*>(kr));
          kv[r][0] = k4.x; kv[r][1] = k4.y; kv[r][2] = k4.z; kv[r][3] = k4.w;
        } else {
          const float2 k2 = __ldg(reinterpret_cast<const float2*>(kr));
          kv[r][0] = k2.x; kv[r][1] = k2.y;
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float s = 0.f;
#pragma unroll
        for (int i = PL - 1; i >= 0; --i) s = fmaf(qr[i], kv[r][i], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const int J = J0 + 8 * r;
        if (lane == 0 && J < p.nKB) sc[J] = sanitize(s);
      }
    }
  } else {
    const int nq = min(p.block_q, p.N - I * p.block_q);
    for (int J = tid; J < p.nKB; J += 256) {
      const int nk = min(p.block_k, p.N - J * p.block_k);
      sc[J] = sanitize(p.apool[row * p.nKB + J] / ((float)nq * (float)nk));
    }
  }
  for (int J = tid; J < p.nKB; J += 256) keep[J] = 0;
  __syncthreads();

  const bool full_row = p.keep_text && I < p.ntbq;
  if (full_row) {
    for (int J = tid; J < p.nKB; J += 256) keep[J] = 1;
  } else {
    if (p.keep_text)
      for (int J = tid; J < min(p.ntbk, p.nKB); J += 256) keep[J] = 1;
    for (int g = 0; g < p.n_groups; ++g) {
      const int b = p.groups[g].begin, e = min(p.groups[g].end, p.nKB), k = p.groups[g].k;
      for (int J = b + tid; J < e; J += 256) {
        const float sj = sc[J];
        int rank = 0;
        for (int J2 = b; J2 < e; ++J2) {
          const float s2 = sc[J2];
          rank += (s2 > sj) || (s2 == sj && J2 < J);
        }
        if (rank < k) keep[J] = 1;
      }
    }
  }
  __syncthreads();

  // ascending compaction
  int32_t* idx = p.idx + row * p.max_k;
  uint8_t* flag = p.flag + row * p.max_k;
  int base = 0;
  for (int J0 = 0; J0 < p.nKB; J0 += 256) {
    const int J = J0 + tid;
    const bool kk = J < p.nKB && keep[J];
    const unsigned bal = __ballot_sync(0xffffffffu, kk);
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 8; ++w) {
      before += (w < warp) ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    if (kk) {
      const int pos = base + before + __popc(bal & ((1u << lane) - 1u));
      idx[pos] = J;
      flag[pos] = BSA_BLOCK_FULL;
    }
    if (J < p.nKB && p.bitmap) p.bitmap[row * p.nKB + J] = kk ? BSA_BLOCK_FULL : BSA_BLOCK_NONE;
    base += total;
    __syncthreads();
  }
  for (int e = base + tid; e < p.max_k; e += 256) {
    idx[e] = -1;
    flag[e] = 0;
  }
  if (tid == 0) p.cnt[row] = base;
}

// The same selection with one warp per (b, h, query block) row and eight rows
// per CTA (lists of at most kRowsMaxKB key blocks). The eight rows of a CTA
// are consecutive query blocks of one (b, h), so the pooled key rows they all
// read stay in L1; scores are made 32 keys at a time, each lane accumulating
// its slice of the 32 dot products, and one transpose-reduction (31 shuffles)
// leaves the full dot product of key J0 + i in lane i. Rank-and-cut and the
// ascending compaction are warp-level (no CTA-wide barriers).
constexpr int kRowsPerCta = 8;
constexpr int kRowsMaxKB = 1024;

// After it, lane i holds the sum over the warp of v[i] (v has 32 entries per
// lane): five halving exchange steps, each sending half of the live values.
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      // keep v[i + (upper ? half : 0)], send the other one to the partner lane
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

template <int D>
__global__ void __launch_bounds__(256) select_rows_kernel(SelectParams p) {
  extern __shared__ float rsc[];  // [kRowsPerCta][nKB] scores, then [kRowsPerCta][nKB] keep bytes
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per_bh = (p.nQB + kRowsPerCta - 1) / kRowsPerCta;
  const int bh = blockIdx.x / per_bh;
  const int I = (blockIdx.x % per_bh) * kRowsPerCta + warp;
  if (I >= p.nQB) return;  // warp-uniform; no CTA-wide barrier follows
  const size_t row = (size_t)bh * p.nQB + I;
  float* sc = rsc + warp * p.nKB;
  uint8_t* keep = reinterpret_cast<uint8_t*>(rsc + kRowsPerCta * p.nKB) + warp * p.nKB;

  if (p.method == BSA_SELECT_POOLED_QK) {
    constexpr int PL = D / 32;  // channels per lane
    float qr[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) qr[i] = p.qbar[row * D + lane * PL + i];
    const float* kb = p.kbar + (size_t)bh * p.nKB * D;
    for (int J0 = 0; J0 < p.nKB; J0 += 32) {
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int J = J0 + i < p.nKB ? J0 + i : p.nKB - 1;
        const float* kr = kb + (size_t)J * D + lane * PL;
        float a = 0.f;
        if constexpr (PL == 4) {
          const float4 k4 = __ldg(reinterpret_cast<const float4*>(kr));
          a = fmaf(qr[0], k4.x, fmaf(qr[1], k4.y, fmaf(qr[2], k4.z, qr[3] * k4.w)));
        } else {
          const float2 k2 = __ldg(reinterpret_cast<const float2*>(kr));
          a = fmaf(qr[0], k2.x, qr[1] * k2.y);
        }
        acc[i] = a;
      }
      const float s = transpose_reduce32(acc, lane);
      if (J0 + lane < p.nKB) sc[J0 + lane] = sanitize(s);
    }
  } else {
    const int nq = min(p.block_q, p.N - I * p.block_q);
    for (int J = lane; J < p.nKB; J += 32) {
      const int nk = min(p.block_k, p.N - J * p.block_k);
      sc[J] = sanitize(p.apool[row * p.nKB + J] / ((float)nq * (float)nk));
    }
  }
  for (int J = lane; J < p.nKB; J += 32) keep[J] = 0;
  __syncwarp();

  const bool full_row = p.keep_text && I < p.ntbq;
  if (full_row) {
    for (int J = lane; J < p.nKB; J += 32) keep[J] = 1;
  } else {
    if (p.keep_text)
      for (int J = lane; J < min(p.ntbk, p.nKB); J += 32) keep[J] = 1;
    for (int g = 0; g < p.n_groups; ++g) {
      const int b = p.groups[g].begin, e = min(p.groups[g].end, p.nKB), k = p.groups[g].k;
      for (int J = b + lane; J < e; J += 32) {
        const float sj = sc[J];
        int rank = 0;
        for (int J2 = b; J2 < e; ++J2) {
          const float s2 = sc[J2];
          rank += (s2 > sj) || (s2 == sj && J2 < J);
        }
        if (rank < k) keep[J] = 1;
      }
    }
  }
  __syncwarp();

  // ascending compaction, 32 key blocks at a time
  int32_t* idx = p.idx + row * p.max_k;
  uint8_t* flag = p.flag + row * p.max_k;
  int base = 0;
  for (int J0 = 0; J0 < p.nKB; J0 += 32) {
    const int J = J0 + lane;
    const bool kk = J < p.nKB && keep[J];
    const unsigned bal = __ballot_sync(0xffffffffu, kk);
    if (kk) {
      const int pos = base + __popc(bal & ((1u << lane) - 1u));
      idx[pos] = J;
      flag[pos] = BSA_BLOCK_FULL;
    }
    if (J < p.nKB && p.bitmap) p.bitmap[row * p.nKB + J] = kk ? BSA_BLOCK_FULL : BSA_BLOCK_NONE;
    base += __popc(bal);
  }
  for (int e = base + lane; e < p.max_k; e += 32) {
    idx[e] = -1;
    flag[e] = 0;
  }
  if (lane == 0) p.cnt[row] = base;
}

cudaError_t launch_block_pool(int d, const PoolParams& p, cudaStream_t stream) {
  dim3 grid(max(p.nQB, p.nKB), p.B * p.H, 2);
  if (d == 64)
    block_pool_kernel<64><<<grid, 256, 0, stream>>>(p);
  else
    block_pool_kernel<128><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_select(int d, const SelectParams& p, cudaStream_t stream) {
  if (p.nKB <= kRowsMaxKB) {
    const size_t smem = (size_t)kRowsPerCta * p.nKB * (sizeof(float) + 1);
    const unsigned grid = (unsigned)((size_t)p.B * p.H * ((p.nQB + kRowsPerCta - 1) / kRowsPerCta));
    if (d == 64)
      select_rows_kernel<64><<<grid, 32 * kRowsPerCta, smem, stream>>>(p);
    else
      select_rows_kernel<128><<<grid, 32 * kRowsPerCta, smem, stream>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)p.nKB * sizeof(float) + (size_t)p.nKB;
  const unsigned grid = (unsigned)((size_t)p.B * p.H * p.nQB);
  if (d == 64)
    select_kernel<64><<<grid, 256, smem, stream>>>(p);
  else
    select_kernel<128><<<grid, 256, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsa
