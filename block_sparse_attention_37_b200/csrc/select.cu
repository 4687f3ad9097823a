// Content-driven block selection.
//  * block_pool_kernel: mean of every 64/128/256-token block of Q and K in
//    fp32 (lmnt.cn BSA post, section 2.2, mean-pooled block vectors). HBM
//    bound: one bulk copy of the block's rows into shared memory per CTA.
//  * select_kernel: per (b, h, query block) row, the score of every KV block
//    (pooled dot product, or the SparseD avg-pooled softmax mass from the
//    block sums of A' the score kernel writes), then an exact cut per key
//    group (descending score, ties to the lower index) and an ascending
//    block list.
#include "select.cuh"
#include "tiles.cuh"

namespace bsa {

// grid: (nB, B*H, 2 tensors); block 256. out[t][bh][I][:] = mean of block I.
// The block's rows are one contiguous run of rows * D * 2 bytes: one thread
// moves it into shared memory with bulk copies of up to kPoolChunkRows rows
// (no registers hold data in flight, so many CTAs per SM keep HBM busy),
// then every thread adds its 16-byte column chunk over rows rr, rr + RPI, ...
// in order, and the RPI partial rows are added in order.
constexpr int kPoolChunkRows = 256;

template <int D>
__global__ void __launch_bounds__(256) block_pool_kernel(PoolParams p) {
  constexpr int CH = D / 8;           // 16-byte chunks per row
  constexpr int RPI = 256 / CH;       // rows per step
  extern __shared__ __align__(128) uint8_t rows_smem[];  // [rows][D] bf16
  __shared__ float red[RPI][D + 1];
  __shared__ __align__(8) uint64_t full;
  __shared__ int no_abort;
  // the selection kernel after this one may be scheduled now (it waits for
  // this grid's completion before reading the pooled vectors)
  asm volatile("griddepcontrol.launch_dependents;");
  const int I = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int bs = which ? p.block_k : p.block_q;
  const int nb = which ? p.nKB : p.nQB;
  if (I >= nb) return;
  const __nv_bfloat16* src = (which ? p.K : p.Q) + ((size_t)bh * p.N) * D;
  float* dst = (which ? p.kbar : p.qbar) + ((size_t)bh * nb + I) * D;
  const int r0 = I * bs;
  const int rows = min(bs, p.N - r0);
  if (threadIdx.x == 0) {
    no_abort = 0;
    mbar_init(&full, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const int c = threadIdx.x % CH, rr = threadIdx.x / CH;
  const uint4* rowp = reinterpret_cast<const uint4*>(rows_smem) + c;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  uint32_t phase = 0u;
  // chunks start at multiples of kPoolChunkRows (a multiple of RPI), so each
  // thread still visits its rows rr, rr + RPI, ... in order
  for (int c0 = 0; c0 < rows; c0 += kPoolChunkRows) {
    const int n = min(kPoolChunkRows, rows - c0);
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();  // the previous chunk's reads come before the copy over them
      mbar_arrive_expect_tx(&full, (uint32_t)n * D * 2);
      bulk_load_1d(rows_smem, src + (size_t)(r0 + c0) * D, (uint32_t)n * D * 2, &full);
    }
    if (!mbar_wait(&full, phase, &no_abort)) {
      // the copy never landed: wait (bounded) so nothing is in flight at exit
      if (threadIdx.x == 0) {
        record_error(BSA_DEVERR_TIMEOUT);
        mbar_drain(&full, phase);
      }
      return;
    }
    phase ^= 1u;
    for (int r = rr; r < n; r += RPI) {
      const uint4 v = rowp[(size_t)r * CH];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        acc[2 * j] += f.x;
        acc[2 * j + 1] += f.y;
      }
    }
    __syncthreads();  // every thread is done with the chunk before the next copy
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

// An unsigned key whose order is the float order of a non-NaN score; -0 and
// +0 (equal as floats) map to one key.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA per (b, h, query block). Block 256 threads.
template <int D>
__global__ void __launch_bounds__(256) select_kernel(SelectParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernel's output is complete
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
    const int np = min(p.parts, p.nQT - I * p.parts);  // partial rows that exist
    for (int J = tid; J < p.nKB; J += 256) {
      const int nk = min(p.block_k, p.N - J * p.block_k);
      float a = 0.f;
      for (int j = 0; j < np; ++j) a += p.apool[((size_t)row * p.parts + j) * p.nKB + J];
      sc[J] = sanitize(a / ((float)nq * (float)nk));
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
// leaves the full dot product of key J0 + i in lane i. The cut of each group
// is a warp-wide radix select of its k-th largest score (32 counting steps,
// linear in the group's size); it and the ascending compaction are
// warp-level (no CTA-wide barriers).
constexpr int kRowsPerCta = 8;
constexpr int kRowsMaxKB = 1024;


// Keep the k largest scores of sc[b, e) (0 < k < e - b <= 32 * NPL), ties to
// the lower index, by a warp-wide radix select of the k-th largest order key,
// one bit at a time from the top. After the loop `prefix` is that key and
// `kr` its rank among the keys equal to it: keys above it are kept, and of
// the keys equal to it the kr with the lowest block indices - the same k
// blocks as ranking by descending score with ties to the lower index. Each
// lane holds the keys of b + lane + 32q in registers; padding keys are 0,
// below every score's key (order_key(-inf) = 0x007fffff).
template <int NPL>
__device__ __forceinline__ void radix_cut(const float* sc, uint8_t* keep, int b, int e, int k, int lane) {
  uint32_t key[NPL];
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int J = b + lane + 32 * q;
    key[q] = J < e ? order_key(sc[J]) : 0u;
  }
  uint32_t prefix = 0u, pmask = 0u;
  int kr = k;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t bm = 1u << bit, want = prefix | bm, m = pmask | bm;
    int c = 0;
#pragma unroll
    for (int q = 0; q < NPL; ++q) c += (key[q] & m) == want;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= kr)
      prefix = want;
    else
      kr -= c;
    pmask = m;
  }
  int taken = 0;
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int J = b + lane + 32 * q;
    const bool eq = key[q] == prefix;  // padding keys are never equal (prefix >= 0x007fffff)
    const unsigned be = __ballot_sync(0xffffffffu, eq);
    if (key[q] > prefix || (eq && taken + __popc(be & ((1u << lane) - 1u)) < kr)) keep[J] = 1;
    taken += __popc(be);
  }
}

template <int D>
__global__ void __launch_bounds__(256) select_rows_kernel(SelectParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernel's output is complete
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
    const int np = min(p.parts, p.nQT - I * p.parts);  // partial rows that exist
    for (int J = lane; J < p.nKB; J += 32) {
      const int nk = min(p.block_k, p.N - J * p.block_k);
      float a = 0.f;
      for (int j = 0; j < np; ++j) a += p.apool[((size_t)row * p.parts + j) * p.nKB + J];
      sc[J] = sanitize(a / ((float)nq * (float)nk));
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
      if (k >= e - b) {
        for (int J = b + lane; J < e; J += 32) keep[J] = 1;
        continue;
      }
      if (k <= 0) continue;
      const int per = (e - b + 31) >> 5;  // keys per lane
      if (per <= 1)
        radix_cut<1>(sc, keep, b, e, k, lane);
      else if (per <= 2)
        radix_cut<2>(sc, keep, b, e, k, lane);
      else if (per <= 4)
        radix_cut<4>(sc, keep, b, e, k, lane);
      else if (per <= 8)
        radix_cut<8>(sc, keep, b, e, k, lane);
      else if (per <= 16)
        radix_cut<16>(sc, keep, b, e, k, lane);
      else
        radix_cut<32>(sc, keep, b, e, k, lane);
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

template <int D>
static cudaError_t launch_block_pool_d(const PoolParams& p, cudaStream_t stream) {
  // dynamic shared memory: one chunk of the larger block's rows (at most 64 KB)
  static DeviceOnce once;
  const cudaError_t e = once.run([&]() -> cudaError_t {
    return cudaFuncSetAttribute(block_pool_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kPoolChunkRows * D * 2);
  });
  if (e != cudaSuccess) return e;
  const int rows = min(max(p.block_q, p.block_k), kPoolChunkRows);
  dim3 grid(max(p.nQB, p.nKB), p.B * p.H, 2);
  block_pool_kernel<D><<<grid, 256, (size_t)rows * D * 2, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_block_pool(int d, const PoolParams& p, cudaStream_t stream) {
  return d == 64 ? launch_block_pool_d<64>(p, stream) : launch_block_pool_d<128>(p, stream);
}

// A programmatic dependent launch: the selection grid may be scheduled while
// the kernel before it (pooling or the score pass) finishes; its kernels
// wait on griddepcontrol.wait before reading anything that kernel wrote.
template <class K>
static cudaError_t launch_dependent(K kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                                   const SelectParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

cudaError_t launch_select(int d, const SelectParams& p, cudaStream_t stream) {
  if (p.nKB <= kRowsMaxKB) {
    const size_t smem = (size_t)kRowsPerCta * p.nKB * (sizeof(float) + 1);
    const unsigned grid = (unsigned)((size_t)p.B * p.H * ((p.nQB + kRowsPerCta - 1) / kRowsPerCta));
    return d == 64 ? launch_dependent(select_rows_kernel<64>, grid, 32 * kRowsPerCta, smem, stream, p)
                   : launch_dependent(select_rows_kernel<128>, grid, 32 * kRowsPerCta, smem, stream, p);
  }
  const size_t smem = (size_t)p.nKB * sizeof(float) + (size_t)p.nKB;
  const unsigned grid = (unsigned)((size_t)p.B * p.H * p.nQB);
  return d == 64 ? launch_dependent(select_kernel<64>, grid, 256, smem, stream, p)
                 : launch_dependent(select_kernel<128>, grid, 256, smem, stream, p);
}

}  // namespace bsa
