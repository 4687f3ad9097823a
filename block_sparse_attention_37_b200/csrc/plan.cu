// Head-wise compression plan (DiTFastAttnV2, "efficient compression plan
// search"): the single-layer relative squared error of a method's output per
// head (bsa_rse, an HBM-bound reduction on the GPU) and the exact plan under
// an error budget (bsa_plan_heads, host only).
#include <algorithm>
#include <cmath>
#include <vector>

#include "common.cuh"

namespace bsa {

// bf16 pairs of one 16-byte chunk of each tensor into the three fp64 sums.
// bf16 -> fp32 is exact (the bf16 bits are the high half of the fp32), and so
// is fp32 -> fp64.
__device__ __forceinline__ void rse_add(const uint4& a, const uint4& o, double& num, double& s, double& ss) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double a0 = (double)__uint_as_float(aw[k] << 16), a1 = (double)__uint_as_float(aw[k] & 0xffff0000u);
    const double o0 = (double)__uint_as_float(ow[k] << 16), o1 = (double)__uint_as_float(ow[k] & 0xffff0000u);
    num += (a0 - o0) * (a0 - o0) + (a1 - o1) * (a1 - o1);
    s += o0 + o1;
    ss += o0 * o0 + o1 * o1;
  }
}

// Per head h (blockIdx.y) and batch item b (blockIdx.z): sum (y_m - y_o)^2,
// sum y_o and sum y_o^2 over the item's tokens and channels, in fp64. The
// (b, h) slab is one contiguous run of 16-byte chunks (8 bf16); the blocks of
// the slab grid-stride over it with four chunk pairs in flight per thread. A
// block reduces with warp shuffles and adds its three partial sums to
// sums[3h .. 3h + 2] atomically.
__global__ void __launch_bounds__(256) rse_kernel(const uint4* __restrict__ ym, const uint4* __restrict__ yo,
                                                  int H, long long chunks_per_bh, double* sums) {
  const int h = blockIdx.y;
  const long long base = ((long long)blockIdx.z * H + h) * chunks_per_bh;
  const uint4* pa = ym + base;
  const uint4* po = yo + base;
  double num = 0.0, s = 0.0, ss = 0.0;
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < chunks_per_bh; i += 4 * stride) {
    uint4 a[4], o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a[u] = __ldg(pa + i + u * stride);
      o[u] = __ldg(po + i + u * stride);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) rse_add(a[u], o[u], num, s, ss);
  }
  for (; i < chunks_per_bh; i += stride) rse_add(__ldg(pa + i), __ldg(po + i), num, s, ss);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_down_sync(0xffffffffu, num, off);
    s += __shfl_down_sync(0xffffffffu, s, off);
    ss += __shfl_down_sync(0xffffffffu, ss, off);
  }
  __shared__ double part[3][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    part[0][warp] = num;
    part[1][warp] = s;
    part[2][warp] = ss;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[threadIdx.x][w];
    atomicAdd(&sums[3 * h + threadIdx.x], t);
  }
}

// out[h] = num / (sum y_o^2 - (sum y_o)^2 / n): the denominator is
// sum (y_o - mean)^2 written with the sums the reduction keeps.
__global__ void rse_finalize(const double* sums, double* out, int H, double n) {
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const double num = sums[3 * h], s = sums[3 * h + 1], ss = sums[3 * h + 2];
    out[h] = num / (ss - s * s / n);
  }
}

}  // namespace bsa

using namespace bsa;

extern "C" int bsa_rse(const bsa_dims* dims, const void* y_m, const void* y_o, double* out, void* stream) {
  if (!dims || !y_m || !y_o || !out) return BSA_ERR_INVALID_ARG;
  if (dims->B < 1 || dims->H < 1 || dims->N < 1 || dims->d < 1) return BSA_ERR_INVALID_ARG;
  if (!aligned16(y_m) || !aligned16(y_o)) return BSA_ERR_INVALID_ARG;
  const long long nd = (long long)dims->N * dims->d;
  if (nd % 8 != 0) return BSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* sums = out + dims->H;
  if (cudaMemsetAsync(sums, 0, sizeof(double) * 3 * (size_t)dims->H, st) != cudaSuccess) return BSA_ERR_CUDA;
  // one grid slab per (b, h), with enough blocks per slab to give every SM
  // about eight blocks
  if (dims->B > 65535 || dims->H > 65535) return BSA_ERR_UNSUPPORTED;
  const long long slabs = (long long)dims->B * dims->H;
  long long bx = (8ll * num_sms() + slabs - 1) / slabs;
  const long long need = (nd / 8 + 255) / 256;
  if (bx > need) bx = need;
  if (bx < 1) bx = 1;
  rse_kernel<<<dim3((unsigned)bx, (unsigned)dims->H, (unsigned)dims->B), 256, 0, st>>>(
      static_cast<const uint4*>(y_m), static_cast<const uint4*>(y_o), dims->H, nd / 8, sums);
  if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  rse_finalize<<<1, 256, 0, st>>>(sums, out, dims->H, (double)dims->B * (double)nd);
  return cuda_status(cudaGetLastError());
}

// Minimum total cost with sum of errors <= delta and every error <= cap:
// best[C] is the least error sum of the heads so far at total cost exactly C
// (errors added in head order); the plan is the smallest C whose best is
// within the budget, traced back through the per-head choices.
extern "C" int bsa_plan_heads(int32_t H, int32_t M, const double* rse, const int64_t* cost, double delta, double c,
                              int32_t* choice, int64_t* total_cost) {
  if (H < 1 || M < 1 || M > 32767 || !rse || !cost || !choice) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(delta) || !std::isfinite(c) || delta < 0.0 || c < 0.0) return BSA_ERR_INVALID_ARG;
  const double cap = c * delta / H;
  long long max_total = 0;
  for (int h = 0; h < H; ++h) {
    long long mx = 0;
    for (int m = 0; m < M; ++m) {
      if (cost[(size_t)h * M + m] < 0) return BSA_ERR_INVALID_ARG;
      if (cost[(size_t)h * M + m] > mx) mx = cost[(size_t)h * M + m];
    }
    max_total += mx;
  }
  // the tables hold H * (max_total + 1) choices: keep them within 2^28
  // entries (costs in coarse units, such as blocks, stay far below)
  if ((long long)H * (max_total + 1) > (1ll << 28)) return BSA_ERR_UNSUPPORTED;
  const size_t W = (size_t)max_total + 1;
  const double inf = INFINITY;
  std::vector<double> best(W, inf), next(W);
  std::vector<int16_t> pick((size_t)H * W, -1);
  best[0] = 0.0;
  for (int h = 0; h < H; ++h) {
    std::fill(next.begin(), next.end(), inf);
    int16_t* ph = pick.data() + (size_t)h * W;
    for (int m = 0; m < M; ++m) {
      const double e = rse[(size_t)h * M + m];
      if (!(e <= cap)) continue;  // over the per-head cap, or NaN
      const size_t k = (size_t)cost[(size_t)h * M + m];
      for (size_t C = k; C < W; ++C) {
        if (best[C - k] == inf) continue;
        const double v = best[C - k] + e;
        if (v < next[C]) {  // ties keep the earlier method
          next[C] = v;
          ph[C] = (int16_t)m;
        }
      }
    }
    best.swap(next);
  }
  size_t Cb = W;
  for (size_t C = 0; C < W; ++C)
    if (best[C] <= delta) {
      Cb = C;
      break;
    }
  if (Cb == W) return BSA_ERR_INFEASIBLE;
  size_t C = Cb;
  for (int h = H - 1; h >= 0; --h) {
    const int m = pick[(size_t)h * W + C];
    choice[h] = m;
    C -= (size_t)cost[(size_t)h * M + m];
  }
  if (total_cost) *total_cost = (int64_t)Cb;
  return BSA_OK;
}
