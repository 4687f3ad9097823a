// FP8 (e4m3) operands of the forward (jsqmd.com GNA article, Blackwell adaptation: FP8 for
// more tensor throughput; the article gives no scheme). Each 64-token block of each (b, h) of
// Q, K and V gets its own scale s = amax / 448 (1 for an all-zero block); the stored code of x
// is e4m3(x * r) with r = 448 / amax taken once per block in fp32, the product rounded to fp32
// and then to e4m3 (nearest even, saturating at 448). Q and K keep their [B, H, N, d] layout at
// one byte a value. V is written transposed per head, [B, H, d, Nt] with Nt = N rounded up to
// 16 (the columns in [N, Nt) are zero), so that a 128-key tile of it is the K-major B operand
// of the PV contraction. d = 128.
#include "quant.cuh"

namespace bsa {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float amax8(const uint4& v) {
  float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
  return fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
}

__device__ __forceinline__ uint2 codes8(const uint4& v, float r) {
  uint2 o;
  o.x = (uint32_t)e4m3x2(bf16_lo(v.x) * r, bf16_hi(v.x) * r) |
        ((uint32_t)e4m3x2(bf16_lo(v.y) * r, bf16_hi(v.y) * r) << 16);
  o.y = (uint32_t)e4m3x2(bf16_lo(v.z) * r, bf16_hi(v.z) * r) |
        ((uint32_t)e4m3x2(bf16_lo(v.w) * r, bf16_hi(v.w) * r) << 16);
  return o;
}

// block-wide max of one value per thread (256 threads)
__device__ __forceinline__ float block_max256(float m, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
  return m;
}

// Q and K: one CTA per (64-token block, b*h, tensor); 64 rows x 128 values = 1024 chunks of
// 16 bytes, four per thread, all loaded before the block max is known
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantParams p) {
  __shared__ float red[8];
  const int blk = blockIdx.x, t = blockIdx.z;
  const long long bh = blockIdx.y;
  const size_t base = ((size_t)bh * p.N + (size_t)blk * 64) * 128;
  const uint4* src = reinterpret_cast<const uint4*>((t == 0 ? p.q : p.k) + base);
  uint2* dst = reinterpret_cast<uint2*>((t == 0 ? p.q8 : p.k8) + base);
  const int rows = min(64, p.N - blk * 64);
  const int n16 = rows * 16;
  uint4 v[4];
  float m = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = threadIdx.x + 256 * u;
    v[u] = c < n16 ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    m = fmaxf(m, amax8(v[u]));
  }
  m = block_max256(m, red);
  const float r = m > 0.f ? 448.f / m : 1.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = threadIdx.x + 256 * u;
    if (c < n16) dst[c] = codes8(v[u], r);
  }
  if (threadIdx.x == 0) (t == 0 ? p.sq : p.sk)[bh * p.nS + blk] = m > 0.f ? m / 448.f : 1.f;
}

// Row pitch of the staged V codes: a multiple of 8 (every key row is written with 8-byte
// stores) that is not a multiple of 128, so the column reads of the transpose spread over banks.
constexpr int kStPitch = 136;

// V: one CTA per (128-key tile, b*h). The tile's two 64-key blocks are scaled on their own,
// staged as codes [key][channel] (row pitch kStPitch), then written transposed: channel c's 128
// codes of the tile are one contiguous 128-byte run of v8t
__global__ void __launch_bounds__(256) quant_vt_kernel(QuantParams p) {
  __shared__ float red[8];
  __shared__ __align__(16) uint8_t st[128 * kStPitch];
  const int tile = blockIdx.x;
  const long long bh = blockIdx.y;
  const int key0 = tile * 128;
  const uint4* src = reinterpret_cast<const uint4*>(p.v + ((size_t)bh * p.N + key0) * 128);
  const int keys = min(128, p.N - key0);
  // thread -> (key = i / 16, chunk = i % 16) for i = threadIdx.x + 256 u; u < 4 covers 64 keys,
  // the first half (u = 0, 1) and the second half (u = 2, 3) of the tile's 128 keys per pass
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint4 v[4];
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = threadIdx.x + 256 * u;     // 0 .. 1023: 64 keys x 16 chunks
      const int key = half * 64 + (i >> 4);
      v[u] = key < keys ? __ldg(src + (size_t)key * 16 + (i & 15)) : make_uint4(0u, 0u, 0u, 0u);
      m = fmaxf(m, amax8(v[u]));
    }
    m = block_max256(m, red);
    const float r = m > 0.f ? 448.f / m : 1.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = threadIdx.x + 256 * u;
      const int key = half * 64 + (i >> 4);
      *reinterpret_cast<uint2*>(st + key * kStPitch + (i & 15) * 8) = codes8(v[u], r);
    }
    if (threadIdx.x == 0 && tile * 2 + half < p.nS) p.sv[bh * p.nS + tile * 2 + half] = m > 0.f ? m / 448.f : 1.f;
    __syncthreads();  // red[] is reused by the second half; st[] is read below
  }
  // transposed write: thread -> (channel c = j / 8, 16-key group g = j % 8) for j = threadIdx.x + 256 u
  uint8_t* dst = p.v8t + (size_t)bh * 128 * p.Nt;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = threadIdx.x + 256 * u;       // 0 .. 1023: 128 channels x 8 groups
    const int c = j >> 3, g = j & 7;
    const int k0 = key0 + g * 16;
    if (k0 >= p.Nt) continue;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t x = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) x |= (uint32_t)st[(g * 16 + q * 4 + b) * kStPitch + c] << (8 * b);
      w[q] = x;
    }
    // Nt is a multiple of 16 and k0 a multiple of 16: the 16 bytes stay inside the row
    *reinterpret_cast<uint4*>(dst + (size_t)c * p.Nt + k0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

cudaError_t launch_quant_fp8(const QuantParams& p, cudaStream_t stream) {
  dim3 g1((unsigned)p.nS, (unsigned)p.BH, 2);
  quant_rows_kernel<<<g1, 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((unsigned)((p.N + 127) / 128), (unsigned)p.BH);
  quant_vt_kernel<<<g2, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsa
