// Fused token permutation + padding between raster order and GNA tile order
// (jsqmd.com GNA article, section 2.2: a dedicated copy kernel replacing
// permute().contiguous(), fused with padding). Every token row is d bf16
// values contiguous in memory, so both directions move whole rows with
// 16-byte vector loads and stores; one thread moves one 16-byte chunk and the
// grid strides over (tensor, b*h, tile-order row, chunk).
#include "permute.cuh"

namespace bsa {

// Raster row feeding tile-order position `pos`, or -1 for a padding slot.
__host__ __device__ __forceinline__ int tile_source_row(const GnaDev& g, int pos) {
  if (pos < g.n_text) return pos;
  if (pos < g.text_span) return -1;
  const int v = pos - g.text_span;
  const int tile = v / g.vol;
  const int l = v - tile * g.vol;
  const int t = (tile / (g.tiles[1] * g.tiles[2])) * g.tile[0] + l / (g.tile[1] * g.tile[2]);
  const int y = ((tile / g.tiles[2]) % g.tiles[1]) * g.tile[1] + (l / g.tile[2]) % g.tile[1];
  const int x = (tile % g.tiles[2]) * g.tile[2] + l % g.tile[2];
  if (t >= g.grid[0] || y >= g.grid[1] || x >= g.grid[2]) return -1;
  return g.n_text + (t * g.grid[1] + y) * g.grid[2] + x;
}

template <bool FORWARD>
__global__ void __launch_bounds__(256) permute_kernel(PermuteParams p) {
  const int chunks = p.d >> 3;  // 16-byte chunks per row
  const long long per_tensor = (long long)p.BH * p.n_tiled * chunks;
  const long long total = per_tensor * p.n_tensors;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_tensor);
    long long rem = i - (long long)t * per_tensor;
    const int c = (int)(rem % chunks);
    rem /= chunks;
    const int pos = (int)(rem % p.n_tiled);
    const long long bh = rem / p.n_tiled;
    const int src = tile_source_row(p.g, pos);
    if (FORWARD) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (src >= 0) v = __ldg(reinterpret_cast<const uint4*>(p.in[t] + (bh * p.n_raster + src) * p.d) + c);
      reinterpret_cast<uint4*>(p.out[t] + (bh * p.n_tiled + pos) * p.d)[c] = v;
    } else if (src >= 0) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.in[t] + (bh * p.n_tiled + pos) * p.d) + c);
      reinterpret_cast<uint4*>(p.out[t] + (bh * p.n_raster + src) * p.d)[c] = v;
    }
  }
}

cudaError_t launch_permute(bool forward, const PermuteParams& p, int num_sms, cudaStream_t stream) {
  const long long total = (long long)p.BH * p.n_tiled * (p.d >> 3) * p.n_tensors;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (forward)
    permute_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(p);
  else
    permute_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsa
