// Fused token permutation + padding between raster order and GNA tile order
// (jsqmd.com GNA article, section 2.2: a dedicated copy kernel replacing
// permute().contiguous(), fused with padding). Every token row is d bf16
// values contiguous in memory, so both directions move whole rows with
// 16-byte vector loads and stores. One warp owns one tile-order row: its
// source row is mapped once, then the warp moves that row for every tensor
// and (b, h), so the index arithmetic is paid once per row, not per chunk.
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

// Lanes cover (b*h, chunk) pairs: with cpr 16-byte chunks per row, 32 / cpr
// rows of different heads sit side by side in the warp (d = 128: 2, d = 64:
// 4), each a contiguous run of cpr chunks, and every lane keeps four loads in
// flight (four heads apart).
template <bool FORWARD>
__global__ void __launch_bounds__(256, 4) permute_kernel(PermuteParams p) {
  const int lane = threadIdx.x & 31;
  const int cpr = p.d >> 3;                         // 16-byte chunks per row
  const int nsub = cpr >= 32 ? 1 : 32 / cpr;        // heads side by side in one warp
  const int sub = cpr >= 32 ? 0 : lane / cpr;       // this lane's head within them
  const int c_first = cpr >= 32 ? lane : lane % cpr;
  const int c_step = cpr >= 32 ? 32 : cpr;          // one pass when a row fits the warp
  const bool on = sub < nsub;                       // lanes past nsub * cpr idle
  const long long bh_step = 4ll * nsub;
  const int wpb = blockDim.x >> 5;
  const int n_warps = gridDim.x * wpb;
  for (int pos = blockIdx.x * wpb + (threadIdx.x >> 5); pos < p.n_tiled; pos += n_warps) {
    int src = lane == 0 ? tile_source_row(p.g, pos) : 0;
    src = __shfl_sync(0xffffffffu, src, 0);
    if ((!FORWARD && src < 0) || !on) continue;  // padding rows are dropped by the inverse
    for (int t = 0; t < p.n_tensors; ++t) {
      const uint4* __restrict__ in = reinterpret_cast<const uint4*>(p.in[t]);
      uint4* __restrict__ out = reinterpret_cast<uint4*>(p.out[t]);
      for (long long bh0 = sub; bh0 < p.BH; bh0 += bh_step) {
        for (int c = c_first; c < cpr; c += c_step) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const long long bh = bh0 + (long long)u * nsub;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (bh < p.BH && src >= 0) {
              const long long row = FORWARD ? bh * p.n_raster + src : bh * p.n_tiled + pos;
              v[u] = __ldg(in + row * cpr + c);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const long long bh = bh0 + (long long)u * nsub;
            if (bh < p.BH) {
              const long long row = FORWARD ? bh * p.n_tiled + pos : bh * p.n_raster + src;
              out[row * cpr + c] = v[u];
            }
          }
        }
      }
    }
  }
}

// One warp per row, up to 4 blocks of 8 warps per SM (64 registers a thread,
// no spills; 32 warps x 4 loads of 16 B per lane keep ~64 KB per SM in flight).
cudaError_t launch_permute(bool forward, const PermuteParams& p, int num_sms, cudaStream_t stream) {
  long long blocks = ((long long)p.n_tiled + 7) / 8;
  const long long cap = (long long)num_sms * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (forward)
    permute_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(p);
  else
    permute_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsa
