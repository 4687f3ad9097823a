// Block-list builder for the fixed patterns: arrow (DiTFastAttnV2, "Head-wise
// Arrow Attention") and GNA window + stride over tile-ordered tokens
// (jsqmd.com GNA article, section 1.1). One warp per (b, h, query block):
// lanes classify 32 KV blocks at a time and a ballot keeps the output sorted.
#include "mask.cuh"

namespace bsa {

// Sum over queries i in [q_lo, q_hi) of |[start(i), start(i)+k) intersect [k_lo, k_hi)|.
__host__ __device__ __forceinline__ long long pair_count_1d(int q_lo, int q_hi, int k_lo, int k_hi, int L,
                                                            int k, int s) {
  long long c = 0;
  for (int i = q_lo; i < q_hi; ++i) {
    const int st = gna_window_start(i, L, k, s);
    const int a = max(st, k_lo), b = min(st + k, k_hi);
    c += b > a ? (b - a) : 0;
  }
  return c;
}

// Does KV block J hold padded (invalid) key slots?
__host__ __device__ bool gna_kv_padded(const GnaDev& g, int J) {
  const int ntb = g.text_span / g.vol;
  if (J < ntb) return g.text_span > g.n_text && (J + 1) * g.vol > g.n_text;
  const int tile = J - ntb;
  const int c[3] = {tile / (g.tiles[1] * g.tiles[2]), (tile / g.tiles[2]) % g.tiles[1],
                    tile % g.tiles[2]};
  bool pad = false;
  for (int d = 0; d < 3; ++d) pad |= (c[d] + 1) * g.tile[d] > g.grid[d];
  return pad;
}

// Class of (query tile I, KV tile J) under the GNA window; text rows and
// columns are full, padded key slots make a block partial.
__host__ __device__ int gna_class(const GnaDev& g, int I, int J) {
  const int ntb = g.text_span / g.vol;
  const bool kpad = gna_kv_padded(g, J);
  if (I < ntb || J < ntb) return kpad ? BSA_BLOCK_PARTIAL : BSA_BLOCK_FULL;
  const int ti = I - ntb, tj = J - ntb;
  const int ci[3] = {ti / (g.tiles[1] * g.tiles[2]), (ti / g.tiles[2]) % g.tiles[1], ti % g.tiles[2]};
  const int cj[3] = {tj / (g.tiles[1] * g.tiles[2]), (tj / g.tiles[2]) % g.tiles[1], tj % g.tiles[2]};
  bool full = true;
  for (int d = 0; d < 3; ++d) {
    const int qlo = ci[d] * g.tile[d], qhi = min(qlo + g.tile[d], g.grid[d]);
    const int klo = cj[d] * g.tile[d], khi = min(klo + g.tile[d], g.grid[d]);
    const long long c = pair_count_1d(qlo, qhi, klo, khi, g.grid[d], g.win[d], g.stride[d]);
    if (c == 0) return BSA_BLOCK_NONE;
    full &= c == (long long)(qhi - qlo) * (khi - klo);
  }
  return (full && !kpad) ? BSA_BLOCK_FULL : BSA_BLOCK_PARTIAL;
}

__global__ void build_mask_kernel(MaskParams p) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long rows = (long long)p.B * p.H * p.nQB;
  if (row >= rows) return;
  const int I = (int)(row % p.nQB);
  const int h = (int)((row / p.nQB) % p.H);
  int mode = p.head_mode ? p.head_mode[h] : BSA_HEAD_SPARSE;
  if (mode < BSA_HEAD_FULL || mode > BSA_HEAD_SKIP) {
    if (lane == 0) record_error(BSA_DEVERR_BAD_INDEX);
    mode = BSA_HEAD_SKIP;
  }
  int w = 0;
  if (p.kind == BSA_MASK_ARROW && mode == BSA_HEAD_SPARSE) w = p.window ? p.window[h] : 0;
  int32_t* idx = p.idx + row * p.max_k;
  uint8_t* flag = p.flag + row * p.max_k;
  uint8_t* bm = p.bitmap ? p.bitmap + row * p.nKB : nullptr;
  int count = 0;
  for (int J0 = 0; J0 < p.nKB; J0 += 32) {
    const int J = J0 + lane;
    int cls = BSA_BLOCK_NONE;
    if (J < p.nKB) {
      if (mode == BSA_HEAD_SKIP) {
        cls = BSA_BLOCK_NONE;
      } else if (p.kind == BSA_MASK_ARROW) {
        const bool keep = mode == BSA_HEAD_FULL || I < p.ntb || J < p.ntb || abs(I - J) <= w;
        cls = keep ? BSA_BLOCK_FULL : BSA_BLOCK_NONE;
      } else {
        if (mode == BSA_HEAD_FULL) {
          cls = gna_kv_padded(p.g, J) ? BSA_BLOCK_PARTIAL : BSA_BLOCK_FULL;
        } else {
          cls = gna_class(p.g, I, J);
        }
      }
      if (bm) bm[J] = (uint8_t)cls;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, cls != BSA_BLOCK_NONE);
    if (cls != BSA_BLOCK_NONE) {
      const int pos = count + __popc(bal & ((1u << lane) - 1u));
      idx[pos] = J;
      flag[pos] = (uint8_t)cls;
    }
    count += __popc(bal);
  }
  for (int e = count + lane; e < p.max_k; e += 32) {
    idx[e] = -1;
    flag[e] = 0;
  }
  if (lane == 0) p.cnt[row] = count;
}

cudaError_t launch_build_mask(const MaskParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.H * p.nQB;
  const int warps_per_block = 8;
  const long long blocks = (rows + warps_per_block - 1) / warps_per_block;
  build_mask_kernel<<<(unsigned)blocks, warps_per_block * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsa
