// Helpers for 64-key segments and the GNA fine mask, shared by the forward
// and the selection score passes.
#pragma once

#include "attention.cuh"

namespace bsa {

#define kNegInf (-__int_as_float(0x7f800000))
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSegIdxMask = (1 << 24) - 1;

__device__ __forceinline__ void cta_fail(volatile int* abort_flag, int code) {
  *abort_flag = 1;
  record_error(code);
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 arithmetic shared by the softmax of the forward and of the score passes.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (x0, x1) * c + (o, o), two lanes in one instruction
__device__ __forceinline__ void fma2(float& x0, float& x1, float c, float o) {
  uint64_t v, cc, oo;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(oo) : "f"(o));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(v) : "l"(v), "l"(cc), "l"(oo));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(v));
}

__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  uint64_t a, b;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(a) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(a));
}

__device__ __forceinline__ uint32_t bit_range(int a, int b) {  // bits [a, b), clipped to [0, 32)
  a = max(a, 0);
  b = min(b, 32);
  if (a >= b) return 0u;
  const uint32_t hi = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  const uint32_t lo = (1u << a) - 1u;
  return hi & ~lo;
}

__host__ __device__ __forceinline__ uint64_t bit_range64(int a, int b) {  // bits [a, b), clipped to [0, 64)
  a = a > 0 ? a : 0;
  b = b < 64 ? b : 64;
  if (a >= b) return 0ull;
  const uint64_t hi = b >= 64 ? ~0ull : ((1ull << b) - 1ull);
  const uint64_t lo = (1ull << a) - 1ull;
  return hi & ~lo;
}

// Keys of segment `seg` below N.
__device__ __forceinline__ uint64_t tail_bits(int N, int seg) {
  const int n = N - seg * 64;
  return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
}

// Does KV block J of a GNA tile layout hold padded (invalid) key slots?
__device__ __forceinline__ bool gna_block_padded(const GnaDev& g, int J) {
  const int ntb = g.text_span / g.vol;
  if (J < ntb) return g.text_span > g.n_text && (J + 1) * g.vol > g.n_text;
  const int tile = J - ntb;
  const int c2 = tile % g.tiles[2];
  const int c1 = (tile / g.tiles[2]) % g.tiles[1];
  const int c0 = tile / (g.tiles[2] * g.tiles[1]);
  return (c0 + 1) * g.tile[0] > g.grid[0] || (c1 + 1) * g.tile[1] > g.grid[1] ||
         (c2 + 1) * g.tile[2] > g.grid[2];
}

// A query's key window per dimension, [lo, hi) (text and full rows: everything).
struct QWin {
  int lo0, lo1, lo2, hi0, hi1, hi2;
};

__host__ __device__ __forceinline__ QWin gna_query_window(const GnaDev& g, int pq, bool windowed) {
  QWin w{0, 0, 0, 1 << 30, 1 << 30, 1 << 30};
  if (!windowed || pq < g.text_span) return w;
  const int v = pq - g.text_span;
  const int tile = v / g.vol, l = v - tile * g.vol;
  const int c0 = (tile / (g.tiles[2] * g.tiles[1])) * g.tile[0] + l / (g.tile[1] * g.tile[2]);
  const int c1 = ((tile / g.tiles[2]) % g.tiles[1]) * g.tile[1] + (l / g.tile[2]) % g.tile[1];
  const int c2 = (tile % g.tiles[2]) * g.tile[2] + l % g.tile[2];
  if (c0 >= g.grid[0] || c1 >= g.grid[1] || c2 >= g.grid[2]) return w;  // padding row
  w.lo0 = gna_window_start(c0, g.grid[0], g.win[0], g.stride[0]);
  w.lo1 = gna_window_start(c1, g.grid[1], g.win[1], g.stride[1]);
  w.lo2 = gna_window_start(c2, g.grid[2], g.win[2], g.stride[2]);
  w.hi0 = w.lo0 + g.win[0];
  w.hi1 = w.lo1 + g.win[1];
  w.hi2 = w.lo2 + g.win[2];
  return w;
}

// Allowed-key bits of one 64-key segment (tile order) for a query window.
// Needs the tile's x-extent to divide 64 or be a multiple of 64. The segment's
// place in the tile grid takes five divisions by launch invariants (multiply-
// high and shift); the rows of the segment step a (t, y) counter.
__host__ __device__ __forceinline__ uint64_t gna_segment_bits(const GnaDev& g, int seg, const QWin& q) {
  const int k0 = seg * 64;
  if (k0 < g.text_span) {
    const int nt = g.n_text - k0;
    return nt <= 0 ? 0ull : (nt >= 64 ? ~0ull : ((1ull << nt) - 1ull));
  }
  const int v0 = k0 - g.text_span;
  const int tile = fdiv(v0, g.f_vol);
  const int l0 = v0 - tile * g.vol;
  const int q2 = fdiv(tile, g.f_tiles2);
  const int tx = tile - q2 * g.tiles[2];
  const int tt = fdiv(q2, g.f_tiles1);
  const int ty = q2 - tt * g.tiles[1];
  const int bt = tt * g.tile[0], by = ty * g.tile[1], bx = tx * g.tile[2];
  const int Tx = g.tile[2], Ty = g.tile[1];
  const int xlo = q.lo2 > 0 ? q.lo2 : 0;
  const int xhi = q.hi2 < g.grid[2] ? q.hi2 : g.grid[2];
  const int tlo = q.lo0, thi = q.hi0 < g.grid[0] ? q.hi0 : g.grid[0];
  const int ylo = q.lo1, yhi = q.hi1 < g.grid[1] ? q.hi1 : g.grid[1];
  uint64_t m = 0ull;
  if (g.seg_one_slice) {
    // one t-slice: t is fixed and the rows in the window form the range
    // [rlo, rhi) of the segment's 64 / Tx rows
    const int rows = 64 / Tx;
    const int R0 = fdiv(l0, g.f_tile2);
    const int tq = fdiv(R0, g.f_tile1);
    const int t = bt + tq, y0 = by + (R0 - tq * Ty);
    if (t >= tlo && t < thi) {
      const int rlo = ylo - y0 > 0 ? ylo - y0 : 0;
      const int rhi = yhi - y0 < rows ? yhi - y0 : rows;
      const uint64_t xb = bit_range64(xlo - bx, xhi - bx) & bit_range64(0, Tx);
      if (rlo < rhi) m = (xb * g.x_rep) & bit_range64(rlo * Tx, rhi * Tx);
    }
  } else if (Tx <= 64) {
    const int rows = 64 / Tx;  // Tx divides 64 (host check)
    const int R0 = fdiv(l0, g.f_tile2);
    int tq = fdiv(R0, g.f_tile1);
    int yq = R0 - tq * Ty;
    const uint64_t xb = bit_range64(xlo - bx, xhi - bx) & bit_range64(0, Tx);
    for (int rr = 0; rr < rows; ++rr) {
      const int t = bt + tq, y = by + yq;
      if (t >= tlo && t < thi && y >= ylo && y < yhi) m |= xb << (rr * Tx);
      if (++yq == Ty) {
        yq = 0;
        ++tq;
      }
    }
  } else {
    const int R = fdiv(l0, g.f_tile2);
    const int xo = bx + (l0 - R * Tx);
    const int tq = fdiv(R, g.f_tile1);
    const int t = bt + tq, y = by + (R - tq * Ty);
    if (t >= tlo && t < thi && y >= ylo && y < yhi) m = bit_range64(xlo - xo, xhi - xo);
  }
  return m;
}

// Precomputed segment geometry (one-slice layouts). The forward computes,
// once per CTA while it builds the key schedule, where each partial 64-key
// segment sits in the grid: the t, y and x of its first key (17 bits each;
// a sequence of at most 131072 tokens keeps every coordinate below 2^17). A
// text segment is marked instead and keeps the text rule. Each softmax
// thread then needs only a few compares per segment against its query's
// clamped window (QBox), computed once before the tile loop.
constexpr uint64_t kGeoText = 1ull << 63;

__host__ __device__ inline uint64_t gna_segment_geo(const GnaDev& g, int seg) {
  const int k0 = seg * 64;
  if (k0 < g.text_span) return kGeoText;
  const int v0 = k0 - g.text_span;
  const int tile = fdiv(v0, g.f_vol);
  const int l0 = v0 - tile * g.vol;
  const int q2 = fdiv(tile, g.f_tiles2);
  const int tx = tile - q2 * g.tiles[2];
  const int tt = fdiv(q2, g.f_tiles1);
  const int ty = q2 - tt * g.tiles[1];
  const int R0 = fdiv(l0, g.f_tile2);
  const int tq = fdiv(R0, g.f_tile1);
  const int t = tt * g.tile[0] + tq;
  const int y0 = ty * g.tile[1] + (R0 - tq * g.tile[1]);
  const int x0 = tx * g.tile[2];
  return (uint64_t)t | ((uint64_t)y0 << 17) | ((uint64_t)x0 << 34);
}

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

struct QBox {
  int tlo, thi, ylo, yhi, xlo, xhi;
};

// A query's window clamped to the grid (padding keys fall outside it).
__host__ __device__ inline QBox gna_query_box(const GnaDev& g, const QWin& q) {
  QBox b;
  b.tlo = q.lo0 > 0 ? q.lo0 : 0;
  b.thi = q.hi0 < g.grid[0] ? q.hi0 : g.grid[0];
  b.ylo = q.lo1 > 0 ? q.lo1 : 0;
  b.yhi = q.hi1 < g.grid[1] ? q.hi1 : g.grid[1];
  b.xlo = q.lo2 > 0 ? q.lo2 : 0;
  b.xhi = q.hi2 < g.grid[2] ? q.hi2 : g.grid[2];
  return b;
}

// gna_segment_bits for a one-slice layout from the precomputed geometry.
__host__ __device__ __forceinline__ uint64_t gna_segment_bits_geo(const GnaDev& g, int seg, uint64_t geo,
                                                                  const QBox& b) {
  if (geo & kGeoText) {
    const int nt = g.n_text - seg * 64;
    return nt <= 0 ? 0ull : (nt >= 64 ? ~0ull : ((1ull << nt) - 1ull));
  }
  const int t = (int)(geo & 0x1FFFFull), y0 = (int)((geo >> 17) & 0x1FFFFull), x0 = (int)((geo >> 34) & 0x1FFFFull);
  if (t < b.tlo || t >= b.thi) return 0ull;
  const int rlo = b.ylo - y0 > 0 ? b.ylo - y0 : 0;
  const int rhi = b.yhi - y0 < g.seg_rows ? b.yhi - y0 : g.seg_rows;
  if (rlo >= rhi) return 0ull;
  const int Tx = g.tile[2];
  const uint64_t xb = bit_range64(b.xlo - x0, b.xhi - x0) & g.x_mask;
  return (xb * g.x_rep) & bit_range64(rlo * Tx, rhi * Tx);
}

// The window of a GNA query group (64 rows that form one box of the grid in a
// one-slice layout), as the bounding box of its rows' windows: per dimension
// [start(first coordinate), start(last coordinate) + window). The window
// start is nondecreasing in the coordinate, so every row's window lies
// inside it. `ok` is false for a group of text rows or one that reaches past
// the grid (padding rows), whose rows see every key: such a group is never
// narrowed.
struct GroupWin {
  int t0, t1, y0, y1, x0, x1;
  bool ok;
};

__host__ __device__ inline GroupWin gna_group_window(const GnaDev& g, int qseg) {
  GroupWin w{0, 0, 0, 0, 0, 0, false};
  const uint64_t geo = gna_segment_geo(g, qseg);
  if (geo & kGeoText) return w;
  const int t = (int)(geo & 0x1FFFFull), y = (int)((geo >> 17) & 0x1FFFFull), x = (int)((geo >> 34) & 0x1FFFFull);
  const int ny = g.seg_rows, nx = g.tile[2];
  if (t >= g.grid[0] || y + ny > g.grid[1] || x + nx > g.grid[2]) return w;
  w.t0 = gna_window_start(t, g.grid[0], g.win[0], g.stride[0]);
  w.t1 = w.t0 + g.win[0];
  w.y0 = gna_window_start(y, g.grid[1], g.win[1], g.stride[1]);
  w.y1 = gna_window_start(y + ny - 1, g.grid[1], g.win[1], g.stride[1]) + g.win[1];
  w.x0 = gna_window_start(x, g.grid[2], g.win[2], g.stride[2]);
  w.x1 = gna_window_start(x + nx - 1, g.grid[2], g.win[2], g.stride[2]) + g.win[2];
  w.ok = true;
  return w;
}

// Does a key segment (one-slice layout; `geo` from gna_segment_geo) have a key
// inside the group window? A segment outside it is masked for every row of
// the group: the mask is the product of one interval test per dimension.
__host__ __device__ __forceinline__ bool gna_segment_meets(const GnaDev& g, uint64_t geo, const GroupWin& w) {
  if (!w.ok || (geo & kGeoText)) return true;
  const int t = (int)(geo & 0x1FFFFull), y = (int)((geo >> 17) & 0x1FFFFull), x = (int)((geo >> 34) & 0x1FFFFull);
  return t >= w.t0 && t < w.t1 && y < w.y1 && y + g.seg_rows > w.y0 && x < w.x1 && x + g.tile[2] > w.x0;
}

}  // namespace bsa
