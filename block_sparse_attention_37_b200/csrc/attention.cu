// Block-sparse attention on sm_100a: TMA-fed, tcgen05 tensor-core tiles with
// fp32 accumulators in tensor memory, online softmax in registers.
//
// One CTA computes one 128-row query tile of one (b, h). The key side is a
// list of 64-key segments built from the block list at CTA start (two kept
// 64-blocks, or one half of a 128/256-block, fill one 128-key tile), so the
// same kernel serves block sizes 64, 128 and 256. Roles (192 threads):
//   warp 0     TMA producer: Q once, then K (and V) tiles into a smem ring
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2-5  softmax warpgroup: thread r owns row r of the tile (TMEM lane r)
// Tensor memory (512 columns): S/P double buffer at columns 0 and 128, the
// fp32 output accumulator O at column 256.
//
// Per KV tile t:  S_t = Q K_t^T (SS form) -> softmax reads S_t, writes
// P_t = exp2(x - m) as bf16 over S_t -> O += P_t V_t (TS form, A from TMEM).
// S_{t+1} is computed while the softmax works on S_t. The running max is
// updated lazily: O is rescaled only when the max grows by more than 2^8.
//
// Three kinds share the pipeline:
//   KIND_FWD   the forward (lmnt.cn BSA post, section 3.1; DiTFastAttnV2
//              "Fused Kernel"; GNA fine mask only on partial tiles)
//   KIND_LSE   per-row log-sum-exp over all keys (first pass of the SparseD
//              full-score selection)
//   KIND_POOL  block sums of softmax(z) given the row LSE, i.e. the SparseD
//              A' = avgpool(A, block) numerators ("Isolated Selection")
#include "attention.cuh"

namespace bsa {

#define kNegInf (-__int_as_float(0x7f800000))
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleTau = 8.0f;

template <int D>
struct Cfg {
  static constexpr int STAGES = D == 64 ? 3 : 2;
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128-row bf16 operand tile
  static constexpr int CHUNK_BYTES = 128 * 128;   // 128 rows x 64 bf16 (one swizzle column)
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STAGES * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STAGES * TILE_BYTES;
  static constexpr int NBAR = 1 + 4 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BITS_OFF = MISC_OFF + 64;
  static constexpr int SCHED_OFF = BITS_OFF + 3 * 64 * 4;
  static constexpr int SMEM_BYTES = SCHED_OFF + kMaxSeg * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
};

static_assert(Cfg<128>::SMEM_ALLOC <= 227 * 1024, "smem budget");
static_assert(Cfg<64>::SMEM_ALLOC > 114 * 1024, "one CTA per SM (tensor memory is allocated whole)");

// Entry bits of the per-CTA segment schedule.
constexpr int kSegIdxMask = (1 << 24) - 1;
constexpr int kSegValid0 = 1 << 24;
constexpr int kSegValid1 = 1 << 25;
constexpr int kSegPartial = 1 << 26;

__device__ __forceinline__ void cta_fail(volatile int* abort_flag, int code) {
  *abort_flag = 1;
  record_error(code);
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

__device__ __forceinline__ uint32_t bit_range(int a, int b) {  // bits [a, b) of a 32-bit word
  a = max(a, 0);
  b = min(b, 32);
  if (a >= b) return 0u;
  const uint32_t hi = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  const uint32_t lo = (1u << a) - 1u;
  return hi & ~lo;
}

__device__ __forceinline__ uint64_t bit_range64(int a, int b) {  // bits [a, b), clipped to [0, 64)
  a = max(a, 0);
  b = min(b, 64);
  if (a >= b) return 0ull;
  const uint64_t hi = b >= 64 ? ~0ull : ((1ull << b) - 1ull);
  const uint64_t lo = (1ull << a) - 1ull;
  return hi & ~lo;
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

// Allowed-key bits of one 64-key segment for a query whose window is
// [lo, hi) per dimension (text and full rows pass lo = 0, hi = grid).
__device__ uint64_t gna_segment_bits(const GnaDev& g, int seg, const int* lo, const int* hi) {
  const int k0 = seg * 64;
  if (k0 < g.text_span) {
    const int nt = g.n_text - k0;
    return nt <= 0 ? 0ull : (nt >= 64 ? ~0ull : ((1ull << nt) - 1ull));
  }
  const int v0 = k0 - g.text_span;
  const int tile = v0 / g.vol;
  const int l0 = v0 - tile * g.vol;
  const int tx = tile % g.tiles[2];
  const int ty = (tile / g.tiles[2]) % g.tiles[1];
  const int tt = tile / (g.tiles[2] * g.tiles[1]);
  const int bt = tt * g.tile[0], by = ty * g.tile[1], bx = tx * g.tile[2];
  const int Tx = g.tile[2], Ty = g.tile[1];
  const int xlo = max(lo[2], 0), xhi = min(hi[2], g.grid[2]);
  uint64_t m = 0ull;
  if (Tx <= 64) {
    const int rows = 64 / Tx;
    const int R0 = l0 / Tx;
    const uint64_t xb = bit_range64(xlo - bx, xhi - bx) & bit_range64(0, Tx);
    for (int rr = 0; rr < rows; ++rr) {
      const int R = R0 + rr;
      const int t = bt + R / Ty, y = by + R % Ty;
      const bool ok = t >= lo[0] && t < hi[0] && t < g.grid[0] && y >= lo[1] && y < hi[1] &&
                      y < g.grid[1];
      if (ok) m |= xb << (rr * Tx);
    }
  } else {
    const int R = l0 / Tx;
    const int xo = bx + (l0 - R * Tx);
    const int t = bt + R / Ty, y = by + R % Ty;
    const bool ok = t >= lo[0] && t < hi[0] && t < g.grid[0] && y >= lo[1] && y < hi[1] &&
                    y < g.grid[1];
    if (ok) m = bit_range64(xlo - xo, xhi - xo);
  }
  return m;
}

// Build the CTA's sorted segment schedule (warp 0, all lanes). Returns count.
__device__ int build_schedule(const AttnParams& p, int mode, int bh, int row0, uint32_t* vb0,
                              uint32_t* vb1, uint32_t* pb, int32_t* sched, int lane) {
  const int nwords = (p.nSeg + 31) >> 5;
  for (int w = lane; w < 64; w += 32) vb0[w] = vb1[w] = pb[w] = 0u;
  __syncwarp();
  const bool h1 = row0 + 64 < p.N;
  const int I0 = row0 / p.block_q;
  const int I1 = h1 ? (row0 + 64) / p.block_q : I0;
  const int spb = p.block_k >> 6;
  if (mode == BSA_HEAD_FULL) {
    for (int w = lane; w < nwords; w += 32) {
      const uint32_t bits = bit_range(0, min(32, p.nSeg - w * 32));
      vb0[w] = bits;
      vb1[w] = bits;
    }
    if (p.has_gna && p.g.has_padding) {
      __syncwarp();
      for (int J = lane; J < p.nKB; J += 32) {
        if (!gna_block_padded(p.g, J)) continue;
        for (int u = 0; u < spb; ++u) {
          const int s = J * spb + u;
          if (s < p.nSeg) atomicOr(&pb[s >> 5], 1u << (s & 31));
        }
      }
    }
  } else {
    const int nh = (p.cnt == nullptr) ? 0 : ((I1 == I0) ? 1 : 2);
    if (p.cnt == nullptr && lane == 0) record_error(BSA_DEVERR_BAD_INDEX);
    for (int hh = 0; hh < nh; ++hh) {
      uint32_t* vb = hh ? vb1 : vb0;
      const size_t row = (size_t)bh * p.nQB + (hh ? I1 : I0);
      int n = p.cnt[row];
      if (n < 0 || n > p.max_k) {
        if (lane == 0) record_error(BSA_DEVERR_BAD_INDEX);
        n = n < 0 ? 0 : p.max_k;
      }
      const int32_t* ip = p.idx + row * p.max_k;
      const uint8_t* fp = p.flag + row * p.max_k;
      for (int e = lane; e < n; e += 32) {
        const int J = ip[e];
        if (J < 0 || J >= p.nKB) {
          record_error(BSA_DEVERR_BAD_INDEX);
          continue;
        }
        bool part = fp[e] == BSA_BLOCK_PARTIAL;
        if (part && !p.has_gna) {
          record_error(BSA_DEVERR_NO_GEOMETRY);
          part = false;
        }
        for (int u = 0; u < spb; ++u) {
          const int s = J * spb + u;
          if (s >= p.nSeg) break;
          atomicOr(&vb[s >> 5], 1u << (s & 31));
          if (part) atomicOr(&pb[s >> 5], 1u << (s & 31));
        }
      }
    }
    __syncwarp();
    if (nh <= 1)
      for (int w = lane; w < 64; w += 32) vb1[w] = vb0[w];
  }
  __syncwarp();
  // Compaction in ascending segment order: words 0..31 on lanes, then 32..63.
  const int w0 = lane, w1 = lane + 32;
  const uint32_t a0 = w0 < nwords ? (vb0[w0] | vb1[w0]) : 0u;
  const uint32_t a1 = w1 < nwords ? (vb0[w1] | vb1[w1]) : 0u;
  const int c0 = __popc(a0), c1 = __popc(a1);
  int i0 = c0, i1 = c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t0 = __shfl_up_sync(0xffffffffu, i0, o);
    const int t1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += t0;
      i1 += t1;
    }
  }
  const int tot0 = __shfl_sync(0xffffffffu, i0, 31);
  const int tot1 = __shfl_sync(0xffffffffu, i1, 31);
  int off = i0 - c0;
  for (uint32_t a = a0; a; a &= a - 1) {
    const int b = __ffs(a) - 1;
    const int s = w0 * 32 + b;
    int e = s;
    if (vb0[w0] >> b & 1u) e |= kSegValid0;
    if (vb1[w0] >> b & 1u) e |= kSegValid1;
    if (pb[w0] >> b & 1u) e |= kSegPartial;
    sched[off++] = e;
  }
  off = tot0 + i1 - c1;
  for (uint32_t a = a1; a; a &= a - 1) {
    const int b = __ffs(a) - 1;
    const int s = w1 * 32 + b;
    int e = s;
    if (vb0[w1] >> b & 1u) e |= kSegValid0;
    if (vb1[w1] >> b & 1u) e |= kSegValid1;
    if (pb[w1] >> b & 1u) e |= kSegPartial;
    sched[off++] = e;
  }
  return tot0 + tot1;
}

template <int D>
__device__ void skip_copy(const AttnParams& p, int bh, int row0) {
  if (p.cache_in == nullptr) {
    if (threadIdx.x == 0) record_error(BSA_DEVERR_BAD_INDEX);
    return;
  }
  const int rows = min(128, p.N - row0);
  const size_t base = ((size_t)bh * p.N + row0) * D;
  const float4* src = reinterpret_cast<const float4*>(p.cache_in + base);
  uint2* dst = reinterpret_cast<uint2*>(p.O + base);
  const int n4 = rows * D / 4;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = __ldg(src + i);
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    dst[i] = o;
  }
}

template <int D, int KIND>
__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Cfg<D>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int work = p.order ? p.order[blockIdx.x] : (int)blockIdx.x;
  const int qt = work % p.nQT;
  const int bh = work / p.nQT;
  const int h = bh % p.H;
  const int row0 = qt * 128;

  int mode = BSA_HEAD_FULL;
  if (KIND == KIND_FWD) {
    mode = p.head_mode[h];
    if (mode < BSA_HEAD_FULL || mode > BSA_HEAD_SKIP) {
      if (tid == 0) record_error(BSA_DEVERR_BAD_INDEX);
      return;
    }
    if (mode == BSA_HEAD_SKIP) {
      skip_copy<D>(p, bh, row0);
      return;
    }
  }

  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + S;
  uint64_t* v_full = k_empty + S;
  uint64_t* v_empty = v_full + S;
  uint64_t* s_full = v_empty + S;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_ready = p_full + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  uint32_t* vb0 = reinterpret_cast<uint32_t*>(smem + C::BITS_OFF);
  int32_t* sched = reinterpret_cast<int32_t*>(smem + C::SCHED_OFF);

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    mbar_init(o_ready, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(misc, 512);
    tmem_relinquish();
  }
  if (warp == 0) {
    const int n = build_schedule(p, mode, bh, row0, vb0, vb0 + 64, vb0 + 128, sched, lane);
    if (lane == 0) misc[2] = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int nseg = (int)misc[2];
  const int T = (nseg + 1) >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && T > 0) {  // no work: no copies, so nothing can be in flight at exit
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      if (KIND == KIND_FWD) tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
#pragma unroll
        for (int r = 0; r < 2; ++r)
          tma_load_3d(sQ + c * C::CHUNK_BYTES + r * (C::CHUNK_BYTES / 2), &tmQ, q_full, c * 64,
                      row0 + 64 * r, bh);
      int k_issued = 0, v_issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % S;
        const uint32_t ph = (uint32_t)(t / S) & 1u;
        const int sa = sched[2 * t] & kSegIdxMask;
        const int sb = (2 * t + 1 < nseg) ? (sched[2 * t + 1] & kSegIdxMask) : sa;
        if (t >= S && !mbar_wait(&k_empty[st], ph ^ 1u, abort_flag)) {
          cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
        uint8_t* dk = sK + st * C::TILE_BYTES;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(dk + c * C::CHUNK_BYTES, &tmK, &k_full[st], c * 64, sa * 64, bh);
          tma_load_3d(dk + c * C::CHUNK_BYTES + C::CHUNK_BYTES / 2, &tmK, &k_full[st], c * 64,
                      sb * 64, bh);
        }
        k_issued = t + 1;
        if (KIND == KIND_FWD) {
          if (t >= S && !mbar_wait(&v_empty[st], ph ^ 1u, abort_flag)) {
            cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&v_full[st], C::TILE_BYTES);
          uint8_t* dv = sV + st * C::TILE_BYTES;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(dv + c * C::CHUNK_BYTES, &tmV, &v_full[st], c * 64, sa * 64, bh);
            tma_load_3d(dv + c * C::CHUNK_BYTES + C::CHUNK_BYTES / 2, &tmV, &v_full[st], c * 64,
                        sb * 64, bh);
          }
          v_issued = t + 1;
        }
      }
      if (*abort_flag) {
        // Aborting: wait (bounded) for this thread's own copies still in flight.
        const uint64_t t0 = globaltimer_ns();
        auto drain = [&](uint64_t* bar, uint32_t ph) {
          while (!mbar_try_wait(smem_u32(bar), ph) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        };
        drain(q_full, 0u);
        for (int t = k_issued - S < 0 ? 0 : k_issued - S; t < k_issued; ++t)
          drain(&k_full[t % S], (uint32_t)(t / S) & 1u);
        for (int t = v_issued - S < 0 ? 0 : v_issued - S; t < v_issued; ++t)
          drain(&v_full[t % S], (uint32_t)(t / S) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      auto do_pv = [&](int u) -> bool {
        const int buf = u & 1, st = u % S;
        if (!mbar_wait(&p_full[buf], (uint32_t)(u >> 1) & 1u, abort_flag)) return false;
        if (!mbar_wait(&v_full[st], (uint32_t)(u / S) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = sVa + st * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 2048, C::CHUNK_BYTES, 1024);
          umma_ts(tmem + 256, tmem + buf * 128 + kk * 8, bdesc, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&v_empty[st]);
        tc_commit(o_ready);
        return true;
      };
      for (int t = 0; t < T && ok; ++t) {
        const int st = t % S, buf = t & 1;
        if (KIND != KIND_FWD && t >= 2)
          ok = mbar_wait(&p_full[buf], (uint32_t)((t - 2) >> 1) & 1u, abort_flag);
        ok = ok && mbar_wait(&k_full[st], (uint32_t)(t / S) & 1u, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sKa + st * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(sQa + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(kbase + off, 16, 1024);
          umma_ss(tmem + buf * 128, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[buf]);
        tc_commit(&k_empty[st]);
        if (KIND == KIND_FWD && t > 0) ok = do_pv(t - 1);
      }
      if (KIND == KIND_FWD && ok) ok = do_pv(T - 1);
      if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int pq = row0 + r;
    const bool row_valid = pq < p.N;
    const int half = r >> 6;
    const uint32_t lbase = tmem + ((uint32_t)(q4 * 32) << 16);
    const int Iq = (row_valid ? pq : (p.N - 1)) / p.block_q;
    const size_t bias_row = ((size_t)h * p.nQB + Iq) * p.nKB;

    // query window for the GNA fine mask
    int lo[3] = {0, 0, 0}, hi[3] = {1 << 30, 1 << 30, 1 << 30};
    if (p.has_gna && mode == BSA_HEAD_SPARSE && pq >= p.g.text_span) {
      const GnaDev& g = p.g;
      const int v = pq - g.text_span;
      const int tile = v / g.vol, l = v - tile * g.vol;
      const int c[3] = {(tile / (g.tiles[2] * g.tiles[1])) * g.tile[0] + l / (g.tile[1] * g.tile[2]),
                        ((tile / g.tiles[2]) % g.tiles[1]) * g.tile[1] + (l / g.tile[2]) % g.tile[1],
                        (tile % g.tiles[2]) * g.tile[2] + l % g.tile[2]};
      if (c[0] < g.grid[0] && c[1] < g.grid[1] && c[2] < g.grid[2]) {
#pragma unroll
        for (int dd = 0; dd < 3; ++dd) {
          lo[dd] = gna_window_start(c[dd], g.grid[dd], g.win[dd], g.stride[dd]);
          hi[dd] = lo[dd] + g.win[dd];
        }
      }
    }
    const int my_valid = half ? kSegValid1 : kSegValid0;

    float m = kNegInf, l = 0.f;
    float lse2 = 0.f;
    if (KIND == KIND_POOL) lse2 = row_valid ? p.lse[(size_t)bh * p.N + pq] : 0.f;
    bool ok = true;
    float s[128];
    for (int t = 0; t < T; ++t) {
      const int buf = t & 1;
      ok = warp_all(mbar_wait(&s_full[buf], (uint32_t)(t >> 1) & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lbase + buf * 128 + c * 32, s + c * 32);
      tc_wait_ld();
      if (KIND != KIND_FWD) {
        tc_fence_before();
        mbar_arrive(&p_full[buf]);
      }
      const int ea = sched[2 * t];
      const int eb = (2 * t + 1 < nseg) ? sched[2 * t + 1] : -1;
      const int sa = ea & kSegIdxMask;
      const int sb = eb >= 0 ? (eb & kSegIdxMask) : sa;
      float ba = 0.f, bb = 0.f;
      if (p.bias != nullptr) {
        ba = __ldg(p.bias + bias_row + (sa * 64) / p.block_k) * kLog2e;
        bb = __ldg(p.bias + bias_row + (sb * 64) / p.block_k) * kLog2e;
      }
#pragma unroll
      for (int j = 0; j < 64; ++j) s[j] = fmaf(s[j], p.scale_log2, ba);
#pragma unroll
      for (int j = 64; j < 128; ++j) s[j] = fmaf(s[j], p.scale_log2, bb);
      const bool tail = (sa + 1) * 64 > p.N || (sb + 1) * 64 > p.N;
      const bool need = !(ea & my_valid) || eb < 0 || !(eb & my_valid) || tail ||
                        ((ea | (eb < 0 ? 0 : eb)) & kSegPartial);
      if (need) {
        uint64_t ma = 0ull, mb = 0ull;
        if (ea & my_valid) {
          ma = (p.N - sa * 64 >= 64) ? ~0ull : ((1ull << (p.N - sa * 64)) - 1ull);
          if ((ea & kSegPartial) && p.has_gna) ma &= gna_segment_bits(p.g, sa, lo, hi);
        }
        if (eb >= 0 && (eb & my_valid)) {
          mb = (p.N - sb * 64 >= 64) ? ~0ull : ((1ull << (p.N - sb * 64)) - 1ull);
          if ((eb & kSegPartial) && p.has_gna) mb &= gna_segment_bits(p.g, sb, lo, hi);
        }
#pragma unroll
        for (int j = 0; j < 64; ++j) s[j] = ((ma >> j) & 1ull) ? s[j] : kNegInf;
#pragma unroll
        for (int j = 0; j < 64; ++j) s[64 + j] = ((mb >> j) & 1ull) ? s[64 + j] : kNegInf;
      }

      if (KIND == KIND_FWD) {
        float mx = s[0];
#pragma unroll
        for (int j = 1; j < 128; ++j) mx = fmaxf(mx, s[j]);
        const float m_new = fmaxf(m, mx);
        float alpha = 1.f;
        if (m_new > m + kRescaleTau) {
          alpha = fast_exp2(m - m_new);
          m = m_new;
        }
        const float mu = (m == kNegInf) ? 0.f : m;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float p0 = fast_exp2(s[64 * c + 2 * j] - mu);
            const float p1 = fast_exp2(s[64 * c + 2 * j + 1] - mu);
            sum += p0 + p1;
            pk[j] = pack_bf16x2(p0, p1);
          }
          tmem_st32(lbase + buf * 128 + c * 32, pk);
        }
        l = l * alpha + sum;
        if (t > 0) {
          ok = warp_all(mbar_wait(o_ready, (uint32_t)(t - 1) & 1u, abort_flag));
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float o[32];
              tmem_ld32(lbase + 256 + c * 32, o);
              tc_wait_ld();
              uint32_t* ou = reinterpret_cast<uint32_t*>(o);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= alpha;
              tmem_st32(lbase + 256 + c * 32, ou);
            }
          }
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[buf]);
      } else if (KIND == KIND_LSE) {
        float mx = s[0];
#pragma unroll
        for (int j = 1; j < 128; ++j) mx = fmaxf(mx, s[j]);
        const float m_new = fmaxf(m, mx);
        if (m_new > m) {
          l *= fast_exp2(m - m_new);
          m = m_new;
        }
        const float mu = (m == kNegInf) ? 0.f : m;
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 128; ++j) sum += fast_exp2(s[j] - mu);
        l += sum;
      } else {  // KIND_POOL
        float sa_sum = 0.f, sb_sum = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) sa_sum += fast_exp2(s[j] - lse2);
#pragma unroll
        for (int j = 64; j < 128; ++j) sb_sum += fast_exp2(s[j] - lse2);
        if (!row_valid) sa_sum = sb_sum = 0.f;
        const int Ja = (sa * 64) / p.block_k, Jb = (sb * 64) / p.block_k;
        if (eb >= 0 && Ja == Jb) {
          sa_sum += sb_sum;
          sb_sum = 0.f;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sa_sum += __shfl_xor_sync(0xffffffffu, sa_sum, o);
          sb_sum += __shfl_xor_sync(0xffffffffu, sb_sum, o);
        }
        if (lane == 0) {
          float* dst = p.apool + ((size_t)bh * p.nQB + Iq) * p.nKB;
          atomicAdd(dst + Ja, sa_sum);
          if (eb >= 0 && Ja != Jb) atomicAdd(dst + Jb, sb_sum);
        }
      }
    }
    if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);

    if (KIND == KIND_FWD) {
      bool have = ok && T > 0;
      if (have) {
        have = warp_all(mbar_wait(o_ready, (uint32_t)(T - 1) & 1u, abort_flag));
        if (!have) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
        tc_fence_after();
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t obase = ((size_t)bh * p.N + (row_valid ? pq : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (have) {
          tmem_ld32(lbase + 256 + c * 32, o);
          tc_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] *= inv;
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.O + obase + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
            v.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
            v.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
            v.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
            dst[q] = v;
          }
          if (p.cache_out != nullptr) {
            float4* cd = reinterpret_cast<float4*>(p.cache_out + obase + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) cd[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
      }
    } else if (KIND == KIND_LSE) {
      if (row_valid) p.lse[(size_t)bh * p.N + pq] = (l > 0.f) ? m + __log2f(l) : kNegInf;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int KIND>
static cudaError_t launch_one(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                              const AttnParams& p, int grid, cudaStream_t stream) {
  auto fn = attn_kernel<D, KIND>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  fn<<<grid, 192, Cfg<D>::SMEM_ALLOC, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

cudaError_t launch_attention(int d, int kind, const CUtensorMap& q, const CUtensorMap& k,
                             const CUtensorMap& v, const AttnParams& p, int grid, cudaStream_t stream) {
  if (d == 64) {
    if (kind == KIND_FWD) return launch_one<64, KIND_FWD>(q, k, v, p, grid, stream);
    if (kind == KIND_LSE) return launch_one<64, KIND_LSE>(q, k, v, p, grid, stream);
    return launch_one<64, KIND_POOL>(q, k, v, p, grid, stream);
  }
  if (kind == KIND_FWD) return launch_one<128, KIND_FWD>(q, k, v, p, grid, stream);
  if (kind == KIND_LSE) return launch_one<128, KIND_LSE>(q, k, v, p, grid, stream);
  return launch_one<128, KIND_POOL>(q, k, v, p, grid, stream);
}

}  // namespace bsa
