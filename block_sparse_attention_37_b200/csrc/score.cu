// The score passes of the SparseD full-score selection ("Isolated
// Selection": A = attention map, A' = avgpool(A, block_size), top-rho% per
// query block and key group), on tcgen05 tensor cores.
//
//   KIND_TLSE  one pass: per row and 128-key tile the log-sum-exp (log2
//              units) of z = scale*q.k + bias over the tile's keys, kept in a
//              [T][128] slab per query tile, and the row's LSE over all keys
//              carried along; at the end each row reads its slab back (it is
//              still in L2) and the CTA writes its query tile's partial row of
//              A': sum over its rows of 2^(tile LSE - row LSE), per key block
//   KIND_LSE   two-pass form, first pass: per-row LSE over all keys
//   KIND_POOL  two-pass form, second pass: given the LSE, the block sums of
//              softmax(z), i.e. the numerators of A'[I, J]; every 128-row
//              query tile adds its 128 rows into A'[I, J] (one atomic per
//              warp and 64-key half)
// The one-pass form evaluates QK^T and the exps once instead of twice, and
// its sums have a fixed order; the two-pass form needs no per-tile slabs and
// runs where the workspace cannot hold them.
//
// One CTA computes one 128-row query tile of one (b, h) against every key.
// Roles (192 threads): warp 0 TMA producer (Q once, K tiles into a ring),
// warp 1 TMEM allocator and single-thread tcgen05.mma issuer (S = Q K^T into
// a double-buffered fp32 accumulator in tensor memory), warps 2-5 one thread
// per row reading S from tensor memory.
#include "tiles.cuh"

namespace bsa {

// Two CTAs per SM (96 KB of shared memory and 256 tensor-memory columns
// each at d = 128): each scheduler then runs two row warps, whose exps and
// reductions hide each other's latency.
template <int D>
struct ScoreCfg {
  static constexpr int STAGES = D == 64 ? 4 : 2;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;
  static constexpr int BAR_OFF = K_OFF + STAGES * TILE_BYTES;
  // q_full, k_full[S], k_empty[S], s_full[2], s_free[2], mma_done
  static constexpr int NBAR = 1 + 2 * STAGES + 4 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 64;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
};
static_assert(2 * ScoreCfg<128>::SMEM_ALLOC <= 227 * 1024 && 2 * ScoreCfg<64>::SMEM_ALLOC <= 227 * 1024,
              "two CTAs per SM");

template <int D, int KIND>
__global__ void __launch_bounds__(192, 2)
    score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const AttnParams p) {
  using C = ScoreCfg<D>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int qt, bh;
  if (KIND == KIND_TLSE) {
    const int m = p.block_q >> 7;  // query tiles per query block
    const long long u = p.u0 + blockIdx.x / m;
    bh = (int)(u / p.nQB);
    qt = (int)(u % p.nQB) * m + (int)(blockIdx.x % m);
    if (qt >= p.nQT) return;  // the ragged last block of a head has fewer tiles (whole CTA, before any setup)
  } else {
    qt = blockIdx.x % p.nQT;
    bh = blockIdx.x / p.nQT;
  }
  const int h = bh % p.H;
  const int row0 = qt * 128;
  const int T = (p.N + 127) >> 7;  // 128-key tiles

  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + S;
  uint64_t* s_full = k_empty + S;
  uint64_t* s_free = s_full + 2;
  uint64_t* mma_done = s_free + 2;  // every MMA of the CTA complete (teardown)
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
    }
    mbar_init(mma_done, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(misc, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
      for (int c = 0; c < D / 64; ++c)
        for (int r = 0; r < 2; ++r)
          tma_load_3d(sQ + c * C::CHUNK_BYTES + r * (C::CHUNK_BYTES / 2), &tmQ, q_full, c * 64, row0 + 64 * r, bh);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % S;
        if (t >= S && !mbar_wait(&k_empty[st], ((uint32_t)(t / S) & 1u) ^ 1u, abort_flag, p.wait_limit_ns)) {
          cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
        uint8_t* dk = sK + st * C::TILE_BYTES;
        for (int c = 0; c < D / 64; ++c)
          for (int r = 0; r < 2; ++r)
            tma_load_3d(dk + c * C::CHUNK_BYTES + r * (C::CHUNK_BYTES / 2), &tmK, &k_full[st], c * 64,
                        t * 128 + 64 * r, bh);
        issued = t + 1;
      }
      if (*abort_flag) {  // copies in flight land before the CTA ends
        mbar_drain(q_full, 0u);
        for (int t = issued - S < 0 ? 0 : issued - S; t < issued; ++t) mbar_drain(&k_full[t % S], (uint32_t)(t / S) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      bool ok = mbar_wait(q_full, 0u, abort_flag, p.wait_limit_ns);
      int issued = 0;
      for (int t = 0; t < T && ok; ++t) {
        const int st = t % S, buf = t & 1;
        if (t >= 2) ok = mbar_wait(&s_free[buf], (uint32_t)((t - 2) >> 1) & 1u, abort_flag, p.wait_limit_ns);
        ok = ok && mbar_wait(&k_full[st], (uint32_t)(t / S) & 1u, abort_flag, p.wait_limit_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sKa + st * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
          umma_ss(tmem + buf * 128, smem_desc_sw128(sQa + off, 16, 1024), smem_desc_sw128(kbase + off, 16, 1024),
                  idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[buf]);
        tc_commit(&k_empty[st]);
        issued = t + 1;
      }
      if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
      // tensor memory is freed only once every issued MMA has completed (an
      // aborting CTA may leave MMAs in flight)
      if (issued > 0) {
        tc_commit(mma_done);
        mbar_drain(mma_done, 0u);
      }
    }
  } else {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int pq = row0 + r;
    const bool row_valid = pq < p.N;
    const uint32_t lbase = tmem + ((uint32_t)(q4 * 32) << 16);
    const int Iq = (row_valid ? pq : (p.N - 1)) / p.block_q;
    const size_t bias_row = ((size_t)h * p.nQB + Iq) * p.nKB;
    float m = kNegInf, l = 0.f;
    float* tslab = KIND == KIND_TLSE ? p.tlse + (size_t)blockIdx.x * T * 128 : nullptr;
    const float lse2 = (KIND == KIND_POOL && row_valid) ? p.lse[(size_t)bh * p.N + pq] : 0.f;
    bool ok = true;
    float s[128];
    for (int t = 0; t < T; ++t) {
      const int buf = t & 1;
      ok = warp_all(mbar_wait(&s_full[buf], (uint32_t)(t >> 1) & 1u, abort_flag, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lbase + buf * 128 + c * 32, s + c * 32);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[buf]);
      const int sa = 2 * t, sb = 2 * t + 1;  // 64-key halves of the tile
      float ba = 0.f, bb = 0.f;
      if (p.bias != nullptr) {
        ba = __ldg(p.bias + bias_row + (sa * 64) / p.block_k) * kLog2e;
        if (sb < p.nSeg) bb = __ldg(p.bias + bias_row + (sb * 64) / p.block_k) * kLog2e;
      }
      // The per-row reductions below run as several independent chains (a
      // single 128-long chain of dependent max or add instructions would
      // take longer than the exps themselves).
      if (KIND != KIND_POOL) {
        // z = scale * s + bias, per 64-key half
#pragma unroll
        for (int j = 0; j < 64; j += 2) fma2(s[j], s[j + 1], p.scale_log2, ba);
#pragma unroll
        for (int j = 64; j < 128; j += 2) fma2(s[j], s[j + 1], p.scale_log2, bb);
      } else {
        // z - lse in one step: scale * s + (bias - lse)
        const float oa = ba - lse2, ob = bb - lse2;
#pragma unroll
        for (int j = 0; j < 64; j += 2) fma2(s[j], s[j + 1], p.scale_log2, oa);
#pragma unroll
        for (int j = 64; j < 128; j += 2) fma2(s[j], s[j + 1], p.scale_log2, ob);
      }
      if ((t + 1) * 128 > p.N) {  // ragged last tile: keys past N do not exist
        const uint64_t ma = tail_bits(p.N, sa);
        const uint64_t mb = sb < p.nSeg ? tail_bits(p.N, sb) : 0ull;
#pragma unroll
        for (int j = 0; j < 64; ++j) s[j] = ((ma >> j) & 1ull) ? s[j] : kNegInf;
#pragma unroll
        for (int j = 0; j < 64; ++j) s[64 + j] = ((mb >> j) & 1ull) ? s[64 + j] : kNegInf;
      }
      if (KIND == KIND_LSE) {
        // row max: four chains of max3 over the 128 values
        float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
        for (int j = 4; j < 124; j += 8) {
          m0 = max3f(m0, s[j], s[j + 1]);
          m1 = max3f(m1, s[j + 2], s[j + 3]);
          m2 = max3f(m2, s[j + 4], s[j + 5]);
          m3 = max3f(m3, s[j + 6], s[j + 7]);
        }
        m0 = max3f(m0, s[124], s[125]);
        m1 = max3f(m1, s[126], s[127]);
        const float mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        const float m_new = fmaxf(m, mx);
        if (m_new > m) {
          l *= fast_exp2(m - m_new);
          m = m_new;
        }
        const float mu = (m == kNegInf) ? 0.f : m;
        // sum of exp2(z - m): four accumulators, two per packed add
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int j = 0; j < 128; j += 4) {
          float x0 = s[j], x1 = s[j + 1], x2 = s[j + 2], x3 = s[j + 3];
          fma2(x0, x1, 1.f, -mu);
          fma2(x2, x3, 1.f, -mu);
          add2(a0, a1, fast_exp2(x0), fast_exp2(x1));
          add2(a2, a3, fast_exp2(x2), fast_exp2(x3));
        }
        l += (a0 + a1) + (a2 + a3);
      } else if (KIND == KIND_TLSE) {
        // the tile's own LSE: max, then the sum of exp2(z - max), no running state
        float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
        for (int j = 4; j < 124; j += 8) {
          m0 = max3f(m0, s[j], s[j + 1]);
          m1 = max3f(m1, s[j + 2], s[j + 3]);
          m2 = max3f(m2, s[j + 4], s[j + 5]);
          m3 = max3f(m3, s[j + 6], s[j + 7]);
        }
        m0 = max3f(m0, s[124], s[125]);
        m1 = max3f(m1, s[126], s[127]);
        const float mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        const float mu = (mx == kNegInf) ? 0.f : mx;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int j = 0; j < 128; j += 4) {
          float x0 = s[j], x1 = s[j + 1], x2 = s[j + 2], x3 = s[j + 3];
          fma2(x0, x1, 1.f, -mu);
          fma2(x2, x3, 1.f, -mu);
          add2(a0, a1, fast_exp2(x0), fast_exp2(x1));
          add2(a2, a3, fast_exp2(x2), fast_exp2(x3));
        }
        const float lt = (a0 + a1) + (a2 + a3);
        const float xt = (lt > 0.f) ? mx + __log2f(lt) : kNegInf;
        // consecutive rows are consecutive floats: one 128-byte store per warp
        if (row_valid) tslab[(size_t)t * 128 + r] = xt;
        // the row's LSE over the tiles so far, as a running (max, sum)
        if (xt > kNegInf) {
          const float mn = fmaxf(m, xt);
          l = l * fast_exp2(m - mn) + fast_exp2(xt - mn);
          m = mn;
        }
      } else {
        // block sums of exp2(z - lse) per 64-key half, two packed accumulators each
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          add2(a0, a1, fast_exp2(s[j]), fast_exp2(s[j + 1]));
          add2(a2, a3, fast_exp2(s[j + 2]), fast_exp2(s[j + 3]));
          add2(b0, b1, fast_exp2(s[64 + j]), fast_exp2(s[65 + j]));
          add2(b2, b3, fast_exp2(s[66 + j]), fast_exp2(s[67 + j]));
        }
        float suma = (a0 + a1) + (a2 + a3), sumb = (b0 + b1) + (b2 + b3);
        if (!row_valid) suma = sumb = 0.f;
        const int Ja = (sa * 64) / p.block_k, Jb = (sb * 64) / p.block_k;
        if (Ja == Jb) {
          suma += sumb;
          sumb = 0.f;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          suma += __shfl_xor_sync(0xffffffffu, suma, o);
          sumb += __shfl_xor_sync(0xffffffffu, sumb, o);
        }
        if (lane == 0) {
          float* dst = p.apool + ((size_t)bh * p.nQB + Iq) * p.nKB;
          atomicAdd(dst + Ja, suma);
          if (Ja != Jb && sb < p.nSeg) atomicAdd(dst + Jb, sumb);
        }
      }
    }
    if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
    if (KIND == KIND_LSE && row_valid) p.lse[(size_t)bh * p.N + pq] = (l > 0.f) ? m + __log2f(l) : kNegInf;
    if (KIND == KIND_TLSE) {
      // The query tile's partial row of A'. Every MMA has completed (each
      // softmax warp saw the last S land), so the K ring is free: it holds
      // one row of per-warp sums per warp, added in a fixed order. All four
      // warps reach the barrier; in an aborting CTA (where copies into the
      // ring may still be in flight) none of them touches it.
      const bool live = ok && row_valid && l > 0.f;
      const float lse = live ? m + __log2f(l) : 0.f;
      const int tpk = p.block_k >> 7;  // 128-key tiles per key block
      float* red = reinterpret_cast<float*>(sK);
      for (int J0 = 0; J0 < p.nKB; J0 += 32) {
        float acc[32];
        if (tpk == 1) {
          // one tile per key block: 32 independent loads in flight, then the exps
#pragma unroll
          for (int i = 0; i < 32; ++i)
            acc[i] = (live && J0 + i < p.nKB) ? tslab[(size_t)(J0 + i) * 128 + r] : kNegInf;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = fast_exp2(acc[i] - lse);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int J = J0 + i;
            float a = 0.f;
            if (live && J < p.nKB) {
              const int t1 = min((J + 1) * tpk, T);
              for (int t = J * tpk; t < t1; ++t) a += fast_exp2(tslab[(size_t)t * 128 + r] - lse);
            }
            acc[i] = a;
          }
        }
        const float sum = transpose_reduce32(acc, lane);
        if (ok && J0 + lane < p.nKB) red[q4 * p.nKB + J0 + lane] = sum;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!*abort_flag) {
        float* dst = p.apool + ((size_t)p.u0 * (p.block_q >> 7) + blockIdx.x) * p.nKB;
        for (int J = r; J < p.nKB; J += 128)
          dst[J] = (red[J] + red[p.nKB + J]) + (red[2 * p.nKB + J] + red[3 * p.nKB + J]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D, int KIND>
static cudaError_t launch_score_d(const CUtensorMap& q, const CUtensorMap& k, const AttnParams& p, int grid,
                                  cudaStream_t stream) {
  auto fn = score_kernel<D, KIND>;
  static DeviceOnce once;
  const cudaError_t e = once.run([&]() -> cudaError_t {
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, ScoreCfg<D>::SMEM_ALLOC);
  });
  if (e != cudaSuccess) return e;
  fn<<<grid, 192, ScoreCfg<D>::SMEM_ALLOC, stream>>>(q, k, p);
  return cudaGetLastError();
}

cudaError_t launch_score(int d, int kind, const CUtensorMap& q, const CUtensorMap& k, const AttnParams& p,
                         int grid, cudaStream_t stream) {
  if (d == 64) {
    if (kind == KIND_TLSE) return launch_score_d<64, KIND_TLSE>(q, k, p, grid, stream);
    return kind == KIND_LSE ? launch_score_d<64, KIND_LSE>(q, k, p, grid, stream)
                            : launch_score_d<64, KIND_POOL>(q, k, p, grid, stream);
  }
  if (kind == KIND_TLSE) return launch_score_d<128, KIND_TLSE>(q, k, p, grid, stream);
  return kind == KIND_LSE ? launch_score_d<128, KIND_LSE>(q, k, p, grid, stream)
                          : launch_score_d<128, KIND_POOL>(q, k, p, grid, stream);
}

}  // namespace bsa
