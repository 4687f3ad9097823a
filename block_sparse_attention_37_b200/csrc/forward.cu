// The block-sparse forward (bsa_forward) on sm_100a, two query tiles per CTA.
//
// A CTA owns 256 query rows of one (b, h): two 128-row tiles, one per softmax
// warpgroup. The key side is the union, over the four 64-row groups, of the
// kept 64-key segments, with one validity bit per group; a warpgroup skips a
// 128-key tile none of its rows keeps, so each tile costs tensor work only
// for the warpgroups that need it while K and V are loaded once.
// Roles (384 threads, three aligned warpgroups):
//   warp 0      TMA producer: both Q tiles, then the K tiles into their ring
//   warp 1      TMEM allocator and tcgen05.mma issuer (whole warp, one
//               elected lane issues)
//   warp 2      TMA producer of the V tiles into their own ring
//   warp 3      idle (it completes the control warpgroup)
//   warps 4-7   softmax warpgroup 0 (rows 0..127 of the CTA)
//   warps 8-11  softmax warpgroup 1 (rows 128..255)
// The control warpgroup hands registers to the softmax warpgroups
// (setmaxnreg), which keep a whole 128-key row of S in registers.
// Tensor memory (512 columns), per warpgroup w: S at 128w; d = 64: P at
// 256 + 64w and O at 384 + 64w (all 512 columns), so the next QK^T may
// overwrite S while the softmax still works on the row; d = 128: P over S,
// O at 256 + 128w. The tensor core runs one group's PV and next QK^T while
// the other group's softmax runs (lmnt.cn BSA post, section 3.1:
// FlashAttention tiles with online softmax over the selected blocks;
// DiTFastAttnV2 "Fused Kernel").
// Output leaves through shared memory and a TMA store.
#include <utility>

#include <type_traits>

#include "tiles.cuh"

namespace bsa {

constexpr float kRescaleTau = 8.0f;  // O is rescaled only when the row max grows by more than 2^8

// F8: the e4m3 form (d = 128 only). A 128-row tile of e4m3 codes is 128 rows
// of 128 bytes, the byte geometry of a bf16 d = 64 tile, so four K/V stages
// fit; the Q slots keep 32 KB each for the bf16 O staging; V arrives
// transposed (K-major), one 128-byte run of keys per channel.
template <int D, bool F8 = false>
struct FwdCfg {
  static constexpr int STAGES = (D == 64 || F8) ? 4 : 2;
  static constexpr int TILE = F8 ? 128 * 128 : 128 * D * 2;
  static constexpr int QSLOT = F8 ? 128 * D * 2 : TILE;
  static constexpr int NCH = F8 ? 1 : D / 64;  // 128-byte column chunks of a Q / K row
  static constexpr int CHUNK = 128 * 128;      // 128 rows x 128 bytes
  static constexpr int Q_OFF = 0;              // two Q slots (reused as O staging)
  static constexpr int K_OFF = 2 * QSLOT;
  static constexpr int V_OFF = K_OFF + STAGES * TILE;
  static constexpr int BAR_OFF = V_OFF + STAGES * TILE;
  static constexpr int NBAR = 2 + 6 * STAGES + 8 + 1;
  // d = 64: P gets its own tensor-memory columns (S 128 + P 64 + O 64 per
  // warpgroup fill all 512), so the next QK^T can overwrite S as soon as the
  // softmax has read it; d = 128: P is written over S and waits for PV.
  static constexpr bool SEP_P = D == 64 && !F8;
  static constexpr uint32_t S_COL = 0;                     // + 128 w
  static constexpr uint32_t P_COL = SEP_P ? 256 : 0;       // + (SEP_P ? 64 : 128) w
  static constexpr uint32_t P_STRIDE = SEP_P ? 64 : 128;
  static constexpr uint32_t O_COL = SEP_P ? 384 : 256;     // + D w
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BITS_OFF = MISC_OFF + 64;
  static constexpr int SCHED_OFF = BITS_OFF + 5 * 64 * 4;
  static constexpr int TMP_OFF = SCHED_OFF + kMaxSeg * 4;  // F8: scratch of the tile reorder
  static constexpr int GEO_OFF = TMP_OFF + (F8 ? kMaxSeg * 4 : 0);  // segment geometry (GNA)
  static constexpr int SMEM_BYTES = GEO_OFF + kMaxSeg * 8;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  // register split: launched at kLaunchRegs per thread, the control
  // warpgroup drops to REGS_CTL and the two softmax warpgroups rise to REGS_SMX
  static constexpr int THREADS = 384;
  static constexpr int REGS_CTL = 56;
  static constexpr int REGS_SMX = 224;
};
constexpr int kLaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
template <int D>
constexpr bool regs_fit() {
  return 128 * FwdCfg<D>::REGS_CTL + 256 * FwdCfg<D>::REGS_SMX <= FwdCfg<D>::THREADS * kLaunchRegs;
}
static_assert(regs_fit<64>() && regs_fit<128>(), "register split exceeds the launch allocation");
static_assert(FwdCfg<128>::SMEM_ALLOC <= 227 * 1024, "smem budget");
static_assert(FwdCfg<64>::SMEM_ALLOC <= 227 * 1024, "smem budget");
static_assert(FwdCfg<128, true>::SMEM_ALLOC <= 227 * 1024, "smem budget");
static_assert(FwdCfg<64, false>::SMEM_ALLOC <= 227 * 1024 && FwdCfg<128, false>::SMEM_ALLOC <= 227 * 1024, "smem budget");

// Segment entry bits: index in [0, 24), group-valid bits g0..g3 at 24..27, partial at 28.
constexpr int kGrpShift = 24;
constexpr int kPart4 = 1 << 28;

// Mask kind a kernel is compiled for. kMaskAny reads it from the parameters
// (no mask, GNA in any layout); kMaskGnaSlice is GNA in a layout whose 64-key
// segments each lie in one slice of a tile, the form whose fine mask comes
// from the precomputed segment geometry. Compiling that form alone leaves the
// general GNA decoder out of its code.
constexpr int kMaskAny = 0;
constexpr int kMaskGnaSlice = 1;
template <int MK>
__device__ __forceinline__ bool gna_on(const AttnParams& p) {
  return MK == kMaskGnaSlice || p.has_gna;
}
template <int MK>
__device__ __forceinline__ bool gna_slice(const AttnParams& p) {
  return MK == kMaskGnaSlice || (p.has_gna && p.g.seg_one_slice);
}

template <int N>
__device__ __forceinline__ void regs_release() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_claim() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, const void* src, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The staged tile may be reused (or the CTA end) once the copies have read
// it; their global writes complete before the grid does.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Sorted union schedule of the CTA's four 64-row groups (warp 0). Returns count.
// Warp-parallel throughout: the block-list rows of all groups are read in one
// round of loads, and segments are emitted 32 at a time by ballot compaction.
// Sparse GNA heads in a one-slice layout: a partial segment outside a group's
// window loses that group's bit (the group needs neither its QK^T nor its
// PV), and a segment no group needs is left out. `pairs`: segments are kept
// or left out in aligned pairs (the e4m3 V loads take 128-key runs).
template <int MK>
__device__ int build_schedule256(const AttnParams& p, int mode, int bh, int row0, uint32_t* vb,
                                 uint32_t* pb, int32_t* sched, int lane, bool pairs) {
  const int nwords = (p.nSeg + 31) >> 5;
  for (int w = lane; w < 5 * 64; w += 32) vb[w] = 0u;  // vb[4][64] then pb[64]
  __syncwarp();
  const int spb = p.block_k >> 6;
  if (mode == BSA_HEAD_FULL) {
    for (int w = lane; w < nwords; w += 32) vb[w] = bit_range(0, min(32, p.nSeg - w * 32));
    if (gna_on<MK>(p) && p.g.has_padding)
      for (int J = lane; J < p.nKB; J += 32) {
        if (!gna_block_padded(p.g, J)) continue;
        for (int u = 0; u < spb; ++u) {
          const int s = J * spb + u;
          if (s < p.nSeg) atomicOr(&pb[s >> 5], 1u << (s & 31));
        }
      }
    __syncwarp();
    for (int g = 1; g < 4; ++g)
      for (int w = lane; w < 64; w += 32) vb[g * 64 + w] = vb[w];
  } else {
    if (p.cnt == nullptr) {
      if (lane == 0) record_error(BSA_DEVERR_BAD_INDEX);
    } else {
      // lane g < 4: entries of group g's block-list row; 0 when the group is
      // past N or shares its predecessor's query block (it copies them below)
      int n_l = 0;
      if (lane < 4) {
        const int rq = row0 + 64 * lane;
        const int Ig = rq / p.block_q;
        if (rq < p.N && (lane == 0 || Ig != (rq - 64) / p.block_q)) {
          n_l = p.cnt[(size_t)bh * p.nQB + Ig];
          if (n_l < 0 || n_l > p.max_k) {
            record_error(BSA_DEVERR_BAD_INDEX);
            n_l = n_l < 0 ? 0 : p.max_k;
          }
        }
      }
      const int n0 = __shfl_sync(0xffffffffu, n_l, 0), n1 = __shfl_sync(0xffffffffu, n_l, 1);
      const int n2 = __shfl_sync(0xffffffffu, n_l, 2), n3 = __shfl_sync(0xffffffffu, n_l, 3);
      const int e1 = n0, e2 = n0 + n1, e3 = n0 + n1 + n2, tot = e3 + n3;
      for (int e = lane; e < tot; e += 32) {
        const int g = e < e1 ? 0 : e < e2 ? 1 : e < e3 ? 2 : 3;
        const int k = e - (g == 0 ? 0 : g == 1 ? e1 : g == 2 ? e2 : e3);
        const size_t at = ((size_t)bh * p.nQB + (row0 + 64 * g) / p.block_q) * p.max_k + k;
        const int J = p.idx[at];
        if (J < 0 || J >= p.nKB) {
          record_error(BSA_DEVERR_BAD_INDEX);
          continue;
        }
        bool part = p.flag[at] == BSA_BLOCK_PARTIAL;
        if (part && !gna_on<MK>(p)) {
          record_error(BSA_DEVERR_NO_GEOMETRY);
          part = false;
        }
        for (int u = 0; u < spb; ++u) {
          const int s = J * spb + u;
          if (s >= p.nSeg) break;
          atomicOr(&vb[g * 64 + (s >> 5)], 1u << (s & 31));
          if (part) atomicOr(&pb[s >> 5], 1u << (s & 31));
        }
      }
    }
    __syncwarp();
    // groups sharing a query block share its bits; groups past N copy their neighbour
    for (int g = 1; g < 4; ++g) {
      const int rq = row0 + 64 * g;
      if (rq >= p.N || rq / p.block_q == (rq - 64) / p.block_q)
        for (int w = lane; w < 64; w += 32) vb[g * 64 + w] = vb[(g - 1) * 64 + w];
      __syncwarp();
    }
  }
  __syncwarp();
  // the groups' windows (lane g computes group g's, then every lane gets all four)
  const bool narrow = mode != BSA_HEAD_FULL && gna_slice<MK>(p);
  GroupWin gw[4];
  if (narrow) {
    GroupWin mine{0, 0, 0, 0, 0, 0, false};
    if (lane < 4 && row0 + 64 * lane < p.N) mine = gna_group_window(p.g, (row0 >> 6) + lane);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      gw[g].t0 = __shfl_sync(0xffffffffu, mine.t0, g);
      gw[g].t1 = __shfl_sync(0xffffffffu, mine.t1, g);
      gw[g].y0 = __shfl_sync(0xffffffffu, mine.y0, g);
      gw[g].y1 = __shfl_sync(0xffffffffu, mine.y1, g);
      gw[g].x0 = __shfl_sync(0xffffffffu, mine.x0, g);
      gw[g].x1 = __shfl_sync(0xffffffffu, mine.x1, g);
      gw[g].ok = __shfl_sync(0xffffffffu, (int)mine.ok, g) != 0;
    }
  }
  // emit the kept segments in ascending order, 32 at a time
  int base = 0;
  for (int s0 = 0; s0 < p.nSeg; s0 += 32) {
    const int wd = s0 >> 5, s = s0 + lane;
    const uint32_t v0 = vb[wd], v1 = vb[64 + wd], v2 = vb[128 + wd], v3 = vb[192 + wd], pw = pb[wd];
    uint32_t gb = ((v0 >> lane) & 1u) | (((v1 >> lane) & 1u) << 1) | (((v2 >> lane) & 1u) << 2) |
                  (((v3 >> lane) & 1u) << 3);
    if (narrow && s < p.nSeg && gb != 0u && ((pw >> lane) & 1u)) {
      const uint64_t geo = gna_segment_geo(p.g, s);
#pragma unroll
      for (int g = 0; g < 4; ++g)
        if (((gb >> g) & 1u) && !gna_segment_meets(p.g, geo, gw[g])) gb &= ~(1u << g);
    }
    const uint32_t gp = __shfl_xor_sync(0xffffffffu, gb, 1);  // the aligned partner's bits
    const bool keep = s < p.nSeg && (gb != 0u || (pairs && gp != 0u));
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (keep)
      sched[base + __popc(bal & ((1u << lane) - 1u))] =
          s | (int)(gb << kGrpShift) | (((pw >> lane) & 1u) ? kPart4 : 0);
    base += __popc(bal);
  }
  // Each entry was written by the lane that kept it; the caller's lanes read
  // entries other lanes wrote (tile reorder, geometry, tile counts).
  __syncwarp();
  return base;
}

// Work order of the grid (longest first, so no long CTA starts late): all
// FULL heads, then the SPARSE heads (below), then the SKIP heads. A
// bijection from blockIdx.x onto the B*H*nQP (b, h, pair) items; heads with
// an invalid mode count as sparse (their CTA reports it).
// Run by a whole warp; every warp computes the same answer.
__device__ __forceinline__ void map_item(const AttnParams& p, int d, int nQP, int lane, int& bh, int& pair) {
  int nF = 0, nK = 0;
  for (int h0 = 0; h0 < p.H; h0 += 32) {
    const int hh = h0 + lane;
    const int md = hh < p.H ? p.head_mode[hh] : -1;
    nF += __popc(__ballot_sync(0xffffffffu, md == BSA_HEAD_FULL));
    nK += __popc(__ballot_sync(0xffffffffu, md == BSA_HEAD_SKIP));
  }
  const int nS = p.H - nF - nK;
  const int k = (int)blockIdx.x;
  const int perF = p.B * nF * nQP, perS = p.B * nS * nQP;
  int cls, b, m;
  if (k < perF) {
    cls = BSA_HEAD_FULL;
    pair = k % nQP;
    b = (k / nQP) / nF;
    m = (k / nQP) % nF;
  } else if (k < perF + perS) {
    // pair 0 of every (b, sparse head) unit first: the text rows lead the
    // sequence and keep every key, so these are the longest sparse CTAs.
    // The other pairs follow in chunks of units whose K and V fit in a
    // quarter of L2 (32 MiB; measured: chunks near half of L2 thrash),
    // query pair by query pair within a chunk, so the K/V the chunk's CTAs
    // share stay cached.
    int r = k - perF;
    const int units = p.B * nS;
    cls = BSA_HEAD_SPARSE;
    int u;
    if (r < units) {
      pair = 0;
      u = r;
    } else {
      r -= units;
      const int np = nQP - 1;  // pairs 1 .. nQP-1 (np >= 1 here)
      const long long fit = (32ll << 20) / (4ll * p.N * d);
      const int G = (int)(fit < 1 ? 1 : fit > units ? units : fit);
      const int c = r / (G * np);
      const int gsz = min(G, units - c * G);
      const int rr = r - c * G * np;
      u = c * G + rr % gsz;
      pair = 1 + rr / gsz;
    }
    b = u / nS;
    m = u % nS;
  } else {
    const int r = k - perF - perS;
    cls = BSA_HEAD_SKIP;
    pair = r % nQP;
    b = (r / nQP) / nK;
    m = (r / nQP) % nK;
  }
  int h = m;  // every head in one class: the m-th head is head m
  const int ncls = cls == BSA_HEAD_FULL ? nF : cls == BSA_HEAD_SKIP ? nK : nS;
  for (int h0 = 0; ncls < p.H && h0 < p.H; h0 += 32) {
    const int hh = h0 + lane;
    const int md = hh < p.H ? p.head_mode[hh] : -1;
    const bool in = hh < p.H && (cls == BSA_HEAD_SPARSE ? (md != BSA_HEAD_FULL && md != BSA_HEAD_SKIP) : md == cls);
    const uint32_t mask = __ballot_sync(0xffffffffu, in);
    const int c = __popc(mask);
    if (m < c) {  // the m-th set bit of mask
      uint32_t mm = mask;
      for (int i = 0; i < m; ++i) mm &= mm - 1u;
      h = h0 + __ffs((int)mm) - 1;
      break;
    }
    m -= c;
  }
  bh = b * p.H + h;
}

// Bit w of the result: does warpgroup w need tile t?
__device__ __forceinline__ int tile_need(const int32_t* sched, int nseg, int t, int act_mask) {
  const int ea = sched[2 * t];
  const int eb = (2 * t + 1 < nseg) ? sched[2 * t + 1] : 0;
  const int g = ((ea | eb) >> kGrpShift) & 0xF;
  return (((g & 3) ? 1 : 0) | ((g & 12) ? 2 : 0)) & act_mask;
}

// The order in which the CTA walks its full 128-key tiles (F8, four stages):
// tiles both warpgroups need first, then the tiles of one warpgroup only,
// alternating between the two while both have some. When the two groups'
// lists differ, consecutive ring stages then hold tiles of different groups,
// so neither waits behind a run of the other's tiles. A trailing half tile
// stays last. Warp-parallel (a rank per class from ballots); `tmp` holds 2n
// entries.
__device__ void reorder_tiles(int32_t* sched, int32_t* tmp, int n, int act, int lane) {
  const int full = n >> 1;
  if (full < 3) return;
  int c[4] = {0, 0, 0, 0};
  for (int t0 = 0; t0 < full; t0 += 32) {
    const int t = t0 + lane;
    int cls = -1;
    if (t < full) {
      cls = tile_need(sched, n, t, act);
      if (cls == 0) cls = 3;
    }
#pragma unroll
    for (int k = 1; k < 4; ++k) c[k] += __popc(__ballot_sync(0xffffffffu, cls == k));
  }
  const int n3 = c[3], m = min(c[1], c[2]);
  int base[4] = {0, 0, 0, 0};
  for (int t0 = 0; t0 < full; t0 += 32) {
    const int t = t0 + lane;
    int cls = -1;
    if (t < full) {
      cls = tile_need(sched, n, t, act);
      if (cls == 0) cls = 3;
    }
    int pos = 0;
#pragma unroll
    for (int k = 1; k < 4; ++k) {
      const uint32_t bal = __ballot_sync(0xffffffffu, cls == k);
      if (cls == k) {
        const int r = base[k] + __popc(bal & ((1u << lane) - 1u));
        pos = k == 3 ? r : n3 + (r < m ? 2 * r + (k - 1) : 2 * m + (r - m));
      }
      base[k] += __popc(bal);
    }
    if (t < full) {
      tmp[2 * pos] = sched[2 * t];
      tmp[2 * pos + 1] = sched[2 * t + 1];
    }
  }
  __syncwarp();
  for (int i = lane; i < 2 * full; i += 32) sched[i] = tmp[i];
  __syncwarp();
}

// S = Q K^T over D/16 k-steps of 16 (K-major SW128 operands: k-step kk sits
// in 64-column chunk kk/4 (16 KB apart) at byte offset 32*(kk%4)).
template <int KK>
__device__ __forceinline__ void qk_step(uint32_t s_tmem, uint64_t qd, uint64_t kd, uint32_t idesc) {
  constexpr uint32_t off = ((KK >> 2) * 16384 + (KK & 3) * 32) >> 4;
  umma_ss_at_warp<off, off>(s_tmem, qd, kd, idesc, KK > 0 ? 1u : 0u);
}
template <int... KK>
__device__ __forceinline__ void qk_all(uint32_t s_tmem, uint64_t qd, uint64_t kd, uint32_t idesc,
                                       std::integer_sequence<int, KK...>) {
  (qk_step<KK>(s_tmem, qd, kd, idesc), ...);
}

// O (+)= P V over 8 k-steps of 16 keys: P from tensor memory (8 columns per
// step), V MN-major SW128 (16 rows = 2048 bytes per step).
template <int KK>
__device__ __forceinline__ void pv_step(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, uint32_t idesc, uint32_t first) {
  constexpr uint32_t voff = KK * 2048 / 16;
  umma_ts_at_warp<KK * 8, voff>(o_tmem, p_tmem, vd, idesc, (KK > 0 || !first) ? 1u : 0u);
}
template <int... KK>
__device__ __forceinline__ void pv_all(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, uint32_t idesc, uint32_t first,
                                       std::integer_sequence<int, KK...>) {
  (pv_step<KK>(o_tmem, p_tmem, vd, idesc, first), ...);
}

// e4m3: S = Q K^T over 4 k-steps of 32 values (32 bytes of the one 128-byte
// chunk of a row), and O (+)= P V over 4 k-steps of 32 keys: P packed four to
// a tensor-memory column (8 columns per step), V transposed (K-major, 32 bytes
// per step).
template <int KK>
__device__ __forceinline__ void qk8_step(uint32_t s_tmem, uint64_t qd, uint64_t kd, uint32_t idesc) {
  umma8_ss_at_warp<KK * 2, KK * 2>(s_tmem, qd, kd, idesc, KK > 0 ? 1u : 0u);
}
template <int KK>
__device__ __forceinline__ void pv8_step(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, uint32_t idesc,
                                         uint32_t first) {
  umma8_ts_at_warp<KK * 8, KK * 2>(o_tmem, p_tmem, vd, idesc, (KK > 0 || !first) ? 1u : 0u);
}
template <int... KK>
__device__ __forceinline__ void qk8_all(uint32_t s_tmem, uint64_t qd, uint64_t kd, uint32_t idesc,
                                        std::integer_sequence<int, KK...>) {
  (qk8_step<KK>(s_tmem, qd, kd, idesc), ...);
}
template <int... KK>
__device__ __forceinline__ void pv8_all(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, uint32_t idesc,
                                        uint32_t first, std::integer_sequence<int, KK...>) {
  (pv8_step<KK>(o_tmem, p_tmem, vd, idesc, first), ...);
}

template <int D>
__device__ void skip_copy256(const AttnParams& p, int bh, int row0) {
  if (p.cache_in == nullptr) {
    if (threadIdx.x == 0) record_error(BSA_DEVERR_BAD_INDEX);
    return;
  }
  const int rows = min(256, p.N - row0);
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

template <int D, bool F8 = false, int MK = kMaskAny>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const AttnParams p) {
  using C = FwdCfg<D, F8>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nQP = (p.N + 255) >> 8;
  int bh, pair;
  map_item(p, D, nQP, lane, bh, pair);
  const int h = bh % p.H;
  const int row0 = pair * 256;

  const int mode = p.head_mode[h];
  if (mode < BSA_HEAD_FULL || mode > BSA_HEAD_SKIP) {
    if (tid == 0) record_error(BSA_DEVERR_BAD_INDEX);
    return;
  }
  if (mode == BSA_HEAD_SKIP) {
    skip_copy256<D>(p, bh, row0);
    return;
  }

  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;          // [2]
  uint64_t* k_full = bars + 2;      // [S]
  uint64_t* v_full = k_full + S;         // [S]
  uint64_t* k_empty = v_full + S;        // [S][2]: stage released by warpgroup w
  uint64_t* v_empty = k_empty + 2 * S;   // [S][2]
  uint64_t* s_full = v_empty + 2 * S;  // [2]
  uint64_t* p_full = s_full + 2;    // [2]
  uint64_t* o_ready = p_full + 2;   // [2]
  uint64_t* s_free = o_ready + 2;   // [2] (separate-P layout: S read by the softmax)
  uint64_t* mma_done = s_free + 2;  // every MMA of the CTA complete (teardown)
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  uint32_t* vb = reinterpret_cast<uint32_t*>(smem + C::BITS_OFF);
  int32_t* sched = reinterpret_cast<int32_t*>(smem + C::SCHED_OFF);

  if (tid == 0) {
    for (int w = 0; w < 2; ++w) {
      mbar_init(&q_full[w], 1);
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], 128);
      mbar_init(&o_ready[w], 1);
      mbar_init(&s_free[w], 128);
    }
    mbar_init(mma_done, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
    }
    for (int s = 0; s < 2 * S; ++s) {
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    misc[1] = 0;
    fence_barrier_init();
    // Q does not depend on the key schedule: both tiles are loaded now and
    // land while warp 0 builds it (rows past N read as zeros)
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      mbar_arrive_expect_tx(&q_full[w], C::TILE);
      for (int c = 0; c < C::NCH; ++c)
        for (int h2 = 0; h2 < 2; ++h2)
          tma_load_3d(sQ + w * C::QSLOT + c * C::CHUNK + h2 * (C::CHUNK / 2), &tmQ, &q_full[w], c * 64,
                      row0 + 128 * w + 64 * h2, bh);
    }
  }
  if (warp == 1) {
    tmem_alloc(misc, 512);
    tmem_relinquish();
  }
  if (warp == 0) {
    const int n = build_schedule256<MK>(p, mode, bh, row0, vb, vb + 256, sched, lane, F8);
    // tiles each warpgroup needs
    const int act = 1 | ((row0 + 128 < p.N) ? 2 : 0);
    if constexpr (F8) reorder_tiles(sched, reinterpret_cast<int32_t*>(smem + C::TMP_OFF), n, act, lane);
    // where every partial segment sits in the grid, once for the whole CTA
    if (gna_slice<MK>(p)) {
      uint64_t* geo = reinterpret_cast<uint64_t*>(smem + C::GEO_OFF);
      for (int i = lane; i < n; i += 32) {
        const int e = sched[i];
        if (e & kPart4) geo[i] = gna_segment_geo(p.g, e & kSegIdxMask);
      }
    }
    const int T = (n + 1) >> 1;
    int c0 = 0, c1 = 0;
    for (int t = lane; t < T; t += 32) {
      const int nw = tile_need(sched, n, t, act);
      c0 += nw & 1;
      c1 += nw >> 1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c0 += __shfl_xor_sync(0xffffffffu, c0, o);
      c1 += __shfl_xor_sync(0xffffffffu, c1, o);
    }
    if (lane == 0) {
      misc[2] = n;
      misc[3] = c0;
      misc[4] = c1;
      misc[5] = act;
    }
  }
  if constexpr (F8) {
    // sigma: the head's largest V scale; P is stored as p * sv / sigma, so
    // every key block's V scale folds into the exponent, and O is scaled by
    // sigma at the end
    if (warp == 2) {
      float m = 0.f;
      for (int i = lane; i < p.nSeg; i += 32) m = fmaxf(m, __ldg(p.sv + (size_t)bh * p.nSeg + i));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) misc[6] = __float_as_uint(m > 0.f ? m : 1.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int nseg = (int)misc[2];
  const int T = (nseg + 1) >> 1;
  const int act = (int)misc[5];
  const int wg_tiles0 = (int)misc[3], wg_tiles1 = (int)misc[4];

  // every role ends with its own copy of the teardown (a shared tail would
  // make the register allocator apply the control warpgroup's limit to all)
  auto teardown = [&]() {
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  };
  if (warp < 4) {
    regs_release<C::REGS_CTL>();
    if (warp == 0 || warp == 2) {
    // ---------------------------------------------------------------- producers
    // One ring each, in two warps (a wait of one does not hold up the other):
    // warp 0 loads K tiles, warp 2 V tiles. A stage of either ring is
    // reloaded once the warpgroups that used its previous tile have released
    // it (QK^T for K, PV for V), so K runs ahead of the PVs instead of
    // queueing behind V.
    // the ring's loop, instantiated once per ring (no runtime branch on the kind)
    auto produce = [&](auto ring) {
      constexpr bool IS_K = decltype(ring)::value;
      uint64_t* const full = IS_K ? k_full : v_full;
      uint64_t* const empty = IS_K ? k_empty : v_empty;
      int issued = 0;
      uint32_t par = 0u;  // phase parity per (stage, warpgroup) release barrier
      for (int t = 0; t < T; ++t) {
        const int st = t % S;
        const int sa = sched[2 * t] & kSegIdxMask;
        const int sb = (2 * t + 1 < nseg) ? (sched[2 * t + 1] & kSegIdxMask) : sa;
        // the warpgroups that used this stage's previous tile must have released it
        const int prev_need = t >= S ? tile_need(sched, nseg, t - S, act) : 0;
        bool released = true;
        for (int w = 0; w < 2 && released; ++w)
          if ((prev_need >> w) & 1) {
            const int b = 2 * st + w;
            released = mbar_wait(&empty[b], (par >> b) & 1u, abort_flag, p.wait_limit_ns);
            par ^= 1u << b;
          }
        if (!released) {
          cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
          break;
        }
        if constexpr (IS_K) {
          // a withheld tile (failure-detection test) is never loaded: its
          // consumers' waits run out
          if (t != p.withhold_tile) {
            mbar_arrive_expect_tx(&k_full[st], C::TILE);
            uint8_t* dk = sK + st * C::TILE;
            for (int c = 0; c < C::NCH; ++c) {
              tma_load_3d(dk + c * C::CHUNK, &tmK, &k_full[st], c * 64, sa * 64, bh);
              tma_load_3d(dk + c * C::CHUNK + C::CHUNK / 2, &tmK, &k_full[st], c * 64, sb * 64, bh);
            }
          }
        } else {
          mbar_arrive_expect_tx(&v_full[st], C::TILE);
          uint8_t* dv = sV + st * C::TILE;
          if constexpr (F8) {
            // V transposed: the tile's 128 keys are one 128-byte run per channel
            // row. Key blocks of 128 or more make every tile an aligned pair of
            // segments (the host checks); anything else is recorded, and the
            // load still goes out so the pipeline stays whole
            if ((sa & 1) || (2 * t + 1 < nseg && sb != sa + 1)) record_error(BSA_DEVERR_SCHEDULE);
            for (int h2 = 0; h2 < 2; ++h2) tma_load_3d(dv + h2 * (C::CHUNK / 2), &tmV, &v_full[st], sa * 64, 64 * h2, bh);
          } else {
            for (int c = 0; c < D / 64; ++c) {
              tma_load_3d(dv + c * C::CHUNK, &tmV, &v_full[st], c * 64, sa * 64, bh);
              tma_load_3d(dv + c * C::CHUNK + C::CHUNK / 2, &tmV, &v_full[st], c * 64, sb * 64, bh);
            }
          }
        }
        issued = t + 1;
      }
      if (*abort_flag)  // copies in flight land before the CTA ends
        for (int t = issued - S < 0 ? 0 : issued - S; t < issued; ++t)
          if (!IS_K || t != p.withhold_tile) mbar_drain(&full[t % S], (uint32_t)(t / S) & 1u);
    };
    if (lane == 0 && T > 0) {
      if (warp == 0)
        produce(std::true_type{});
      else
        produce(std::false_type{});
    }
    if (warp == 0 && lane == 0)  // every CTA loaded Q: it must have landed before the CTA ends
      for (int w = 0; w < 2; ++w) mbar_drain(&q_full[w], 0u);
    } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Two issue strategies, chosen by what measured faster for each layout.
    if constexpr (C::SEP_P) {
      // The warp serves both warpgroups by polling: whichever QK^T or PV is
      // ready is issued, so neither warpgroup waits behind the other's barriers.
      // All 32 lanes run the loop, so its state and the operand descriptors are
      // warp-uniform; one elected lane issues each MMA and commit.
      if (T > 0) {
        auto ready = [&](uint64_t* bar, uint32_t parity) -> bool {
          return __all_sync(0xffffffffu, mbar_test(smem_u32(bar), parity));
        };
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
        // per-warpgroup state: next tile to QK (T = none), QK^T count, and the
        // tiles whose PV is outstanding in issue order (f0 first), with their
        // indices among the warpgroup's tiles
        struct WgState {
          int next, cnt, f0, j0, f1, j1;
          bool q_ok;
        };
        auto next_tile = [&](int t, int w) {
          while (t < T && !((tile_need(sched, nseg, t, act) >> w) & 1)) ++t;
          return t;
        };
        WgState g0{next_tile(0, 0), 0, -1, 0, -1, 0, wg_tiles0 == 0};
        WgState g1{next_tile(0, 1), 0, -1, 0, -1, 0, wg_tiles1 == 0};
        // K and V tiles are observed landing in tile order: when tile x is
        // tested, tile x - S (same stage) is known to have landed and tile
        // x + S cannot have been loaded (its stage waits for the users of x),
        // so a one-bit parity test cannot alias another phase of the stage
        int k_seen = 0, v_seen = 0;
        // PV of the oldest outstanding tile, if its P and V are ready
        auto try_pv = [&](WgState& g, int w) -> bool {
          if (g.f0 < 0) return false;
          const int u = g.f0, st = u % S;
          while (v_seen <= u && ready(&v_full[v_seen % S], (uint32_t)(v_seen / S) & 1u)) ++v_seen;
          if (v_seen <= u || !ready(&p_full[w], (uint32_t)g.j0 & 1u)) return false;
          tc_fence_after();
          pv_all(tmem + C::O_COL + w * D, tmem + C::P_COL + w * C::P_STRIDE,
                 smem_desc_sw128(sVa + st * C::TILE, C::CHUNK, 1024), idesc_pv, g.j0 == 0 ? 1u : 0u,
                 std::make_integer_sequence<int, 8>{});
          tc_commit_warp(&o_ready[w]);
          tc_commit_warp(&v_empty[2 * st + w]);
          g.f0 = g.f1;
          g.j0 = g.j1;
          g.f1 = -1;
          return true;
        };
        // QK^T of the warpgroup's next tile, if Q, K and the S columns are ready
        auto try_qk = [&](WgState& g, int w) -> bool {
          if (g.next >= T || g.f1 >= 0) return false;
          const int t = g.next, st = t % S;
          if (!g.q_ok) {
            if (!ready(&q_full[w], 0u)) return false;
            g.q_ok = true;
          }
          // S is free once the softmax has read it (own P columns) or once the
          // previous PV is issued (P written over S: the tensor pipe keeps order)
          const bool s_ok = C::SEP_P ? (g.cnt == 0 || ready(&s_free[w], (uint32_t)(g.cnt - 1) & 1u))
                                     : (g.f0 < 0);
          if (!s_ok) return false;
          while (k_seen <= t && ready(&k_full[k_seen % S], (uint32_t)(k_seen / S) & 1u)) ++k_seen;
          if (k_seen <= t) return false;
          tc_fence_after();
          qk_all(tmem + C::S_COL + w * 128, smem_desc_sw128(sQa + w * C::QSLOT, 16, 1024),
                 smem_desc_sw128(sKa + st * C::TILE, 16, 1024), idesc_qk, std::make_integer_sequence<int, D / 16>{});
          tc_commit_warp(&s_full[w]);
          tc_commit_warp(&k_empty[2 * st + w]);
          if (g.f0 < 0) {
            g.f0 = t;
            g.j0 = g.cnt;
          } else {
            g.f1 = t;
            g.j1 = g.cnt;
          }
          ++g.cnt;
          g.next = next_tile(t + 1, w);
          return true;
        };
        // separate P: the next QK^T first (it unblocks the softmax); shared columns: PV first
        auto step = [&](WgState& g, int w) -> bool {
          if (C::SEP_P) {
            const bool q = try_qk(g, w);
            return try_pv(g, w) || q;
          }
          const bool v = try_pv(g, w);
          return try_qk(g, w) || v;
        };
        uint64_t t_idle = globaltimer_ns();
        uint32_t spins = 0;
        while (g0.next < T || g0.f0 >= 0 || g1.next < T || g1.f0 >= 0) {
          const bool a0 = step(g0, 0);
          const bool a1 = step(g1, 1);
          if (a0 || a1) {
            spins = 0;
            continue;
          }
          if ((++spins & 63u) == 0) {
            const uint64_t now = __shfl_sync(0xffffffffu, globaltimer_ns(), 0);
            if (spins == 64) t_idle = now;
            if (__any_sync(0xffffffffu, *abort_flag != 0) || now - t_idle > p.wait_limit_ns) {
              cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
              break;
            }
          }
        }
        // tensor memory is freed only once every issued MMA has completed (an
        // aborting CTA may leave MMAs in flight)
        if (g0.cnt + g1.cnt > 0) {
          tc_commit_warp(mma_done);
          mbar_drain(mma_done, 0u);
        }
      }
    } else {
      // P written over S: fixed issue order with blocking (suspending) waits.
      // Per tile t, for each warpgroup that needs t: the PV of its previous
      // tile, then QK^T(t) (the tensor pipe keeps issue order, so S is
      // overwritten only after P has been read). All 32 lanes run the loop,
      // so its state and the operand descriptors are warp-uniform; one
      // elected lane issues each MMA and commit.
      if (T > 0) {
        constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_pv = F8 ? idesc_e4m3_f32(128, D) : idesc_bf16_f32(128, D, false, true);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
        auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
          return warp_all(mbar_wait(bar, parity, abort_flag, p.wait_limit_ns));
        };
        // per warpgroup: tile whose PV is outstanding (-1: none) and its index
        // among the warpgroup's tiles; QK^T issued so far
        int pt0 = -1, pj0 = 0, pt1 = -1, pj1 = 0, c0 = 0, c1 = 0;
        bool q0 = false, q1 = false;
        // V tiles are observed in tile order (K tiles are, by the loop), so a
        // one-bit parity test never aliases another phase of a shared stage:
        // when tile x is waited for, tile x - S has landed, and tile x + S
        // cannot have been loaded before this warp released x
        int v_seen = 0;
        auto pv = [&](int w) -> bool {
          const int u = w ? pt1 : pt0, jj = w ? pj1 : pj0;
          for (; v_seen <= u; ++v_seen)
            if (!wwait(&v_full[v_seen % S], (uint32_t)(v_seen / S) & 1u)) return false;
          if (!wwait(&p_full[w], (uint32_t)jj & 1u)) return false;
          tc_fence_after();
          if constexpr (F8)
            pv8_all(tmem + C::O_COL + w * D, tmem + C::P_COL + w * C::P_STRIDE,
                    smem_desc_sw128(sVa + (u % S) * C::TILE, 16, 1024), idesc_pv, jj == 0 ? 1u : 0u,
                    std::make_integer_sequence<int, 4>{});
          else
            pv_all(tmem + C::O_COL + w * D, tmem + C::P_COL + w * C::P_STRIDE,
                   smem_desc_sw128(sVa + (u % S) * C::TILE, C::CHUNK, 1024), idesc_pv, jj == 0 ? 1u : 0u,
                   std::make_integer_sequence<int, 8>{});
          tc_commit_warp(&o_ready[w]);
          tc_commit_warp(&v_empty[2 * (u % S) + w]);
          (w ? pt1 : pt0) = -1;
          return true;
        };
        auto qk = [&](int w, int t) -> bool {
          bool& q = w ? q1 : q0;
          if (!q) {
            if (!wwait(&q_full[w], 0u)) return false;
            q = true;
          }
          // P is written over S: the previous PV must be issued first (the
          // tensor pipe keeps issue order). V of that tile reuses the stage of
          // tile u - S, so the other warpgroup's PV of a tile <= u - S, which
          // releases it, goes before it.
          const int u = w ? pt1 : pt0, uo = w ? pt0 : pt1;
          if (u >= 0) {
            if (uo >= 0 && uo <= u - S && !pv(1 - w)) return false;
            if (!pv(w)) return false;
          }
          tc_fence_after();
          if constexpr (F8)
            qk8_all(tmem + C::S_COL + w * 128, smem_desc_sw128(sQa + w * C::QSLOT, 16, 1024),
                    smem_desc_sw128(sKa + (t % S) * C::TILE, 16, 1024), idesc_qk,
                    std::make_integer_sequence<int, 4>{});
          else
            qk_all(tmem + C::S_COL + w * 128, smem_desc_sw128(sQa + w * C::QSLOT, 16, 1024),
                   smem_desc_sw128(sKa + (t % S) * C::TILE, 16, 1024), idesc_qk,
                   std::make_integer_sequence<int, D / 16>{});
          tc_commit_warp(&s_full[w]);
          tc_commit_warp(&k_empty[2 * (t % S) + w]);
          return true;
        };
        // outstanding PVs of tiles below `limit`, oldest first (a younger
        // one's V can depend on the older one's release)
        auto flush_below = [&](int limit) -> bool {
          const bool f0 = pt0 >= 0 && pt0 < limit, f1 = pt1 >= 0 && pt1 < limit;
          if (f0 && f1 && pt1 < pt0) return pv(1) && pv(0);
          return (!f0 || pv(0)) && (!f1 || pv(1));
        };
        bool ok = true;
        for (int t = 0; t < T && ok; ++t) {
          // K(t) needs only the QK^Ts of tile t - S, issued earlier in this loop
          ok = wwait(&k_full[t % S], (uint32_t)(t / S) & 1u);
          if (!ok) break;
          const int nw = tile_need(sched, nseg, t, act);
          if (nw & 1) ok = qk(0, t);
          if (ok && (nw & 2)) ok = qk(1, t);
          if (nw & 1) {
            pt0 = t;
            pj0 = c0++;
          }
          if (nw & 2) {
            pt1 = t;
            pj1 = c1++;
          }
        }
        ok = ok && flush_below(T);
        if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
        // tensor memory is freed only once every issued MMA has completed (an
        // aborting CTA may leave MMAs in flight)
        if (c0 + c1 > 0) {
          tc_commit_warp(mma_done);
          mbar_drain(mma_done, 0u);
        }
      }
    }
    }
    teardown();
  } else {
    regs_claim<C::REGS_SMX>();
    // ---------------------------------------------------------------- softmax warpgroups
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;              // row within the warpgroup's tile
    const int pq = row0 + 128 * w + r;         // query position
    const bool row_valid = pq < p.N;
    const int grp = 2 * w + (r >> 6);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t stm = tmem + lane_off + C::S_COL + w * 128;
    const uint32_t ptm = tmem + lane_off + C::P_COL + w * C::P_STRIDE;
    const uint32_t otm = tmem + lane_off + C::O_COL + w * D;
    const int Iq = (row_valid ? pq : (p.N - 1)) / p.block_q;
    const size_t bias_row = ((size_t)h * p.nQB + Iq) * p.nKB;
    const int my_bit = 1 << (kGrpShift + grp);

    const QWin qw = gna_query_window(p.g, pq, gna_on<MK>(p) && mode == BSA_HEAD_SPARSE);
    const QBox qb = gna_query_box(p.g, qw);
    const bool geo_fast = gna_slice<MK>(p);
    const uint64_t* geo = reinterpret_cast<const uint64_t*>(smem + C::GEO_OFF);

    const float cscale = p.scale_log2;
    // F8: the row's Q scale, and sigma (the head's largest V scale, from warp 2)
    float sigma = 1.f, rsig = 1.f, sq_row = 1.f;
    if constexpr (F8) {
      sigma = __uint_as_float(misc[6]);
      rsig = 1.f / sigma;
      sq_row = __ldg(p.sq + (size_t)bh * p.nSeg + (row_valid ? pq : p.N - 1) / 64);
    }
    float m = kNegInf, l = 0.f;
    int j = 0;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!((tile_need(sched, nseg, t, act) >> w) & 1)) continue;
      // The tile's schedule entries, block bias and masks depend on the
      // schedule alone: they are worked out while its QK^T is in flight.
      const int ea = sched[2 * t];
      const int eb = (2 * t + 1 < nseg) ? sched[2 * t + 1] : -1;
      const int sa = ea & kSegIdxMask;
      const int sb = eb >= 0 ? (eb & kSegIdxMask) : sa;
      float ba = 0.f, bb = 0.f;
      if (p.bias != nullptr) {
        ba = __ldg(p.bias + bias_row + (sa * 64) / p.block_k) * kLog2e;
        bb = __ldg(p.bias + bias_row + (sb * 64) / p.block_k) * kLog2e;
      }
      const bool tail = (sb + 1) * 64 > p.N || (sa + 1) * 64 > p.N;
      const bool need = !(ea & my_bit) || eb < 0 || !(eb & my_bit) || tail ||
                        ((ea | (eb < 0 ? 0 : eb)) & kPart4);
      uint64_t ma = ~0ull, mb = ~0ull;
      if (need) {
        ma = 0ull;
        mb = 0ull;
        if (ea & my_bit) {
          ma = tail_bits(p.N, sa);
          if ((ea & kPart4) && gna_on<MK>(p))
            ma &= geo_fast ? gna_segment_bits_geo(p.g, sa, geo[2 * t], qb) : gna_segment_bits(p.g, sa, qw);
        }
        if (eb >= 0 && (eb & my_bit)) {
          mb = tail_bits(p.N, sb);
          if ((eb & kPart4) && gna_on<MK>(p))
            mb &= geo_fast ? gna_segment_bits_geo(p.g, sb, geo[2 * t + 1], qb) : gna_segment_bits(p.g, sb, qw);
        }
      }
      ok = warp_all(mbar_wait(&s_full[w], (uint32_t)j & 1u, abort_flag, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      // The whole 128-key row of S is read once into registers: with its own
      // P columns, S is free for the next QK^T as soon as it has landed.
      float sv[128];
      tmem_ld32(stm, sv);
      tmem_ld32(stm + 32, sv + 32);
      tmem_ld32(stm + 64, sv + 64);
      tmem_ld32(stm + 96, sv + 96);
      tc_wait_ld();
      if (C::SEP_P) {
        tc_fence_before();
        mbar_arrive(&s_free[w]);
      }
      if (need) {
#pragma unroll
        for (int i = 0; i < 64; ++i) sv[i] = ((ma >> i) & 1ull) ? sv[i] : kNegInf;
#pragma unroll
        for (int i = 0; i < 64; ++i) sv[64 + i] = ((mb >> i) & 1ull) ? sv[64 + i] : kNegInf;
      }
      // row max of the raw scores, per 64-key half (the bias is constant per
      // half): two independent max3 chains per half
      float xa0 = max3f(sv[0], sv[1], sv[2]), xa1 = max3f(sv[3], sv[4], sv[5]);
      float xb0 = max3f(sv[64], sv[65], sv[66]), xb1 = max3f(sv[67], sv[68], sv[69]);
#pragma unroll
      for (int i = 6; i < 62; i += 4) {
        xa0 = max3f(xa0, sv[i], sv[i + 1]);
        xa1 = max3f(xa1, sv[i + 2], sv[i + 3]);
        xb0 = max3f(xb0, sv[64 + i], sv[65 + i]);
        xb1 = max3f(xb1, sv[66 + i], sv[67 + i]);
      }
      const float xa = max3f(xa0, xa1, fmaxf(sv[62], sv[63]));
      const float xb = max3f(xb0, xb1, fmaxf(sv[126], sv[127]));
      // F8: each 64-key half has its own K and V scale; the logit scale takes
      // sq * sk and the exponent offset log2(sv / sigma), so P holds p * sv / sigma
      float csa = cscale, csb = cscale, lva = 0.f, lvb = 0.f;
      if constexpr (F8) {
        const size_t s0 = (size_t)bh * p.nSeg;
        csa = cscale * sq_row * __ldg(p.sk + s0 + sa);
        csb = cscale * sq_row * __ldg(p.sk + s0 + sb);
        lva = fast_log2(__ldg(p.sv + s0 + sa) * rsig);
        lvb = fast_log2(__ldg(p.sv + s0 + sb) * rsig);
      }
      const float ta = (xa == kNegInf) ? kNegInf : fmaf(xa, csa, ba);
      const float tb = (xb == kNegInf) ? kNegInf : fmaf(xb, csb, bb);
      const float m_new = max3f(m, ta, tb);
      float alpha = 1.f;
      if (m_new > m + kRescaleTau) {
        alpha = fast_exp2(m - m_new);
        m = m_new;
      }
      const float mu = (m == kNegInf) ? 0.f : m;
      const float oa = ba - mu + lva, ob = bb - mu + lvb;
      // P = exp2(x - m), packed in registers first: nothing here touches
      // tensor memory, so the exps overlap the previous PV. bf16: two values
      // per 32-bit column; F8: four e4m3 codes per column, and the row sum
      // takes each half's sigma / sv back out.
      constexpr int NPK = F8 ? 32 : 64;
      uint32_t pk[NPK];
      if constexpr (!F8 && !C::SEP_P) {
        // bf16 over S (d = 128): S(j) landing implies PV(j-1) is complete (its
        // QK^T was issued after that PV, and a commit tracks every earlier
        // MMA), so P is written chunk by chunk as it is made, with fewer
        // registers live than the whole row of P
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float o = c < 2 ? oa : ob;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0 = sv[32 * c + 2 * i], x1 = sv[32 * c + 2 * i + 1];
            fma2(x0, x1, cscale, o);
            x0 = fast_exp2(x0);
            x1 = fast_exp2(x1);
            add2(sum0, sum1, x0, x1);
            pk[16 * c + i] = pack_bf16x2(x0, x1);
          }
          tmem_st16(ptm + 16 * c, pk + 16 * c);
        }
        l = l * alpha + (sum0 + sum1);
      } else if constexpr (F8) {
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float o = i < 32 ? oa : ob;
          const float cs = i < 32 ? csa : csb;
          float x0 = sv[2 * i], x1 = sv[2 * i + 1];
          fma2(x0, x1, cs, o);
          x0 = fast_exp2(x0);
          x1 = fast_exp2(x1);
          if (i < 32)
            add2(sa0, sa1, x0, x1);
          else
            add2(sb0, sb1, x0, x1);
          const uint32_t hw = e4m3x2(x0, x1);
          if (i & 1)
            pk[i >> 1] |= hw << 16;
          else
            pk[i >> 1] = hw;
        }
        l = l * alpha + (sa0 + sa1) * fast_exp2(-lva) + (sb0 + sb1) * fast_exp2(-lvb);
      } else {
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float o = i < 32 ? oa : ob;
          float x0 = sv[2 * i], x1 = sv[2 * i + 1];
          fma2(x0, x1, cscale, o);
          x0 = fast_exp2(x0);
          x1 = fast_exp2(x1);
          add2(sum0, sum1, x0, x1);
          pk[i] = pack_bf16x2(x0, x1);
        }
        l = l * alpha + (sum0 + sum1);
      }
      // PV(j-1) must be complete before P is written (own P columns at d = 64,
      // over S at d = 128) and before O is rescaled; O is rescaled once S is
      // dead (fewer live registers), which is safe because PV(j) waits for p_full
      if (j > 0) {
        ok = warp_all(mbar_wait(&o_ready[w], (uint32_t)(j - 1) & 1u, abort_flag, p.wait_limit_ns));
        if (!ok) break;
        tc_fence_after();
      }
      if constexpr (F8 || C::SEP_P) {
#pragma unroll
        for (int c = 0; c < NPK / 16; ++c) tmem_st16(ptm + 16 * c, pk + 16 * c);
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // 16 columns at a time: few registers live in this rarely taken branch
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          float o[16];
          tmem_ld16(otm + c * 16, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tmem_st16(otm + c * 16, reinterpret_cast<uint32_t*>(o));
        }
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[w]);
      ++j;
    }
    if (!ok) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);

    // ---------------------------------------------------------------- epilogue
    // O is staged over the Q tile: a warpgroup that computed nothing has not
    // seen Q land yet
    if (j == 0 && !warp_all(mbar_wait(&q_full[w], 0u, abort_flag, p.wait_limit_ns)))
      cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
    bool have = ok && j > 0;
    if (have) {
      have = warp_all(mbar_wait(&o_ready[w], (uint32_t)(j - 1) & 1u, abort_flag, p.wait_limit_ns));
      if (!have) cta_fail(abort_flag, BSA_DEVERR_TIMEOUT);
      tc_fence_after();
    }
    const float inv = l > 0.f ? sigma / l : 0.f;
    uint8_t* stage = sQ + w * C::QSLOT;  // the Q tile is no longer read once O is final
    const size_t obase = ((size_t)bh * p.N + (row_valid ? pq : 0)) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      if (have) {
        tmem_ld32(otm + c * 32, o);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= inv;
      const int chunk = c >> 1;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
        v.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
        v.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
        v.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
        const int unit = 4 * (c & 1) + q;
        *reinterpret_cast<uint4*>(stage + chunk * C::CHUNK + r * 128 + ((unit ^ (r & 7)) << 4)) = v;
      }
      if (p.cache_out != nullptr && row_valid) {
        float4* cd = reinterpret_cast<float4*>(p.cache_out + obase + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) cd[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
    }
    fence_proxy_async_smem();
    named_bar(1 + w, 128);
    if (q4 == 0 && lane == 0 && (act >> w) & 1) {
      for (int c = 0; c < D / 64; ++c)
        for (int rr = 0; rr < 2; ++rr)
          if (row0 + 128 * w + 64 * rr < p.N)
            tma_store_3d(&tmO, stage + c * C::CHUNK + rr * (C::CHUNK / 2), c * 64, row0 + 128 * w + 64 * rr,
                         bh);
      bulk_commit();
      bulk_wait_read();
    }
    teardown();
  }
}

template <int D, bool F8, int MK = kMaskAny>
static cudaError_t launch_fwd_d(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const CUtensorMap& o, const AttnParams& p, int grid, cudaStream_t stream) {
  using C = FwdCfg<D, F8>;
  auto fn = fwd_kernel<D, F8, MK>;
  static DeviceOnce once;
  const cudaError_t e = once.run([&]() -> cudaError_t {
    // the register split needs the full launch allocation: a smaller one
    // would leave setmaxnreg.inc waiting, so refuse to launch instead
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, fn);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  });
  if (e != cudaSuccess) return e;
  fn<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(q, k, v, o, p);
  return cudaGetLastError();
}

cudaError_t launch_forward(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const CUtensorMap& o, const AttnParams& p, int grid, cudaStream_t stream) {
  if (d == 64) return launch_fwd_d<64, false>(q, k, v, o, p, grid, stream);
  if (p.has_gna && p.g.seg_one_slice) return launch_fwd_d<128, false, kMaskGnaSlice>(q, k, v, o, p, grid, stream);
  return launch_fwd_d<128, false>(q, k, v, o, p, grid, stream);
}

cudaError_t launch_forward_fp8(const CUtensorMap& q8, const CUtensorMap& k8, const CUtensorMap& v8t,
                               const CUtensorMap& o, const AttnParams& p, int grid, cudaStream_t stream) {
  if (p.has_gna && p.g.seg_one_slice) return launch_fwd_d<128, true, kMaskGnaSlice>(q8, k8, v8t, o, p, grid, stream);
  return launch_fwd_d<128, true>(q8, k8, v8t, o, p, grid, stream);
}

}  // namespace bsa
