/*
 * bsa.h - block-sparse attention for diffusion transformers on B200 (sm_100a).
 *
 * A small C ABI over hand-written CUDA kernels. Every pointer argument named
 * "device" is caller-owned device memory; the library never allocates device
 * memory, never synchronises the host (except bsa_get_device_error) and has
 * no CPU fallback. The one host-only routine, bsa_plan_heads, works on host
 * arrays.
 * All launches are asynchronous on the caller's stream, passed as `void*`
 * holding a cudaStream_t (NULL = legacy default stream).
 *
 * Tensor layout: Q, K, V and O are bf16 [B, H, N, d], row-major, d innermost
 * and contiguous, 16-byte aligned. Text tokens come first in the sequence,
 * followed by the image (or video) tokens.
 *
 * Return values: BSA_OK or one of the BSA_ERR_* codes below. Argument checks
 * happen on the host before any launch; a failed check launches nothing.
 * Faults found by kernels (an out-of-range block index, a bounded pipeline
 * wait that ran out) are recorded in a device error word, read with
 * bsa_get_device_error.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define BSA_OK 0
#define BSA_ERR_INVALID_ARG 1  /* null pointer, bad size, inconsistent shapes  */
#define BSA_ERR_UNSUPPORTED 2  /* valid request outside what the kernels cover */
#define BSA_ERR_WORKSPACE 3    /* workspace missing or smaller than required   */
#define BSA_ERR_CUDA 4         /* a CUDA runtime/driver call failed            */
#define BSA_ERR_DEVICE 5       /* a kernel recorded a fault (see below)        */
#define BSA_ERR_INFEASIBLE 6   /* no plan meets the error budget               */

/* device error word values (bsa_get_device_error) */
#define BSA_DEVERR_NONE 0
#define BSA_DEVERR_BAD_INDEX 1     /* block index outside [0, nKB) or count > max_k */
#define BSA_DEVERR_TIMEOUT 2       /* a bounded mbarrier wait gave up              */
#define BSA_DEVERR_SCHEDULE 3      /* a row's KV schedule exceeded the kernel cap  */
#define BSA_DEVERR_NO_GEOMETRY 4   /* a PARTIAL block met without a fine-mask geometry */

/* ---- per-head modes (DiTFastAttnV2, "Fused Kernel": each head picks full,
 *      skip with the cached output of the previous step, or arrow) ------- */
#define BSA_HEAD_FULL 0    /* all KV blocks                              */
#define BSA_HEAD_SPARSE 1  /* the KV blocks of the block list            */
#define BSA_HEAD_SKIP 2    /* O = bf16(cache_in), nothing computed       */

/* ---- block classes (bitmap values and block-list flags) ----------------- */
#define BSA_BLOCK_NONE 0
#define BSA_BLOCK_FULL 1     /* every real (query, key) pair allowed           */
#define BSA_BLOCK_PARTIAL 2  /* some pairs allowed: fine mask inside the block */

#define BSA_MASK_ARROW 1
#define BSA_MASK_GNA 2

/* ---- denoising-step actions (bsa_step_action) ------------------------- */
#define BSA_STEP_FULL 0    /* full attention, no pattern yet              */
#define BSA_STEP_SELECT 1  /* select the head-specific pattern, then sparse */
#define BSA_STEP_REUSE 2   /* sparse with the pattern selected earlier    */

#define BSA_SELECT_POOLED_QK 1    /* mean-pooled Q/K block scores              */
#define BSA_SELECT_FULL_SCORE 2   /* avg-pooled softmax map (SparseD)          */

/* Problem shape. block_q / block_k: tokens per query / key block (the mask
 * granularity); n_text: text tokens at the front of the sequence. */
typedef struct {
  int32_t B, H, N, d;
  int32_t block_q, block_k;
  int32_t n_text;
} bsa_dims;

/* GNA geometry (jsqmd.com GNA article, section 1.1): a 1..3-D token grid
 * (outermost dimension first), tile extent, window and stride per dimension.
 * Per dimension of length L, window k and stride s, query i reads keys
 * [start, start + k) with start = clamp(s*floor(i/s) - s*floor((k-s)/(2s)),
 * 0, L-k). Tokens are in tile order (see bsa_permute_tiles). */
typedef struct {
  int32_t ndim;
  int32_t grid[3];
  int32_t tile[3];
  int32_t window[3];
  int32_t stride[3];
} bsa_gna_geom;

typedef struct {
  int32_t kind;               /* BSA_MASK_ARROW or BSA_MASK_GNA               */
  const int32_t* head_mode;   /* device int32 [H], BSA_HEAD_*; NULL = all SPARSE */
  const int32_t* window;      /* device int32 [H], arrow half-width in blocks  */
  bsa_gna_geom gna;           /* GNA only                                      */
} bsa_mask_spec;

/* Block list (one row per (b, h, query block)). idx holds the kept KV block
 * indices in ascending order, padded with -1; flag holds each entry's class
 * (BSA_BLOCK_FULL / BSA_BLOCK_PARTIAL), padded with 0. bitmap (optional,
 * NULL to skip) holds the class of every (query block, KV block) pair. */
typedef struct {
  int32_t* cnt;     /* device int32 [B, H, nQB]          */
  int32_t* idx;     /* device int32 [B, H, nQB, max_k]   */
  uint8_t* flag;    /* device uint8 [B, H, nQB, max_k]   */
  uint8_t* bitmap;  /* device uint8 [B, H, nQB, nKB] or NULL */
  int32_t max_k;    /* row capacity, 1 <= max_k          */
} bsa_block_list;

/* A range [begin, end) of KV blocks whose top-k is cut on its own. */
typedef struct {
  int32_t begin, end, k;
} bsa_key_group;

typedef struct {
  int32_t method;            /* BSA_SELECT_POOLED_QK or BSA_SELECT_FULL_SCORE */
  int32_t n_groups;          /* 1..4                                          */
  bsa_key_group groups[4];
  int32_t keep_text;         /* 1: text KV blocks always kept, text rows full */
  float scale;               /* logit scale (FULL_SCORE), usually 1/sqrt(d)   */
} bsa_select_spec;

/* Library version (major*10000 + minor*100 + patch). */
int bsa_version(void);

/* Human-readable text of a BSA_* status code (static storage). */
const char* bsa_error_string(int status);

/* bsa_build_mask: fixed patterns to a block list.
 *  ARROW (DiTFastAttnV2, "Head-wise Arrow Attention" and "Fused Kernel"):
 *    block (I, J) is kept iff I or J holds a text token or |I - J| <= w_h;
 *    kept blocks are dense (FULL). Needs block_q == block_k.
 *  GNA (jsqmd.com GNA article, sections 1.1 and 2.1): tile-order tokens,
 *    block size == tile volume; a (Q tile, KV tile) pair is FULL when every
 *    real pair is inside the window, PARTIAL when some are, dropped when none
 *    are; text rows and columns are full; padded tokens are never keys.
 *  FULL heads keep every block, SKIP heads keep none (cnt = 0).
 *  Writes cnt, idx, flag (and bitmap if non-NULL) for all B*H*nQB rows.
 *  Errors: INVALID_ARG (null pointers, max_k < nKB, bad geometry),
 *  UNSUPPORTED (arrow with block_q != block_k; GNA with tile x-extent that is
 *  neither a divisor nor a multiple of 64, or block size != tile volume). */
int bsa_build_mask(const bsa_dims* dims, const bsa_mask_spec* spec,
                   const bsa_block_list* out, void* stream);

/* Workspace bytes bsa_select_topk needs for these dims and spec. POOLED_QK:
 * the pooled Q and K blocks, fp32. FULL_SCORE: A' (B*H*nQB*nKB floats)
 * plus the per-tile row LSEs of the one-pass form, 4 * ceil(N/128) * block_q
 * bytes per query block, for all B*H*nQB query blocks or as many as 1 GiB
 * holds (the selection then runs over the query blocks in chunks of that
 * many): e.g. 1.07 GB at 32 heads x 32768 tokens, block 128. */
size_t bsa_select_workspace_size(const bsa_dims* dims, const bsa_select_spec* spec);

/* bsa_select_topk: content-driven block selection.
 *  POOLED_QK (lmnt.cn BSA post, sections 2.2-2.3): each block is mean-pooled
 *    (fp32, ragged last block over its real tokens); score(I,J) = Qbar_I .
 *    Kbar_J in fp32; each group keeps its top k by descending score, ties to
 *    the lower index. keep_text: text KV blocks always kept (not counted in
 *    k) and text query rows keep every block.
 *  FULL_SCORE (SparseD, "Isolated Selection"): A = softmax(scale*QK^T + bias)
 *    over all keys, A' = avgpool(A, block); each group (e.g. prefill and
 *    generation key blocks) keeps its own top k per query block. QK^T and
 *    its exps are evaluated once: the log-sum-exp of every row over every
 *    128-key tile, then each row's LSE and A' from those alone.
 *  block_bias: optional device fp32 [H, nQB, nKB] logit offset (FULL_SCORE).
 *  Writes the block list (all entries FULL). Workspace: device, at least
 *  bsa_select_workspace_size bytes, 256-byte aligned; contents are scratch.
 *  Errors: INVALID_ARG, UNSUPPORTED (d not 64/128, FULL_SCORE with block size
 *  not a multiple of 128 or block_q != block_k), WORKSPACE. */
int bsa_select_topk(const bsa_dims* dims, const void* Q, const void* K,
                    const bsa_select_spec* spec, const float* block_bias,
                    void* workspace, size_t workspace_bytes,
                    const bsa_block_list* out, void* stream);

/* Size of the library-owned scratch behind bsa_select_topk_static: 16 MiB,
 * enough for the pooled selection at 24 heads x 16896 tokens (3.2 MB) and the
 * full-score selection at 32 heads x 32768 tokens (12 MB in its two-pass
 * form, below). */
#define BSA_STATIC_SCRATCH_BYTES (16u << 20)

/* bsa_select_topk_static: bsa_select_topk without a caller workspace. The
 * pages have no counterpart; this entry point exists for callers that cannot
 * allocate device memory at call time - runtimes that plan every device
 * buffer ahead in a fixed arena, or latency-critical loops that must not
 * call cudaMalloc (which can synchronise the device) - but still own Q, K
 * and the block list.
 *  Same arguments and results as bsa_select_topk, minus the workspace. For
 *  FULL_SCORE the scratch runs the one-pass form when it holds the per-tile
 *  LSEs of at least 1024 query tiles (or of all of them), in as many chunks
 *  as it takes; otherwise the two-pass form: a first pass over QK^T for each
 *  row's LSE (B*H*N floats), a second that adds exp2(z - LSE) into A' (B*H*
 *  nQB*nKB floats). The two forms round differently, so a near-tie between
 *  two key blocks may fall the other way than in bsa_select_topk.
 *  The scratch is a fixed BSA_STATIC_SCRATCH_BYTES array inside the library; every
 *  GPU that loads the library holds it until the process exits. Nothing is
 *  allocated: no cudaMalloc, no cudaFree, no allocating library call.
 *  The first call on a device looks up the array's device address
 *  (cudaGetSymbolAddress) with that device current; make that first call
 *  before any stream capture on the device. The address is cached for the
 *  life of the process: it is not valid across a device reset
 *  (cudaDeviceReset or a primary-context reset), after which this entry
 *  point must not be called again in the same process.
 *  All calls share the one array, which keeps the previous call's contents
 *  (the kernels clear what must start at zero). Calls whose kernels overlap on
 *  the GPU (e.g. on two streams) race on the scratch: serialise them.
 *  Errors: bsa_select_topk's argument checks run first and give the same
 *  INVALID_ARG / UNSUPPORTED status; then BSA_ERR_WORKSPACE when neither
 *  form fits in BSA_STATIC_SCRATCH_BYTES (POOLED_QK: when
 *  bsa_select_workspace_size exceeds it); then the CUDA errors of
 *  bsa_select_topk. */
int bsa_select_topk_static(const bsa_dims* dims, const void* Q, const void* K,
                           const bsa_select_spec* spec, const float* block_bias,
                           const bsa_block_list* out, void* stream);

/* bsa_forward: FlashAttention-style forward over the kept blocks only
 * (lmnt.cn BSA post, section 3.1: tiles, online softmax, a block-index
 * variant; DiTFastAttnV2 "Fused Kernel": three per-head modes).
 *  For each (b, h): SKIP -> O = bf16(cache_in), round to nearest even.
 *  Otherwise each query row attends the keys of its kept blocks:
 *    z = scale * q.k + bias(I, J); o = softmax(z) V, fp32 accumulation,
 *    O rounded to bf16; PARTIAL blocks apply the GNA fine mask from `gna`.
 *  A row with no kept key gives 0.
 *  head_mode: device int32 [H]. list: needed when any head is SPARSE.
 *  gna: host struct, NULL unless the list has PARTIAL blocks or the tile
 *  layout has padding. cache_in: device fp32 [B,H,N,d], needed when any head
 *  is SKIP. cache_out: NULL or device fp32 [B,H,N,d]; receives the fp32
 *  output of computed heads (SKIP heads are not written).
 *  block_bias: NULL or device fp32 [H, nQB, nKB], natural-log units.
 *  Errors: INVALID_ARG, UNSUPPORTED (d not 64/128, block sizes not multiples
 *  of 64, N > 131072), CUDA. */
int bsa_forward(const bsa_dims* dims, const void* Q, const void* K, const void* V,
                const bsa_block_list* list, const int32_t* head_mode,
                const bsa_gna_geom* gna, const float* cache_in, float* cache_out,
                const float* block_bias, float scale, void* O, void* stream);

/* bsa_quantize_fp8: the e4m3 operands of bsa_forward_fp8 (jsqmd.com GNA
 * article, section 2.1, Blackwell adaptation: FP8 for more tensor-core
 * throughput; the article gives no scheme). Each 64-token block of each
 * (b, h) of Q, K and V gets one scale s = amax / 448 (1 for an all-zero
 * block); the code of x is e4m3(fl32(x * r)) with r = fl32(448 / amax), round
 * to nearest even, saturating at 448.
 *  Q, K, V: device bf16 [B, H, N, 128].
 *  q8, k8: device uint8 [B, H, N, 128] (codes, the layout of Q and K).
 *  v8t: device uint8 [B, H, 128, Nt], V transposed per head, Nt = N rounded
 *    up to a multiple of 16; columns N..Nt-1 are written as zero.
 *  sq, sk, sv: device float [B, H, ceil(N / 64)] (the dequantisation scales).
 *  All caller-owned; every output is overwritten.
 *  Errors: INVALID_ARG (null or misaligned pointer, bad dims), UNSUPPORTED
 *  (d != 128, B * H > 65535), CUDA. */
int bsa_quantize_fp8(const bsa_dims* dims, const void* Q, const void* K, const void* V, uint8_t* q8,
                     uint8_t* k8, uint8_t* v8t, float* sq, float* sk, float* sv, void* stream);

/* bsa_forward_fp8: bsa_forward on the e4m3 operands of bsa_quantize_fp8 (same
 * sections as bsa_quantize_fp8): the attention of the dequantised Q, K and V
 * (code * scale) over the kept blocks, with the tensor-core products on the
 * e4m3 codes, P rounded to e4m3 (scaled into range: P holds p * sv / sigma,
 * sigma the head's largest V scale) and fp32 accumulation; O is bf16
 * [B, H, N, 128]. Arguments as bsa_forward, with q8, k8, v8t, sq, sk, sv in
 * place of Q, K and V.
 *  Errors: as bsa_forward, and UNSUPPORTED for d != 128, block_k not a
 *  multiple of 128, or a GNA tile volume not a multiple of 128. */
int bsa_forward_fp8(const bsa_dims* dims, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t,
                    const float* sq, const float* sk, const float* sv, const bsa_block_list* list,
                    const int32_t* head_mode, const bsa_gna_geom* gna, const float* cache_in,
                    float* cache_out, const float* block_bias, float scale, void* O, void* stream);

/* Length of the tile-order sequence for a raster sequence of n_text text
 * tokens plus the GNA grid: text padded to a multiple of the tile volume,
 * plus every (padded) tile. Host only. */
int bsa_gna_tiled_len(int32_t n_text, const bsa_gna_geom* geom, int32_t* n_tiled);

/* bsa_permute_tiles / bsa_unpermute_tiles (jsqmd.com GNA article, section
 * 2.2: token permutation fused with padding in one copy kernel).
 *  permute: `in[t]` raster [B, H, n_text + prod(grid), d] bf16 ->
 *    `out[t]` tile order [B, H, n_tiled, d] bf16, padding rows zeroed.
 *  unpermute: the inverse; padding rows are dropped.
 *  dims: B, H, d and n_text are read (N and block sizes are ignored).
 *  in/out: HOST arrays of n_tensors (1..4) device pointers.
 *  Errors: INVALID_ARG, UNSUPPORTED (d not a multiple of 8). */
int bsa_permute_tiles(const bsa_dims* dims, const bsa_gna_geom* geom, int32_t n_tensors,
                      const void* const* in, void* const* out, void* stream);
int bsa_unpermute_tiles(const bsa_dims* dims, const bsa_gna_geom* geom, int32_t n_tensors,
                        const void* const* in, void* const* out, void* stream);

/* bsa_rse: the single-layer relative squared error of a compressed output,
 * per head (DiTFastAttnV2, "efficient compression plan search"):
 *   I(h) = sum (y_m - y_o)^2 / sum (y_o - mean(y_o))^2
 * with the sums over head h's outputs of every batch item, token and channel
 * (the printed numerator subtracts mean(y_o); read as y_m - y_o).
 *  dims: B, H, N and d are read (block sizes and n_text are ignored).
 *  y_m, y_o: device bf16 [B, H, N, d]: the output under a method m and the
 *    uncompressed output of the same layer and inputs.
 *  out: device double [4 * H], caller-owned, overwritten: out[h] = I(h);
 *    out[H + 3h + 0..2] = sum (y_m - y_o)^2, sum y_o, sum y_o^2 (fp64).
 *    A head whose y_o is constant has a zero denominator (I = inf or NaN).
 *  Errors: INVALID_ARG (null pointer, bad dims), UNSUPPORTED (N*d not a
 *  multiple of 8, or B or H above 65535), CUDA. */
int bsa_rse(const bsa_dims* dims, const void* y_m, const void* y_o, double* out, void* stream);

/* bsa_plan_heads: the head-wise compression plan of one layer and step
 * (DiTFastAttnV2, "efficient compression plan search"): one method per head
 * minimising the total latency subject to
 *   I(h, m_h) <= c * delta / H   for every head (c = 1.5 in the pages), and
 *   sum_h I(h, m_h) <= delta.
 * Exact: a dynamic program over the integer total cost. Host only (no GPU).
 *  rse: host double [H * M], rse[h * M + m] = I(h, m) (from bsa_rse).
 *  cost: host int64 [H * M], >= 0, the latency of method m on head h in any
 *    integer unit (the number of computed blocks for the attention modes).
 *  choice: host int32 [H] out, the chosen method per head. Among plans of
 *    equal cost the one with the least total error is returned.
 *  total_cost: host int64 out, may be NULL.
 *  Uses host memory proportional to H * (sum over heads of the largest cost).
 *  Errors: INVALID_ARG (null pointer, H or M < 1, negative cost, delta or c
 *  negative or not finite), UNSUPPORTED (H * (that sum + 1) above 2^28:
 *  express costs in coarser units), INFEASIBLE. */
int bsa_plan_heads(int32_t H, int32_t M, const double* rse, const int64_t* cost, double delta, double c,
                   int32_t* choice, int64_t* total_cost);

/* Step schedule of the sparse path (SparseD, "overall framework": the first
 * T x skip% denoising steps run full attention, the head-specific pattern is
 * selected once at that step and reused by every later step; the GNA
 * article's image results split 9 full steps of 28 the same way). Host only.
 *  bsa_schedule_full_steps: *n_full = ceil(n_steps * skip_pct / 100).
 *  bsa_step_action: *action = BSA_STEP_FULL for step < n_full,
 *    BSA_STEP_SELECT at step == n_full, BSA_STEP_REUSE after.
 *  Errors: INVALID_ARG (null output, n_steps < 1, step outside
 *  [0, n_steps), n_full outside [0, n_steps], skip_pct outside [0, 100]). */
int bsa_schedule_full_steps(int32_t n_steps, int32_t skip_pct, int32_t* n_full);
int bsa_step_action(int32_t step, int32_t n_steps, int32_t n_full, int32_t* action);

/* bsa_keep_pct: the kept-block percentage of a layer and denoising step
 * (lmnt.cn BSA post, section 3.3: shallow layers and early steps keep more,
 * about 30%, deep layers and late steps fewer, 10-15%; no formula is given).
 * Reading: hi - (hi - lo) * (layer / (n_layers - 1) + step / (n_steps - 1)) / 2,
 * a fraction being 0 when its count is 1, rounded to the nearest integer,
 * halves up; exact integer arithmetic. Host only.
 *  Errors: INVALID_ARG (null output, counts < 1, indices out of range,
 *  percentages outside [0, 100]). */
int bsa_keep_pct(int32_t layer, int32_t n_layers, int32_t step, int32_t n_steps, int32_t hi, int32_t lo,
                 int32_t* pct);

/* bsa_jaccard: how stable a selection is across steps (SparseD, "sparse
 * reuse"): per (b, h, query block) row, |A n B| / |A u B| of the kept KV
 * block sets of two block lists (two empty rows score 1).
 *  dims: B, H, N and block_q give the rows (B * H * ceil(N / block_q)).
 *  a, b: block lists with ascending rows (as bsa_build_mask and
 *    bsa_select_topk write them); cnt and idx are read.
 *  out: device float [B, H, nQB], caller-owned, overwritten.
 *  A count outside [0, max_k] records BSA_DEVERR_BAD_INDEX (clamped).
 *  Errors: INVALID_ARG, CUDA. */
int bsa_jaccard(const bsa_dims* dims, const bsa_block_list* a, const bsa_block_list* b, float* out, void* stream);

/* Synchronise `stream`, then read and clear the device error word.
 * *code receives a BSA_DEVERR_* value. Returns BSA_OK, or BSA_ERR_CUDA if the
 * synchronisation itself failed. */
int bsa_get_device_error(void* stream, int32_t* code);

/* Failure detection (the pages have none; this is the library's own). Every
 * pipeline wait inside bsa_forward and bsa_select_topk's full-score passes is
 * bounded: a wait that runs out raises BSA_DEVERR_TIMEOUT in the device error
 * word and its CTA aborts: copies and tensor-core operations already in
 * flight are drained (under the default bound), tensor memory is freed and
 * the CTA exits, so the context stays usable. Both settings below are
 * process-wide and apply to calls made after them.
 *
 * bsa_set_wait_limit_ns: the bound of each pipeline wait, in nanoseconds;
 * 0 restores the default of 2 s. Always returns BSA_OK. */
int bsa_set_wait_limit_ns(uint64_t ns);

/* bsa_set_withheld_tile: for tests of the above. When tile >= 0, every
 * bsa_forward CTA that has a key tile with that index in its schedule never
 * loads that tile's K, so the waits on it run out (after the wait limit) and
 * the forward ends with BSA_DEVERR_TIMEOUT and an undefined O. -1 (the
 * default) turns it off. Errors: INVALID_ARG for tile < -1. */
int bsa_set_withheld_tile(int32_t tile);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */
