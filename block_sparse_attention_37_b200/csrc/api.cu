// C ABI of the library (include/bsa.h): argument checks, TMA descriptors and
// launches. No allocation, no host synchronisation except in
// bsa_get_device_error, no CPU fallback.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>

#include "attention.cuh"
#include "mask.cuh"
#include "permute.cuh"
#include "quant.cuh"
#include "select.cuh"

namespace bsa {


namespace {

constexpr int kVersion = 100;  // 0.1.0

int cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

// Failure-detection settings read by every later launch (bsa_set_wait_limit_ns,
// bsa_set_withheld_tile).
std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};
std::atomic<int> g_withheld_tile{-1};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ---- driver entry point for tensor-map encoding (no link-time libcuda) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, N, d] bf16 viewed as a 3-D tensor; 64x64 boxes, 128-byte swizzle.
// Rows past N of a head read as zero.
int make_map(CUtensorMap* m, const void* base, long long BH, int N, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return BSA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSA_OK : BSA_ERR_CUDA;
}

// [BH, rows, inner] bytes (e4m3 codes) as a 3-D tensor; 128-byte x 64-row
// boxes, 128-byte swizzle; reads past `rows` or `inner` give zero.
int make_map8(CUtensorMap* m, const void* base, long long BH, int rows, int inner) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return BSA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)inner, (cuuint64_t)rows * inner};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSA_OK : BSA_ERR_CUDA;
}

int round16(int n) { return (n + 15) & ~15; }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Geometry checks shared by mask building, the forward and the permutation.
int make_gna(const bsa_gna_geom* in, int n_text, GnaDev* g) {
  if (!in || in->ndim < 1 || in->ndim > 3 || n_text < 0) return BSA_ERR_INVALID_ARG;
  const int pad = 3 - in->ndim;
  long long vol = 1, ntiles = 1;
  for (int d = 0; d < 3; ++d) {
    const int s = d - pad;
    g->grid[d] = s < 0 ? 1 : in->grid[s];
    g->tile[d] = s < 0 ? 1 : in->tile[s];
    g->win[d] = s < 0 ? 1 : in->window[s];
    g->stride[d] = s < 0 ? 1 : in->stride[s];
    if (g->grid[d] < 1 || g->tile[d] < 1 || g->stride[d] < 1 || g->stride[d] > g->win[d] ||
        g->win[d] > g->grid[d])
      return BSA_ERR_INVALID_ARG;
    g->tiles[d] = ceil_div(g->grid[d], g->tile[d]);
    vol *= g->tile[d];
    ntiles *= g->tiles[d];
  }
  if (vol > (1 << 20)) return BSA_ERR_UNSUPPORTED;
  g->vol = (int)vol;
  g->n_text = n_text;
  g->text_span = ceil_div(n_text, vol) * (int)vol;
  long long n_tiled = (long long)g->text_span + ntiles * vol;
  if (n_tiled > (1ll << 30)) return BSA_ERR_UNSUPPORTED;
  g->f_vol = make_fastdiv(g->vol);
  g->f_tiles2 = make_fastdiv(g->tiles[2]);
  g->f_tiles1 = make_fastdiv(g->tiles[1]);
  g->f_tile2 = make_fastdiv(g->tile[2]);
  g->f_tile1 = make_fastdiv(g->tile[1]);
  const int tx = g->tile[2];
  g->seg_one_slice = tx <= 64 && 64 % tx == 0 && g->tile[1] % (64 / tx) == 0;
  g->x_rep = 0ull;
  g->seg_rows = 0;
  g->x_mask = 0ull;
  if (g->seg_one_slice) {
    g->seg_rows = 64 / tx;
    for (int r = 0; r < g->seg_rows; ++r) g->x_rep |= 1ull << (tx * r);
    g->x_mask = tx >= 64 ? ~0ull : ((1ull << tx) - 1ull);
  }
  g->has_padding = g->text_span > n_text;
  for (int d = 0; d < 3; ++d) g->has_padding |= (g->grid[d] % g->tile[d]) != 0;
  return BSA_OK;
}

long long tiled_len(const GnaDev& g) {
  return (long long)g.text_span + (long long)g.tiles[0] * g.tiles[1] * g.tiles[2] * g.vol;
}

int check_dims(const bsa_dims* dm) {
  if (!dm) return BSA_ERR_INVALID_ARG;
  if (dm->B < 1 || dm->H < 1 || dm->N < 1 || dm->d < 1 || dm->block_q < 1 || dm->block_k < 1 ||
      dm->n_text < 0 || dm->n_text > dm->N)
    return BSA_ERR_INVALID_ARG;
  if ((long long)dm->B * dm->H * dm->N * dm->d > (1ll << 40)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int check_list(const bsa_block_list* l, int nKB) {
  if (!l || !l->cnt || !l->idx || !l->flag || l->max_k < nKB) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of the selection. POOLED_QK: qbar, kbar. FULL_SCORE, one-pass
// form (chunk > 0): apool (block_q / 128 partial rows per query block), then
// the per-tile LSE slabs of `chunk` query blocks, the selection running over
// the query blocks that many at a time; two-pass form (chunk = 0): lse,
// apool (one row per query block).
struct SelectLayout {
  size_t qbar, kbar, lse, apool, tlse, total;
  long long chunk;
};

// The one-pass slabs of one chunk take at most this many bytes in the
// reported workspace size, so that the workspace stays bounded at any N.
constexpr size_t kTlseCapBytes = size_t(1) << 30;
// A one-pass chunk smaller than this many score CTAs (about three waves at
// two CTAs per SM) would leave much of the GPU idle: the two-pass form then
// runs instead.
constexpr long long kOnePassMinCtas = 1024;

struct FullScoreGeom {
  long long units;    // query blocks, B * H * nQB
  int m;              // 128-row query tiles per query block
  size_t unit_bytes;  // slab bytes of one query block
  long long min_chunk;
};

FullScoreGeom full_score_geom(const bsa_dims* dm) {
  FullScoreGeom g;
  const long long nQB = ceil_div(dm->N, dm->block_q);
  g.units = (long long)dm->B * dm->H * nQB;
  g.m = dm->block_q >= 128 ? dm->block_q / 128 : 1;
  g.unit_bytes = (size_t)g.m * (size_t)ceil_div(dm->N, 128) * 128 * sizeof(float);
  g.min_chunk = std::min(g.units, (kOnePassMinCtas + g.m - 1) / g.m);
  return g;
}

SelectLayout two_pass_layout(const bsa_dims* dm) {
  SelectLayout L{0, 0, 0, 0, 0, 0, 0};
  const size_t BH = (size_t)dm->B * dm->H;
  const size_t nQB = ceil_div(dm->N, dm->block_q), nKB = ceil_div(dm->N, dm->block_k);
  L.apool = align256(BH * dm->N * sizeof(float));
  L.total = L.apool + align256(BH * nQB * nKB * sizeof(float));
  return L;
}

SelectLayout one_pass_layout(const bsa_dims* dm, long long chunk) {
  SelectLayout L{0, 0, 0, 0, 0, 0, chunk};
  const FullScoreGeom g = full_score_geom(dm);
  const size_t nKB = ceil_div(dm->N, dm->block_k);
  L.tlse = align256((size_t)g.units * g.m * nKB * sizeof(float));
  L.total = L.tlse + (size_t)chunk * g.unit_bytes;
  return L;
}

// The layout bsa_select_workspace_size reports: for FULL_SCORE the one-pass
// form with every query block in one chunk, or as many as kTlseCapBytes holds.
SelectLayout select_layout(const bsa_dims* dm, const bsa_select_spec* sp) {
  if (sp->method == BSA_SELECT_POOLED_QK) {
    SelectLayout L{0, 0, 0, 0, 0, 0, 0};
    const size_t BH = (size_t)dm->B * dm->H;
    const size_t nQB = ceil_div(dm->N, dm->block_q), nKB = ceil_div(dm->N, dm->block_k);
    L.kbar = align256(BH * nQB * dm->d * sizeof(float));
    L.total = L.kbar + align256(BH * nKB * dm->d * sizeof(float));
    return L;
  }
  const FullScoreGeom g = full_score_geom(dm);
  const long long cap = std::max(1ll, (long long)(kTlseCapBytes / g.unit_bytes));
  return one_pass_layout(dm, std::min(g.units, std::max(cap, g.min_chunk)));
}

// The layout a workspace of `bytes` runs: for FULL_SCORE the one-pass form
// with as many query blocks per chunk as the bytes hold, if that is at least
// the minimum chunk, else the two-pass form. total > bytes: neither fits.
SelectLayout layout_for_bytes(const bsa_dims* dm, const bsa_select_spec* sp, size_t bytes) {
  if (sp->method == BSA_SELECT_POOLED_QK) return select_layout(dm, sp);
  const FullScoreGeom g = full_score_geom(dm);
  const size_t base = one_pass_layout(dm, 0).tlse;
  if (bytes > base) {
    const long long chunk = std::min(g.units, (long long)((bytes - base) / g.unit_bytes));
    if (chunk >= g.min_chunk) return one_pass_layout(dm, chunk);
  }
  return two_pass_layout(dm);
}

// Every argument check of bsa_select_topk except the workspace's, in the
// order that call makes them. bsa_select_topk_static runs it before its own
// scratch-size check, so both entry points report the same status for the
// same unsupported or invalid request.
int check_select_args(const bsa_dims* dims, const void* Q, const void* K, const bsa_select_spec* spec,
                      const bsa_block_list* out) {
  int st = check_dims(dims);
  if (st != BSA_OK) return st;
  if (!spec || !Q || !K || !aligned16(Q) || !aligned16(K)) return BSA_ERR_INVALID_ARG;
  if (dims->d != 64 && dims->d != 128) return BSA_ERR_UNSUPPORTED;
  const int nKB = ceil_div(dims->N, dims->block_k);
  if ((st = check_list(out, nKB)) != BSA_OK) return st;
  if (spec->n_groups < 0 || spec->n_groups > 4) return BSA_ERR_INVALID_ARG;
  for (int g = 0; g < spec->n_groups; ++g) {
    const bsa_key_group& kg = spec->groups[g];
    if (kg.begin < 0 || kg.end > nKB || kg.begin > kg.end || kg.k < 0) return BSA_ERR_INVALID_ARG;
  }
  if (spec->method != BSA_SELECT_POOLED_QK && spec->method != BSA_SELECT_FULL_SCORE) return BSA_ERR_INVALID_ARG;
  if ((size_t)nKB * 5 > 200 * 1024) return BSA_ERR_UNSUPPORTED;
  if (spec->method == BSA_SELECT_FULL_SCORE) {
    if (dims->block_q != dims->block_k || dims->block_q % 128 != 0) return BSA_ERR_UNSUPPORTED;
    if (ceil_div(dims->N, 64) > kMaxSeg) return BSA_ERR_UNSUPPORTED;
  }
  return BSA_OK;
}

// The checks and parameters both forwards share (everything but the
// operand maps). gna_vol_mult: the tile volume a GNA layout must be a
// multiple of (64 for the bf16 forward, 128 for the e4m3 one).
int forward_params(const bsa_dims* dims, const bsa_block_list* list, const int32_t* head_mode,
                   const bsa_gna_geom* gna, const float* cache_in, float* cache_out, const float* block_bias,
                   float scale, void* O, int gna_vol_mult, AttnParams* out) {
  if (!O || !head_mode || !aligned16(O)) return BSA_ERR_INVALID_ARG;
  if ((cache_in && !aligned16(cache_in)) || (cache_out && !aligned16(cache_out))) return BSA_ERR_INVALID_ARG;
  if (ceil_div(dims->N, 64) > kMaxSeg) return BSA_ERR_UNSUPPORTED;
  const int nQB = ceil_div(dims->N, dims->block_q), nKB = ceil_div(dims->N, dims->block_k);
  if (list && (!list->cnt || !list->idx || !list->flag || list->max_k < 1)) return BSA_ERR_INVALID_ARG;
  AttnParams& ap = *out;
  std::memset(&ap, 0, sizeof(ap));
  if (gna) {
    int st = make_gna(gna, dims->n_text, &ap.g);
    if (st != BSA_OK) return st;
    if (tiled_len(ap.g) != dims->N || dims->block_q != ap.g.vol || dims->block_k != ap.g.vol)
      return BSA_ERR_INVALID_ARG;
    const int tx = ap.g.tile[2];
    if (ap.g.vol % gna_vol_mult != 0 || !((tx <= 64 && 64 % tx == 0) || (tx > 64 && tx % 64 == 0)))
      return BSA_ERR_UNSUPPORTED;
    ap.has_gna = 1;
  }
  ap.B = dims->B;
  ap.H = dims->H;
  ap.N = dims->N;
  ap.block_q = dims->block_q;
  ap.block_k = dims->block_k;
  ap.n_text = dims->n_text;
  ap.nQB = nQB;
  ap.nKB = nKB;
  ap.nQT = ceil_div(dims->N, 128);
  ap.nSeg = ceil_div(dims->N, 64);
  if (list) {
    ap.cnt = list->cnt;
    ap.idx = list->idx;
    ap.flag = list->flag;
    ap.max_k = list->max_k;
  }
  ap.head_mode = head_mode;
  ap.cache_in = cache_in;
  ap.cache_out = cache_out;
  ap.bias = block_bias;
  ap.scale_log2 = scale * 1.4426950408889634f;
  ap.O = static_cast<__nv_bfloat16*>(O);
  ap.wait_limit_ns = g_wait_limit_ns.load();
  ap.withhold_tile = g_withheld_tile.load();
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_version(void) { return kVersion; }

const char* bsa_error_string(int status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case BSA_ERR_WORKSPACE: return "workspace missing or too small";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_DEVICE: return "device-side fault recorded";
    case BSA_ERR_INFEASIBLE: return "no plan meets the error budget";
    default: return "unknown status";
  }
}

int bsa_gna_tiled_len(int32_t n_text, const bsa_gna_geom* geom, int32_t* n_tiled) {
  if (!n_tiled) return BSA_ERR_INVALID_ARG;
  GnaDev g;
  const int st = make_gna(geom, n_text, &g);
  if (st != BSA_OK) return st;
  const long long n = tiled_len(g);
  if (n > (1ll << 31) - 1) return BSA_ERR_UNSUPPORTED;
  *n_tiled = (int32_t)n;
  return BSA_OK;
}

int bsa_build_mask(const bsa_dims* dims, const bsa_mask_spec* spec, const bsa_block_list* out, void* stream) {
  int st = check_dims(dims);
  if (st != BSA_OK) return st;
  if (!spec) return BSA_ERR_INVALID_ARG;
  const int nQB = ceil_div(dims->N, dims->block_q), nKB = ceil_div(dims->N, dims->block_k);
  if ((st = check_list(out, nKB)) != BSA_OK) return st;
  MaskParams p;
  std::memset(&p, 0, sizeof(p));
  p.kind = spec->kind;
  p.B = dims->B;
  p.H = dims->H;
  p.nQB = nQB;
  p.nKB = nKB;
  p.head_mode = spec->head_mode;
  p.window = spec->window;
  p.cnt = out->cnt;
  p.idx = out->idx;
  p.flag = out->flag;
  p.bitmap = out->bitmap;
  p.max_k = out->max_k;
  if (spec->kind == BSA_MASK_ARROW) {
    if (dims->block_q != dims->block_k) return BSA_ERR_UNSUPPORTED;
    p.ntb = ceil_div(dims->n_text, dims->block_k);
  } else if (spec->kind == BSA_MASK_GNA) {
    if ((st = make_gna(&spec->gna, dims->n_text, &p.g)) != BSA_OK) return st;
    if (dims->block_q != p.g.vol || dims->block_k != p.g.vol) return BSA_ERR_UNSUPPORTED;
    if (tiled_len(p.g) != dims->N) return BSA_ERR_INVALID_ARG;
    p.ntb = p.g.text_span / p.g.vol;
  } else {
    return BSA_ERR_INVALID_ARG;
  }
  return cuda_status(launch_build_mask(p, static_cast<cudaStream_t>(stream)));
}

size_t bsa_select_workspace_size(const bsa_dims* dims, const bsa_select_spec* spec) {
  if (check_dims(dims) != BSA_OK || !spec) return 0;
  if (spec->method != BSA_SELECT_POOLED_QK && spec->method != BSA_SELECT_FULL_SCORE) return 0;
  return select_layout(dims, spec).total;
}

// bsa_select_topk after its argument and workspace checks; also the body of
// bsa_select_topk_static. Runs the form that `workspace_bytes` holds.
static int select_topk_in(const bsa_dims* dims, const void* Q, const void* K, const bsa_select_spec* spec,
                          const float* block_bias, void* workspace, size_t workspace_bytes,
                          const bsa_block_list* out, void* stream);

int bsa_select_topk(const bsa_dims* dims, const void* Q, const void* K, const bsa_select_spec* spec,
                    const float* block_bias, void* workspace, size_t workspace_bytes, const bsa_block_list* out,
                    void* stream) {
  int st = check_select_args(dims, Q, K, spec, out);
  if (st != BSA_OK) return st;
  if (!workspace || workspace_bytes < select_layout(dims, spec).total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return BSA_ERR_WORKSPACE;
  return select_topk_in(dims, Q, K, spec, block_bias, workspace, workspace_bytes, out, stream);
}

static int select_topk_in(const bsa_dims* dims, const void* Q, const void* K, const bsa_select_spec* spec,
                          const float* block_bias, void* workspace, size_t workspace_bytes,
                          const bsa_block_list* out, void* stream) {
  int st = BSA_OK;
  const int nQB = ceil_div(dims->N, dims->block_q), nKB = ceil_div(dims->N, dims->block_k);
  const SelectLayout L = layout_for_bytes(dims, spec, workspace_bytes);
  if (L.total > workspace_bytes) return BSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  SelectParams sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.method = spec->method;
  sp.B = dims->B;
  sp.H = dims->H;
  sp.N = dims->N;
  sp.block_q = dims->block_q;
  sp.block_k = dims->block_k;
  sp.nQB = nQB;
  sp.nKB = nKB;
  sp.keep_text = spec->keep_text ? 1 : 0;
  sp.ntbq = ceil_div(dims->n_text, dims->block_q);
  sp.ntbk = ceil_div(dims->n_text, dims->block_k);
  sp.n_groups = spec->n_groups;
  for (int g = 0; g < spec->n_groups; ++g) sp.groups[g] = spec->groups[g];
  sp.cnt = out->cnt;
  sp.idx = out->idx;
  sp.flag = out->flag;
  sp.bitmap = out->bitmap;
  sp.max_k = out->max_k;

  if (spec->method == BSA_SELECT_POOLED_QK) {
    PoolParams pp;
    pp.B = dims->B;
    pp.H = dims->H;
    pp.N = dims->N;
    pp.block_q = dims->block_q;
    pp.block_k = dims->block_k;
    pp.nQB = nQB;
    pp.nKB = nKB;
    pp.Q = static_cast<const __nv_bfloat16*>(Q);
    pp.K = static_cast<const __nv_bfloat16*>(K);
    pp.qbar = reinterpret_cast<float*>(ws + L.qbar);
    pp.kbar = reinterpret_cast<float*>(ws + L.kbar);
    if ((st = cuda_status(launch_block_pool(dims->d, pp, s))) != BSA_OK) return st;
    sp.qbar = pp.qbar;
    sp.kbar = pp.kbar;
  } else {
    const long long BH = (long long)dims->B * dims->H;
    CUtensorMap mq, mk;
    if ((st = make_map(&mq, Q, BH, dims->N, dims->d)) != BSA_OK) return st;
    if ((st = make_map(&mk, K, BH, dims->N, dims->d)) != BSA_OK) return st;
    AttnParams ap;
    std::memset(&ap, 0, sizeof(ap));
    ap.B = dims->B;
    ap.H = dims->H;
    ap.N = dims->N;
    ap.block_q = dims->block_q;
    ap.block_k = dims->block_k;
    ap.n_text = dims->n_text;
    ap.nQB = nQB;
    ap.nKB = nKB;
    ap.nQT = ceil_div(dims->N, 128);
    ap.nSeg = ceil_div(dims->N, 64);
    ap.bias = block_bias;
    ap.scale_log2 = spec->scale * 1.4426950408889634f;
    ap.wait_limit_ns = g_wait_limit_ns.load();
    ap.withhold_tile = -1;
    ap.apool = reinterpret_cast<float*>(ws + L.apool);
    if (L.chunk > 0) {
      // one pass per chunk of query blocks; each query tile writes its partial row of A'
      const FullScoreGeom g = full_score_geom(dims);
      ap.tlse = reinterpret_cast<float*>(ws + L.tlse);
      for (long long u0 = 0; u0 < g.units; u0 += L.chunk) {
        const long long n = std::min(L.chunk, g.units - u0);
        ap.u0 = u0;
        if ((st = cuda_status(launch_score(dims->d, KIND_TLSE, mq, mk, ap, (int)(n * g.m), s))) != BSA_OK)
          return st;
      }
      sp.parts = g.m;
    } else {
      ap.lse = reinterpret_cast<float*>(ws + L.lse);
      const int grid = (int)(BH * ap.nQT);
      if ((st = cuda_status(launch_score(dims->d, KIND_LSE, mq, mk, ap, grid, s))) != BSA_OK) return st;
      if ((st = cuda_status(cudaMemsetAsync(ap.apool, 0, (size_t)BH * nQB * nKB * sizeof(float), s))) != BSA_OK)
        return st;
      if ((st = cuda_status(launch_score(dims->d, KIND_POOL, mq, mk, ap, grid, s))) != BSA_OK) return st;
      sp.parts = 1;
    }
    sp.apool = ap.apool;
    sp.nQT = ap.nQT;
  }
  return cuda_status(launch_select(dims->d, sp, s));
}

int bsa_forward(const bsa_dims* dims, const void* Q, const void* K, const void* V, const bsa_block_list* list,
                const int32_t* head_mode, const bsa_gna_geom* gna, const float* cache_in, float* cache_out,
                const float* block_bias, float scale, void* O, void* stream) {
  int st = check_dims(dims);
  if (st != BSA_OK) return st;
  if (!Q || !K || !V) return BSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return BSA_ERR_INVALID_ARG;
  if (dims->d != 64 && dims->d != 128) return BSA_ERR_UNSUPPORTED;
  if (dims->block_q % 64 != 0 || dims->block_k % 64 != 0) return BSA_ERR_UNSUPPORTED;
  AttnParams ap;
  if ((st = forward_params(dims, list, head_mode, gna, cache_in, cache_out, block_bias, scale, O, 64, &ap)) != BSA_OK)
    return st;
  const long long BH = (long long)dims->B * dims->H;
  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, Q, BH, dims->N, dims->d)) != BSA_OK) return st;
  if ((st = make_map(&mk, K, BH, dims->N, dims->d)) != BSA_OK) return st;
  if ((st = make_map(&mv, V, BH, dims->N, dims->d)) != BSA_OK) return st;
  if ((st = make_map(&mo, O, BH, dims->N, dims->d)) != BSA_OK) return st;
  const long long grid = BH * ceil_div(dims->N, 256);
  if (grid > 0x7fffffffll) return BSA_ERR_UNSUPPORTED;
  return cuda_status(launch_forward(dims->d, mq, mk, mv, mo, ap, (int)grid, static_cast<cudaStream_t>(stream)));
}

int bsa_quantize_fp8(const bsa_dims* dims, const void* Q, const void* K, const void* V, uint8_t* q8, uint8_t* k8,
                     uint8_t* v8t, float* sq, float* sk, float* sv, void* stream) {
  int st = check_dims(dims);
  if (st != BSA_OK) return st;
  const void* ptrs[6] = {Q, K, V, q8, k8, v8t};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return BSA_ERR_INVALID_ARG;
  if (!sq || !sk || !sv) return BSA_ERR_INVALID_ARG;
  if (dims->d != 128) return BSA_ERR_UNSUPPORTED;
  QuantParams p;
  p.q = static_cast<const __nv_bfloat16*>(Q);
  p.k = static_cast<const __nv_bfloat16*>(K);
  p.v = static_cast<const __nv_bfloat16*>(V);
  p.q8 = q8;
  p.k8 = k8;
  p.v8t = v8t;
  p.sq = sq;
  p.sk = sk;
  p.sv = sv;
  p.BH = (long long)dims->B * dims->H;
  p.N = dims->N;
  p.Nt = round16(dims->N);
  p.nS = ceil_div(dims->N, 64);
  if (p.BH > 65535) return BSA_ERR_UNSUPPORTED;  // grid y
  return cuda_status(launch_quant_fp8(p, static_cast<cudaStream_t>(stream)));
}

int bsa_forward_fp8(const bsa_dims* dims, const uint8_t* q8, const uint8_t* k8, const uint8_t* v8t, const float* sq,
                    const float* sk, const float* sv, const bsa_block_list* list, const int32_t* head_mode,
                    const bsa_gna_geom* gna, const float* cache_in, float* cache_out, const float* block_bias,
                    float scale, void* O, void* stream) {
  int st = check_dims(dims);
  if (st != BSA_OK) return st;
  if (!q8 || !k8 || !v8t || !sq || !sk || !sv) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t)) return BSA_ERR_INVALID_ARG;
  if (dims->d != 128) return BSA_ERR_UNSUPPORTED;
  // every 128-key tile must be one aligned run of keys (the transposed V tile is one box)
  if (dims->block_q % 64 != 0 || dims->block_k % 128 != 0) return BSA_ERR_UNSUPPORTED;
  AttnParams ap;
  if ((st = forward_params(dims, list, head_mode, gna, cache_in, cache_out, block_bias, scale, O, 128, &ap)) !=
      BSA_OK)
    return st;
  ap.sq = sq;
  ap.sk = sk;
  ap.sv = sv;
  const long long BH = (long long)dims->B * dims->H;
  CUtensorMap mq, mk, mvt, mo;
  if ((st = make_map8(&mq, q8, BH, dims->N, 128)) != BSA_OK) return st;
  if ((st = make_map8(&mk, k8, BH, dims->N, 128)) != BSA_OK) return st;
  if ((st = make_map8(&mvt, v8t, BH, 128, round16(dims->N))) != BSA_OK) return st;
  if ((st = make_map(&mo, O, BH, dims->N, 128)) != BSA_OK) return st;
  const long long grid = BH * ceil_div(dims->N, 256);
  if (grid > 0x7fffffffll) return BSA_ERR_UNSUPPORTED;
  return cuda_status(launch_forward_fp8(mq, mk, mvt, mo, ap, (int)grid, static_cast<cudaStream_t>(stream)));
}

static int permute_common(bool forward, const bsa_dims* dims, const bsa_gna_geom* geom, int32_t n_tensors,
                          const void* const* in, void* const* out, void* stream) {
  if (!dims || dims->B < 1 || dims->H < 1 || dims->d < 8 || dims->n_text < 0) return BSA_ERR_INVALID_ARG;
  if (dims->d % 8 != 0) return BSA_ERR_UNSUPPORTED;
  if (n_tensors < 1 || n_tensors > 4 || !in || !out) return BSA_ERR_INVALID_ARG;
  PermuteParams p;
  std::memset(&p, 0, sizeof(p));
  int st = make_gna(geom, dims->n_text, &p.g);
  if (st != BSA_OK) return st;
  const long long nr = (long long)dims->n_text + (long long)p.g.grid[0] * p.g.grid[1] * p.g.grid[2];
  const long long nt = tiled_len(p.g);
  if (nr > 0x7fffffffll || nt > 0x7fffffffll) return BSA_ERR_UNSUPPORTED;
  p.n_tensors = n_tensors;
  p.BH = (long long)dims->B * dims->H;
  p.d = dims->d;
  p.n_raster = (int)nr;
  p.n_tiled = (int)nt;
  for (int t = 0; t < n_tensors; ++t) {
    if (!in[t] || !out[t] || !aligned16(in[t]) || !aligned16(out[t])) return BSA_ERR_INVALID_ARG;
    p.in[t] = static_cast<const __nv_bfloat16*>(in[t]);
    p.out[t] = static_cast<__nv_bfloat16*>(out[t]);
  }
  return cuda_status(launch_permute(forward, p, num_sms(), static_cast<cudaStream_t>(stream)));
}

int bsa_permute_tiles(const bsa_dims* dims, const bsa_gna_geom* geom, int32_t n_tensors, const void* const* in,
                      void* const* out, void* stream) {
  return permute_common(true, dims, geom, n_tensors, in, out, stream);
}

int bsa_unpermute_tiles(const bsa_dims* dims, const bsa_gna_geom* geom, int32_t n_tensors, const void* const* in,
                        void* const* out, void* stream) {
  return permute_common(false, dims, geom, n_tensors, in, out, stream);
}

int bsa_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? kWaitLimitNs : ns);
  return BSA_OK;
}

int bsa_set_withheld_tile(int32_t tile) {
  if (tile < -1) return BSA_ERR_INVALID_ARG;
  g_withheld_tile.store(tile);
  return BSA_OK;
}

int bsa_get_device_error(void* stream, int32_t* code) {
  if (!code) return BSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  *code = v;
  return BSA_OK;
}

}  // extern "C"
