// Step schedule of the sparse path: which denoising step runs full attention,
// selects the head-specific pattern or reuses it (SparseD, "overall
// framework"), the kept percentage per layer and step (lmnt.cn BSA post,
// section 3.3), both host only; and the Jaccard similarity of two selections
// (SparseD, "sparse reuse"), on the GPU.
#include "common.cuh"

namespace bsa {

struct JaccardParams {
  const int32_t *cnt_a, *idx_a, *cnt_b, *idx_b;
  int max_k_a, max_k_b;
  long long rows;
  float* out;
};

// One thread per query-block row: both lists are ascending, so one merge
// counts the intersection; |A u B| = |A| + |B| - |A n B|.
__global__ void __launch_bounds__(256) jaccard_kernel(JaccardParams p) {
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= p.rows) return;
  int na = p.cnt_a[r], nb = p.cnt_b[r];
  if (na < 0 || na > p.max_k_a || nb < 0 || nb > p.max_k_b) {
    record_error(BSA_DEVERR_BAD_INDEX);
    na = na < 0 ? 0 : (na > p.max_k_a ? p.max_k_a : na);
    nb = nb < 0 ? 0 : (nb > p.max_k_b ? p.max_k_b : nb);
  }
  const int32_t* a = p.idx_a + r * p.max_k_a;
  const int32_t* b = p.idx_b + r * p.max_k_b;
  int i = 0, j = 0, both = 0;
  while (i < na && j < nb) {
    const int x = a[i], y = b[j];
    both += x == y;
    i += x <= y;
    j += y <= x;
  }
  const int uni = na + nb - both;
  p.out[r] = uni == 0 ? 1.f : (float)both / (float)uni;
}

}  // namespace bsa

using namespace bsa;

extern "C" int bsa_schedule_full_steps(int32_t n_steps, int32_t skip_pct, int32_t* n_full) {
  if (!n_full || n_steps < 1 || skip_pct < 0 || skip_pct > 100) return BSA_ERR_INVALID_ARG;
  *n_full = (int32_t)(((long long)n_steps * skip_pct + 99) / 100);
  return BSA_OK;
}

extern "C" int bsa_step_action(int32_t step, int32_t n_steps, int32_t n_full, int32_t* action) {
  if (!action || n_steps < 1 || step < 0 || step >= n_steps || n_full < 0 || n_full > n_steps)
    return BSA_ERR_INVALID_ARG;
  *action = step < n_full ? BSA_STEP_FULL : (step == n_full ? BSA_STEP_SELECT : BSA_STEP_REUSE);
  return BSA_OK;
}

// hi - (hi - lo) * (l / (L - 1) + s / (T - 1)) / 2 over the common
// denominator 2 (L - 1) (T - 1), rounded to the nearest integer, halves up.
extern "C" int bsa_keep_pct(int32_t layer, int32_t n_layers, int32_t step, int32_t n_steps, int32_t hi, int32_t lo,
                            int32_t* pct) {
  if (!pct || n_layers < 1 || n_steps < 1 || layer < 0 || layer >= n_layers || step < 0 || step >= n_steps ||
      hi < 0 || hi > 100 || lo < 0 || lo > 100)
    return BSA_ERR_INVALID_ARG;
  const long long a = n_layers > 1 ? n_layers - 1 : 1, la = n_layers > 1 ? layer : 0;
  const long long b = n_steps > 1 ? n_steps - 1 : 1, sb = n_steps > 1 ? step : 0;
  const long long den = 2 * a * b;
  const long long num = (long long)hi * den - (long long)(hi - lo) * (la * b + sb * a);  // >= 0
  *pct = (int32_t)((2 * num + den) / (2 * den));
  return BSA_OK;
}

extern "C" int bsa_jaccard(const bsa_dims* dims, const bsa_block_list* a, const bsa_block_list* b, float* out,
                           void* stream) {
  if (check_dims(dims) != BSA_OK || !a || !b || !out) return BSA_ERR_INVALID_ARG;
  if (!a->cnt || !a->idx || !b->cnt || !b->idx || a->max_k < 1 || b->max_k < 1) return BSA_ERR_INVALID_ARG;
  JaccardParams p;
  p.cnt_a = a->cnt;
  p.idx_a = a->idx;
  p.cnt_b = b->cnt;
  p.idx_b = b->idx;
  p.max_k_a = a->max_k;
  p.max_k_b = b->max_k;
  p.rows = (long long)dims->B * dims->H * ((dims->N + dims->block_q - 1) / dims->block_q);
  p.out = out;
  const long long grid = (p.rows + 255) / 256;
  if (grid > 0x7fffffffll) return BSA_ERR_UNSUPPORTED;
  jaccard_kernel<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cuda_status(cudaGetLastError());
}
