// bsa_select_topk_static: bsa_select_topk with its scratch in a fixed array
// that lives inside the library, for callers that cannot allocate device
// memory (see include/bsa.h).
#include <mutex>

namespace bsa {
namespace {

// Scratch shared by every bsa_select_topk_static call on a device. Held by
// each GPU that loads the library until the process exits.
static __device__ __align__(256) uint8_t g_select_scratch[BSA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device. The name of the
// array is only a host-side stand-in; the address comes from the runtime, once
// per device, with that device current.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" int bsa_select_topk_static(const bsa_dims* dims, const void* Q, const void* K,
                                      const bsa_select_spec* spec, const float* block_bias,
                                      const bsa_block_list* out, void* stream) {
  // The same argument checks as bsa_select_topk come first, so an invalid or
  // unsupported request is reported as such even when it is also too large
  // for the scratch.
  const int arg = bsa::check_select_args(dims, Q, K, spec, out);
  if (arg != BSA_OK) return arg;
  // the form the scratch holds: for FULL_SCORE the one-pass form if its
  // slabs fit, else the two-pass form
  if (bsa::layout_for_bytes(dims, spec, BSA_STATIC_SCRATCH_BYTES).total > (size_t)BSA_STATIC_SCRATCH_BYTES)
    return BSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = bsa::scratch_for_current_device(&scratch);
  if (st != BSA_OK) return st;
  return select_topk_in(dims, Q, K, spec, block_bias, scratch, (size_t)BSA_STATIC_SCRATCH_BYTES, out, stream);
}
