// decode_noalloc.cu -- sparse decode for callers that cannot allocate device
// memory.
//
// bsa_sparse_attn_decode needs a scratch buffer for its split partials, and
// the caller normally hands one in.  Some callers have no way to get one: an
// inference server that reserves all of its device memory at start-up and
// forbids any allocation afterwards, or a plugin running inside a host
// framework that owns every device buffer and offers no workspace.  Asking
// them to cudaMalloc is not an option (it may synchronise the device and it
// breaks their memory budget).  This entry point runs the same decode with
// the scratch taken from a fixed array compiled into the library instead.
//
// The array is kNoAllocScratchBytes per GPU, lives in every GPU that loads
// the library until the process exits, and is shared by every call on that
// GPU: calls whose work overlaps on the GPU (different streams, no ordering
// between them) race on it.  Nothing in it has to start at zero -- every
// split writes its whole partial record before the combine step reads it --
// so the contents left by the previous call do no harm.
#include <mutex>

#include "../../include/bsa.h"
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per GPU
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
uint64_t g_noalloc_ctx[kMaxDevices] = {};

// Device address of the array on the current device.  In host code the
// array's name only stands in for the symbol; the address a kernel can use
// must be asked for once per device, with that device current.  The address
// is looked up again when the device's context has changed (a device reset
// reloads the library's module, and the array with it).
bsa_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  const uint64_t ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status_t bsa_sparse_attn_decode_noalloc(const bsa_shape_t* shape, const void* q,
                                                       const void* k_cache, const void* v_cache,
                                                       const int* idx, int idx_stride, float softmax_scale,
                                                       void* o, float* lse, void* stream) {
  if (shape == nullptr || idx_stride < 1) return BSA_ERR_INVALID_ARG;
  const size_t need = bsa_workspace_bytes(BSA_OP_DECODE, shape, idx_stride);
  if (need == 0) return BSA_ERR_INVALID_ARG;
  if (need > bsa::kNoAllocScratchBytes) return BSA_ERR_UNSUPPORTED;   // scratch too small for this shape
  void* scratch = nullptr;
  const bsa_status_t st = bsa::scratch_address(&scratch);
  if (st != BSA_OK) return st;
  return bsa_sparse_attn_decode(shape, q, k_cache, v_cache, idx, idx_stride, softmax_scale, scratch,
                                bsa::kNoAllocScratchBytes, o, lse, stream);
}
