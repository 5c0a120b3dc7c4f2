// api.cu -- the C ABI of libbsa (see include/bsa.h): argument checks, TMA
// tensor maps, workspace layout and kernel dispatch.  No call here allocates
// or frees device memory; scratch comes from the caller.
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/bsa.h"
#include "common.cuh"
#include "kernels.h"

namespace bsa {

// Device status word: kernels OR flags into it instead of trapping.
__device__ uint32_t g_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_status_ptr[kMaxDevices] = {};
uint64_t g_status_ctx[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Split-count override of the decode plan (0: one split range per SM); set
// only through bsa_decode_split_override().
std::atomic<int> g_split_override{0};
// Prefill kernel override (0: chosen by shape); set only through
// bsa_prefill_kernel_override().
std::atomic<int> g_prefill_kernel{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
std::atomic<CtxGetCurrentFn> g_ctx_current{nullptr};
std::atomic<CtxGetIdFn> g_ctx_id{nullptr};

template <typename Fn>
Fn driver_entry(const char* name) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(fn);
}

bsa_status_t device_state(uint32_t** status, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  const uint64_t ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_status_ptr[dev] == nullptr || ctx == 0 || g_status_ctx[dev] != ctx) {
    // first use on this device, or a new context since (a device reset
    // reloads the module, so the status word has a new address); the
    // runtime calls below make the device's primary context current
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return BSA_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BSA_ERR_CUDA;
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
    g_status_ctx[dev] = current_context_id();
    g_num_sms[dev] = sms;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return BSA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (status) *status = g_status_ptr[dev];
  if (num_sms) *num_sms = g_num_sms[dev];
  return BSA_OK;
}

// 2-D bf16 view [rows, 128] with a box of 64 columns x box_rows rows and the
// 128-byte swizzle the MMA descriptors expect.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 view [rows, 128] with a box of 32 columns (128 bytes) x 128 rows
// and the 128-byte swizzle (the decode selector's pooled-key chunks).
bool make_map_f32_rows128(CUtensorMap* m, const void* base, uint64_t rows) {
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128 * 4};
  const cuuint32_t box[2] = {32, 128};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsa_status_t check_shape(const bsa_shape_t* s) {
  if (s == nullptr) return BSA_ERR_INVALID_ARG;
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->Nq <= 0 || s->Nk <= 0 || s->d <= 0 || s->block <= 0)
    return BSA_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0 || s->Nk % s->block != 0) return BSA_ERR_INVALID_ARG;
  if (s->dtype != BSA_F32 && s->dtype != BSA_BF16) return BSA_ERR_INVALID_ARG;
  const int64_t rows_q = static_cast<int64_t>(s->B) * s->Hq * s->Nq;
  const int64_t rows_k = static_cast<int64_t>(s->B) * s->Hkv * s->Nk;
  if (rows_q >= (1ll << 31) || rows_k >= (1ll << 31)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

bsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

float score_scale(int d) { return static_cast<float>(1.0 / sqrt(static_cast<double>(d))); }

// Split-K plan of the decode kernels: the group rows' list positions are laid
// end to end and cut into num_ctas equal ranges (one persistent CTA per SM by
// default); no range may exceed the kernel's 128-tile item capacity.
struct DecodePlan {
  int num_ctas, max_slots, list_len;
};

DecodePlan decode_plan(int rows, int list_len, int num_sms) {
  DecodePlan P;
  P.list_len = list_len;
  const int64_t total = static_cast<int64_t>(rows) * list_len;
  int64_t c = num_sms;
  const int forced = g_split_override.load(std::memory_order_relaxed);
  if (forced > 0) c = forced;
  const int64_t need = (total + 127) / 128;   // ceil(total / c) <= 128
  if (c < need) c = need;
  if (c > total) c = total > 0 ? total : 1;
  P.num_ctas = static_cast<int>(c);
  P.max_slots = decode_slots_for(rows, list_len, P.num_ctas);
  return P;
}

struct GistLayout {
  size_t scores, idx, expanded, union_list, partial, total;
  int union_stride;
  DecodePlan plan;
};

GistLayout gist_layout(const bsa_shape_t* s, int topk, int num_sms) {
  GistLayout L{};
  const int nc = s->Nk / s->block;
  const int G = s->Hq / s->Hkv;
  const int64_t rows = static_cast<int64_t>(s->B) * s->Hq;
  L.union_stride = 1 + G * topk + nc / 64;
  L.plan = decode_plan(s->B * s->Hkv, L.union_stride - 1, num_sms);
  size_t off = 0;
  L.scores = off;
  off = align256(off + rows * nc * sizeof(float));
  L.idx = off;
  off = align256(off + rows * (topk > 0 ? topk : 1) * sizeof(int));
  L.expanded = off;
  off = align256(off + rows * (nc / 32) * sizeof(uint32_t));
  L.union_list = off;
  off = align256(off + static_cast<size_t>(s->B) * s->Hkv * L.union_stride * sizeof(int));
  L.partial = off;
  off = align256(off + rows * L.plan.max_slots * (s->d + 4) * sizeof(float));
  L.total = off;
  return L;
}

// Workspace of the per-head decode: each head's kept-block bitmap, the
// group's union list (count first), the split partials.
struct HeadsLayout {
  size_t expanded, union_list, partial, total;
  int union_stride;
  DecodePlan plan;
};

HeadsLayout heads_layout(const bsa_shape_t* s, int idx_stride, int num_sms) {
  HeadsLayout L{};
  const int nb = s->Nk / s->block;
  const int G = s->Hq / s->Hkv;
  const int64_t rows = static_cast<int64_t>(s->B) * s->Hq;
  L.union_stride = 1 + std::min(nb, G * idx_stride);
  L.plan = decode_plan(s->B * s->Hkv, L.union_stride - 1, num_sms);
  size_t off = 0;
  L.expanded = off;
  off = align256(off + rows * (nb / 32) * sizeof(uint32_t));
  L.union_list = off;
  off = align256(off + static_cast<size_t>(s->B) * s->Hkv * L.union_stride * sizeof(int));
  L.partial = off;
  off = align256(off + rows * L.plan.max_slots * (s->d + 4) * sizeof(float));
  L.total = off;
  return L;
}

// Workspace of the two-level gist decode.
struct HssaLayout {
  size_t meta_scores, meta_idx, fine, pos, chunks, expanded, allow, union_list, partial, total;
  int union_stride, k_stride;
  DecodePlan plan;
};

HssaLayout hssa_layout(const bsa_shape_t* s, int km, int topk, int num_sms) {
  HssaLayout L{};
  const int nc = s->Nk / s->block, nm = nc / 64;
  const int G = s->Hq / s->Hkv;
  const int64_t rows = static_cast<int64_t>(s->B) * s->Hq;
  L.k_stride = topk > 0 ? topk : 1;
  L.union_stride = 1 + std::min(nc, G * topk) + nm + 1;
  L.plan = decode_plan(s->B * s->Hkv, L.union_stride - 1, num_sms);
  size_t off = 0;
  L.meta_scores = off;
  off = align256(off + rows * nm * sizeof(float));
  L.meta_idx = off;
  off = align256(off + rows * km * sizeof(int));
  L.fine = off;
  off = align256(off + rows * km * 64 * sizeof(float));
  L.pos = off;
  off = align256(off + rows * L.k_stride * sizeof(int));
  L.chunks = off;
  off = align256(off + rows * L.k_stride * sizeof(int));
  L.expanded = off;
  off = align256(off + rows * (nc / 32) * sizeof(uint32_t));
  L.allow = off;
  off = align256(off + rows * ((nc + 64) / 32) * sizeof(uint32_t));
  L.union_list = off;
  off = align256(off + static_cast<size_t>(s->B) * s->Hkv * L.union_stride * sizeof(int));
  L.partial = off;
  off = align256(off + rows * L.plan.max_slots * (s->d + 4) * sizeof(float));
  L.total = off;
  return L;
}

// Self-test of the bounded-wait expiry path: one thread waits, with a small
// budget, on a shared-memory barrier that nothing arrives on.  The wait gives
// up, raises BSA_DEV_TIMEOUT in the status word and the kernel returns.
__global__ void wait_expiry_selftest_kernel(long long budget, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait(b, 0, &abort_flag, status, budget);   // phase 0 never completes
}

}  // namespace

uint64_t current_context_id() {
  CtxGetCurrentFn cur = g_ctx_current.load(std::memory_order_acquire);
  CtxGetIdFn id = g_ctx_id.load(std::memory_order_acquire);
  if (cur == nullptr || id == nullptr) {
    cur = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
    id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    if (cur == nullptr || id == nullptr) return 0;
    g_ctx_current.store(cur, std::memory_order_release);
    g_ctx_id.store(id, std::memory_order_release);
  }
  CUcontext ctx = nullptr;
  unsigned long long v = 0;
  if (cur(&ctx) != CUDA_SUCCESS || ctx == nullptr || id(ctx, &v) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(v);
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_version(void) { return 100; }

const char* bsa_status_string(bsa_status_t st) {
  switch (st) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_DEVICE: return "BSA_ERR_DEVICE";
  }
  return "BSA_ERR_UNKNOWN";
}

int bsa_prefill_kernel_override(int kernel) {
  return g_prefill_kernel.exchange(kernel >= 1 && kernel <= 3 ? kernel : 0);
}

int bsa_decode_split_override(int num_splits) {
  return g_split_override.exchange(num_splits > 0 ? num_splits : 0);
}

bsa_status_t bsa_selftest_wait_expiry(long long budget_cycles, void* stream) {
  if (budget_cycles < 0) return BSA_ERR_INVALID_ARG;
  uint32_t* status = nullptr;
  bsa_status_t st = device_state(&status, nullptr);
  if (st != BSA_OK) return st;
  wait_expiry_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_cycles, status);
  return cuda_status(cudaGetLastError());
}

bsa_status_t bsa_device_status(unsigned int* flags, int reset) {
  uint32_t* dev_ptr = nullptr;
  bsa_status_t st = device_state(&dev_ptr, nullptr);
  if (st != BSA_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return BSA_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, dev_ptr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BSA_ERR_CUDA;
  if (reset) {
    const uint32_t zero = 0;
    if (cudaMemcpy(dev_ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return BSA_ERR_CUDA;
  }
  if (flags) *flags = v;
  if (v & BSA_DEV_TIMEOUT) return BSA_ERR_TIMEOUT;
  if (v) return BSA_ERR_DEVICE;
  return BSA_OK;
}

size_t bsa_workspace_bytes(int op, const bsa_shape_t* s, int budget) {
  if (check_shape(s) != BSA_OK || budget < 0) return 0;
  int sms = 0;
  if (device_state(nullptr, &sms) != BSA_OK) return 0;
  if (op == BSA_OP_DECODE) {
    if (budget < 1) return 0;
    const DecodePlan P = decode_plan(s->B * s->Hkv, budget, sms);
    return align256(static_cast<size_t>(s->B) * s->Hq * P.max_slots * (s->d + 4) * sizeof(float));
  }
  if (op == BSA_OP_GIST_DECODE) return gist_layout(s, budget, sms).total;
  if (op == BSA_OP_DECODE_HEADS) {
    if (budget < 1) return 0;
    return heads_layout(s, budget, sms).total;
  }
  return 0;
}

size_t bsa_workspace_bytes_hssa(const bsa_shape_t* s, int km, int topk) {
  if (check_shape(s) != BSA_OK || km < 1 || topk < 0) return 0;
  int sms = 0;
  if (device_state(nullptr, &sms) != BSA_OK) return 0;
  return hssa_layout(s, km, topk, sms).total;
}

bsa_status_t bsa_score_blocks(const bsa_shape_t* s, int mode, const void* q, const void* k,
                              const float* pooled_k_in, float* pooled_q_out, float* pooled_k_out, float* scores,
                              void* stream) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (q == nullptr || scores == nullptr || !aligned16(q) || !aligned16(scores)) return BSA_ERR_INVALID_ARG;
  if (s->d % 8 != 0 || s->d > 1024) return BSA_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool bf16 = s->dtype == BSA_BF16;
  const int nb = s->Nk / s->block;
  const int G = s->Hq / s->Hkv;
  if ((st = device_state(nullptr, nullptr)) != BSA_OK) return st;
  const float scale = score_scale(s->d);
  if (mode == BSA_SCORE_PREFILL) {
    if (s->Nq != s->Nk || k == nullptr || pooled_q_out == nullptr || pooled_k_out == nullptr ||
        pooled_k_in != nullptr)
      return BSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(pooled_q_out) || !aligned16(pooled_k_out)) return BSA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(nb) * nb >= (1ll << 31)) return BSA_ERR_UNSUPPORTED;
    uint32_t* status = nullptr;
    int sms = 0;
    if ((st = device_state(&status, &sms)) != BSA_OK) return st;
    cudaError_t e = launch_pool_prefill(q, k, bf16, s->B, s->Hq, s->Hkv, s->Nk, s->d, s->block, pooled_q_out,
                                        pooled_k_out, sms, status, cs);
    if (e == cudaSuccess) e = launch_score_prefill(pooled_q_out, pooled_k_out, s->B, s->Hkv, nb, s->d, scale, scores, cs);
    return cuda_status(e);
  }
  if (mode == BSA_SCORE_DECODE) {
    if (s->Nq != 1) return BSA_ERR_INVALID_ARG;
    const float* kbar = pooled_k_in;
    cudaError_t e = cudaSuccess;
    if (kbar == nullptr) {
      if (k == nullptr || pooled_k_out == nullptr || !aligned16(k) || !aligned16(pooled_k_out))
        return BSA_ERR_INVALID_ARG;
      e = launch_pool(k, bf16, s->B, s->Hkv, s->Hkv, 1, s->Nk, s->d, s->block, pooled_k_out, cs);
      kbar = pooled_k_out;
    } else if (!aligned16(kbar)) {
      return BSA_ERR_INVALID_ARG;
    }
    if (e == cudaSuccess)
      e = launch_score_decode(q, bf16, kbar, s->B, s->Hq, s->Hkv, nb, s->d, scale, scores, pooled_q_out, cs);
    return cuda_status(e);
  }
  if (mode == BSA_SCORE_DECODE_HEADS) {
    if (s->Nq != 1 || pooled_k_in == nullptr || !aligned16(pooled_k_in) || k || pooled_q_out || pooled_k_out)
      return BSA_ERR_INVALID_ARG;
    if (s->d != 64 && s->d != 128) return BSA_ERR_UNSUPPORTED;
    if (G > 16) return BSA_ERR_UNSUPPORTED;
    return cuda_status(launch_score_heads(q, bf16, pooled_k_in, s->B, s->Hq, s->Hkv, nb, s->d, scale, scores, cs));
  }
  if (mode == BSA_SCORE_GIST) {
    if (s->Nq != 1 || k == nullptr || !aligned16(k) || pooled_k_in || pooled_q_out || pooled_k_out)
      return BSA_ERR_INVALID_ARG;
    if (G > 16) return BSA_ERR_UNSUPPORTED;
    uint32_t* status = nullptr;
    int sms = 0;
    if ((st = device_state(&status, &sms)) != BSA_OK) return st;
    CUtensorMap mg;
    const bool tma = bf16 && s->d == 128;
    if (tma && !make_map_bf16(&mg, k, static_cast<uint64_t>(s->B) * s->Hkv * nb, 64)) return BSA_ERR_CUDA;
    return cuda_status(launch_score_gist(tma ? &mg : nullptr, q, k, bf16, s->B, s->Hq, s->Hkv, nb, s->d, scale,
                                         scores, status, sms, cs));
  }
  return BSA_ERR_INVALID_ARG;
}

bsa_status_t bsa_topk_select(const float* scores, int rows, int ncols, int mode, int kb, int* idx_out,
                             int idx_stride, int* count_out, void* stream) {
  if (scores == nullptr || idx_out == nullptr || rows < 0 || ncols < 1 || kb < 0) return BSA_ERR_INVALID_ARG;
  if (mode != BSA_TOPK_CAUSAL_BLOCK && mode != BSA_TOPK_LAST_BLOCK && mode != BSA_TOPK_PLAIN)
    return BSA_ERR_INVALID_ARG;
  const int forced = (mode == BSA_TOPK_PLAIN) ? 0 : 1;
  if (idx_stride < kb + forced || idx_stride < 1) return BSA_ERR_INVALID_ARG;
  if (ncols > 8192) return BSA_ERR_UNSUPPORTED;
  if (rows == 0) return BSA_OK;
  bsa_status_t st = device_state(nullptr, nullptr);
  if (st != BSA_OK) return st;
  return cuda_status(launch_topk(scores, rows, ncols, mode, kb, idx_out, idx_stride, count_out,
                                 static_cast<cudaStream_t>(stream)));
}

bsa_status_t bsa_decode_select(const bsa_shape_t* s, const void* q, const float* pooled_k, int kb,
                               float* pooled_q_out, float* scores, int* idx_out, int idx_stride, int* count_out,
                               void* stream) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (s->Nq != 1 || !q || !pooled_k || !scores || !idx_out || kb < 0) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pooled_k) || !aligned16(scores)) return BSA_ERR_INVALID_ARG;
  if (idx_stride < kb + 1) return BSA_ERR_INVALID_ARG;
  if (s->d % 8 != 0 || s->d > 1024) return BSA_ERR_UNSUPPORTED;
  const int nb = s->Nk / s->block;
  if (nb > 8192) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  if ((st = device_state(&status, nullptr)) != BSA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool bf16 = s->dtype == BSA_BF16;
  const float scale = score_scale(s->d);
  if (decode_select_fused_ok(s->d, nb)) {
    CUtensorMap mk;
    if (!make_map_f32_rows128(&mk, pooled_k, static_cast<uint64_t>(s->B) * s->Hkv * nb)) return BSA_ERR_CUDA;
    return cuda_status(launch_decode_select(&mk, q, bf16, s->B, s->Hq, s->Hkv, nb, scale, kb, scores, pooled_q_out,
                                            idx_out, idx_stride, count_out, status, cs));
  }
  // other head dimensions or longer rows: the scoring and selection kernels
  cudaError_t e =
      launch_score_decode(q, bf16, pooled_k, s->B, s->Hq, s->Hkv, nb, s->d, scale, scores, pooled_q_out, cs);
  if (e == cudaSuccess)
    e = launch_topk(scores, s->B * s->Hkv, nb, BSA_TOPK_LAST_BLOCK, kb, idx_out, idx_stride, count_out, cs);
  return cuda_status(e);
}

bsa_status_t bsa_topk_select_pattern(const float* scores, int rows, int ncols, int sink, int local, int kb,
                                     int* idx_out, int idx_stride, int* count_out, void* stream) {
  if (scores == nullptr || idx_out == nullptr || rows < 0 || ncols < 1 || kb < 0 || sink < 0 || local < 1)
    return BSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(idx_stride) < static_cast<int64_t>(sink) + local + kb) return BSA_ERR_INVALID_ARG;
  if (ncols > 8192) return BSA_ERR_UNSUPPORTED;
  if (rows == 0) return BSA_OK;
  bsa_status_t st = device_state(nullptr, nullptr);
  if (st != BSA_OK) return st;
  return cuda_status(launch_topk_pattern(scores, rows, ncols, sink, local, kb, idx_out, idx_stride, count_out,
                                         static_cast<cudaStream_t>(stream)));
}

bsa_status_t bsa_topk_select_joint_heads(const float* scores, int rows, int heads, int ncols, int kb_total,
                                         int* idx_out, int idx_stride, int* count_out, void* stream) {
  if (scores == nullptr || idx_out == nullptr || rows < 0 || heads < 1 || ncols < 1 || kb_total < 0)
    return BSA_ERR_INVALID_ARG;
  if (idx_stride < std::min(kb_total, ncols - 1) + 1) return BSA_ERR_INVALID_ARG;
  if (heads > 16 || static_cast<int64_t>(heads) * (ncols - 1) > 8192) return BSA_ERR_UNSUPPORTED;
  if (rows == 0) return BSA_OK;
  bsa_status_t st = device_state(nullptr, nullptr);
  if (st != BSA_OK) return st;
  return cuda_status(launch_topk_joint(scores, rows, heads, ncols, kb_total, idx_out, idx_stride, count_out,
                                       static_cast<cudaStream_t>(stream)));
}

static bsa_status_t prefill_common(const bsa_shape_t* s, const void* q, const void* k, const void* v,
                                   const int* idx, int idx_stride, const float* sel, float scale, void* o,
                                   float* lse, void* stream) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (s->Nq != s->Nk) return BSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !idx || !o) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return BSA_ERR_INVALID_ARG;
  if (idx_stride < 1 || !(scale > 0.0f) || !isfinite(scale)) return BSA_ERR_INVALID_ARG;
  if (idx_stride > 256) return BSA_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  PrefillArgs a;
  a.num_sms = sms;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.N = s->Nk;
  a.bs = s->block;
  a.idx = idx;
  a.idx_stride = idx_stride;
  a.sel_scores = sel;
  a.softmax_scale = scale;
  a.o = o;
  a.lse = lse;
  a.status = status;
  a.kernel = g_prefill_kernel.load(std::memory_order_relaxed);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (s->dtype == BSA_BF16) {
    if (s->d != 128) return BSA_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mv;
    if (!make_map_bf16(&mq, q, static_cast<uint64_t>(s->B) * s->Hq * s->Nq, 64) ||
        !make_map_bf16(&mk, k, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64) ||
        !make_map_bf16(&mv, v, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64))
      return BSA_ERR_CUDA;
    return cuda_status(launch_attn_prefill_bf16(&mq, &mk, &mv, a, cs));
  }
  if (s->d != 64 && s->d != 128) return BSA_ERR_UNSUPPORTED;
  return cuda_status(launch_attn_prefill_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                             static_cast<const float*>(v), a, s->d, cs));
}

bsa_status_t bsa_sparse_attn_prefill(const bsa_shape_t* s, const void* q, const void* k, const void* v,
                                     const int* idx, int idx_stride, float softmax_scale, void* o, float* lse,
                                     void* stream) {
  return prefill_common(s, q, k, v, idx, idx_stride, nullptr, softmax_scale, o, lse, stream);
}

bsa_status_t bsa_gated_attn_fwd(const bsa_shape_t* s, const void* q, const void* k, const void* v,
                                const int* idx, int idx_stride, const float* sel_scores, float softmax_scale,
                                void* o, float* lse, void* stream) {
  if (sel_scores == nullptr) return BSA_ERR_INVALID_ARG;
  return prefill_common(s, q, k, v, idx, idx_stride, sel_scores, softmax_scale, o, lse, stream);
}

static bsa_status_t decode_checks(const bsa_shape_t* s, const void* q, const void* kc, const void* vc, void* o) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (s->Nq != 1 || !q || !kc || !vc || !o) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(o)) return BSA_ERR_INVALID_ARG;
  if (s->dtype != BSA_BF16 || s->d != 128 || s->block != 64) return BSA_ERR_UNSUPPORTED;
  if (s->Hq / s->Hkv > 16) return BSA_ERR_UNSUPPORTED;   // the MMA N tile holds a group of at most 16 heads
  return BSA_OK;
}

bsa_status_t bsa_sparse_attn_decode(const bsa_shape_t* s, const void* q, const void* k_cache, const void* v_cache,
                                    const int* idx, int idx_stride, float softmax_scale, void* workspace,
                                    size_t workspace_bytes, void* o, float* lse, void* stream) {
  bsa_status_t st = decode_checks(s, q, k_cache, v_cache, o);
  if (st != BSA_OK) return st;
  if (!idx || idx_stride < 1 || !(softmax_scale > 0.0f) || !workspace) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  const int G = s->Hq / s->Hkv;
  const DecodePlan P = decode_plan(s->B * s->Hkv, idx_stride, sms);
  const size_t need = align256(static_cast<size_t>(s->B) * s->Hq * P.max_slots * (s->d + 4) * sizeof(float));
  if (workspace_bytes < need) return BSA_ERR_INVALID_ARG;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, q, static_cast<uint64_t>(s->B) * s->Hq, static_cast<uint32_t>(G)) ||
      !make_map_bf16(&mk, k_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64) ||
      !make_map_bf16(&mv, v_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64))
    return BSA_ERR_CUDA;
  DecodeArgs a;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.Nk = s->Nk;
  a.bs = s->block;
  a.list = idx;
  a.list_stride = idx_stride;
  a.list_has_count = 0;
  a.expanded = nullptr;
  a.nc = 0;
  a.list_len = P.list_len;
  a.num_ctas = P.num_ctas;
  a.max_slots = P.max_slots;
  a.softmax_scale = softmax_scale;
  a.partial = static_cast<float*>(workspace);
  a.status = status;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_attn_decode_bf16(&mq, &mk, &mv, nullptr, nullptr, a, cs);
  if (e == cudaSuccess) e = launch_decode_combine(a.partial, a, s->d, true, o, lse, cs);
  return cuda_status(e);
}

bsa_status_t bsa_gist_expand_decode(const bsa_shape_t* s, const void* q, const void* k_cache, const void* v_cache,
                                    const void* gist_k, const void* gist_v, int topk, const int* idx_in,
                                    int* idx_out, float softmax_scale, void* workspace, size_t workspace_bytes,
                                    void* o, float* lse, void* stream) {
  bsa_status_t st = decode_checks(s, q, k_cache, v_cache, o);
  if (st != BSA_OK) return st;
  const int nc = s->Nk / s->block;
  if (!gist_k || !gist_v || !aligned16(gist_k) || !aligned16(gist_v)) return BSA_ERR_INVALID_ARG;
  if (topk < 0 || topk > nc || !(softmax_scale > 0.0f) || !workspace) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  if (nc % 64 != 0 || nc > 8192) return BSA_ERR_UNSUPPORTED;
  if (s->Hq / s->Hkv > 16) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  const GistLayout L = gist_layout(s, topk, sms);
  if (workspace_bytes < L.total) return BSA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int G = s->Hq / s->Hkv;
  const int rows = s->B * s->Hq;
  const int* idx = idx_in;
  const int idx_stride = topk > 0 ? topk : 1;
  cudaError_t e = cudaSuccess;
  uint32_t* expanded = reinterpret_cast<uint32_t*>(ws + L.expanded);
  int* ulist = reinterpret_cast<int*>(ws + L.union_list);
  // every tensor map first, so that nothing is enqueued when one fails
  CUtensorMap mq, mk, mv, mgk, mgv;
  if (!make_map_bf16(&mq, q, static_cast<uint64_t>(rows), static_cast<uint32_t>(G)) ||
      !make_map_bf16(&mk, k_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64) ||
      !make_map_bf16(&mv, v_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64) ||
      !make_map_bf16(&mgk, gist_k, static_cast<uint64_t>(s->B) * s->Hkv * nc, 64) ||
      !make_map_bf16(&mgv, gist_v, static_cast<uint64_t>(s->B) * s->Hkv * nc, 64))
    return BSA_ERR_CUDA;
  if (idx == nullptr) {
    int* idx_dst = (idx_out && topk > 0) ? idx_out : reinterpret_cast<int*>(ws + L.idx);
    if (topk > 0) {
      float* sc = reinterpret_cast<float*>(ws + L.scores);
      e = launch_score_gist(&mgk, q, gist_k, true, s->B, s->Hq, s->Hkv, nc, s->d, score_scale(s->d), sc, status,
                            sms, cs);
      if (e == cudaSuccess) e = launch_topk(sc, rows, nc, BSA_TOPK_PLAIN, topk, idx_dst, idx_stride, nullptr, cs);
    } else {
      e = cudaMemsetAsync(idx_dst, 0xff, static_cast<size_t>(rows) * sizeof(int), cs);
    }
    idx = idx_dst;
  } else if (idx_out != nullptr && topk > 0 && idx_out != idx_in) {
    e = cudaMemcpyAsync(idx_out, idx_in, static_cast<size_t>(rows) * topk * sizeof(int), cudaMemcpyDeviceToDevice, cs);
  }
  // up to 2048 chunks the attention kernel builds the group's union itself
  const bool fused_union = nc <= 2048;
  if (e == cudaSuccess && !fused_union)
    e = launch_gist_union(idx, s->B, s->Hq, s->Hkv, topk, idx_stride, nc, expanded, ulist, L.union_stride, true,
                          status, cs);
  DecodeArgs a;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.Nk = s->Nk;
  a.bs = s->block;
  a.list = ulist;
  a.list_stride = L.union_stride;
  a.list_has_count = 1;
  a.expanded = expanded;
  a.nc = nc;
  a.list_len = L.plan.list_len;
  a.num_ctas = L.plan.num_ctas;
  a.max_slots = L.plan.max_slots;
  a.softmax_scale = softmax_scale;
  a.partial = reinterpret_cast<float*>(ws + L.partial);
  a.status = status;
  if (fused_union) {
    a.list = nullptr;
    a.expanded = nullptr;
    a.heads_idx = idx;
    a.heads_topk = topk;
    a.heads_stride = idx_stride;
  }
  if (e == cudaSuccess) e = launch_attn_decode_bf16(&mq, &mk, &mv, &mgk, &mgv, a, cs);
  if (e == cudaSuccess) e = launch_decode_combine(a.partial, a, s->d, true, o, lse, cs);
  return cuda_status(e);
}

bsa_status_t bsa_sparse_attn_decode_heads(const bsa_shape_t* s, const void* q, const void* k_cache,
                                          const void* v_cache, const int* idx, int idx_stride, float softmax_scale,
                                          void* workspace, size_t workspace_bytes, void* o, float* lse,
                                          void* stream) {
  bsa_status_t st = decode_checks(s, q, k_cache, v_cache, o);
  if (st != BSA_OK) return st;
  const int nb = s->Nk / s->block;
  if (!idx || idx_stride < 1 || !(softmax_scale > 0.0f) || !workspace) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  if (nb % 32 != 0 || nb > 8192) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  const HeadsLayout L = heads_layout(s, idx_stride, sms);
  if (workspace_bytes < L.total) return BSA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int G = s->Hq / s->Hkv;
  const int rows = s->B * s->Hq;
  uint32_t* expanded = reinterpret_cast<uint32_t*>(ws + L.expanded);
  int* ulist = reinterpret_cast<int*>(ws + L.union_list);
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, q, static_cast<uint64_t>(rows), static_cast<uint32_t>(G)) ||
      !make_map_bf16(&mk, k_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64) ||
      !make_map_bf16(&mv, v_cache, static_cast<uint64_t>(s->B) * s->Hkv * s->Nk, 64))
    return BSA_ERR_CUDA;
  // the union of the heads' kept blocks, each head's bitmap; no gists
  cudaError_t e = launch_gist_union(idx, s->B, s->Hq, s->Hkv, idx_stride, idx_stride, nb, expanded, ulist,
                                    L.union_stride, false, status, cs);
  DecodeArgs a;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.Nk = s->Nk;
  a.bs = s->block;
  a.list = ulist;
  a.list_stride = L.union_stride;
  a.list_has_count = 1;
  a.expanded = expanded;
  a.nc = nb;
  a.list_len = L.plan.list_len;
  a.num_ctas = L.plan.num_ctas;
  a.max_slots = L.plan.max_slots;
  a.softmax_scale = softmax_scale;
  a.partial = reinterpret_cast<float*>(ws + L.partial);
  a.status = status;
  if (e == cudaSuccess) e = launch_attn_decode_bf16(&mq, &mk, &mv, &mk, &mv, a, cs);
  if (e == cudaSuccess) e = launch_decode_combine(a.partial, a, s->d, true, o, lse, cs);
  return cuda_status(e);
}

bsa_status_t bsa_sparse_attn_decode_paged(const bsa_shape_t* s, const void* q, const void* k_pool, const void* v_pool,
                                          int num_pages, const int* block_table, int table_stride, const int* idx,
                                          int idx_stride, float softmax_scale, void* workspace,
                                          size_t workspace_bytes, void* o, float* lse, void* stream) {
  bsa_status_t st = decode_checks(s, q, k_pool, v_pool, o);
  if (st != BSA_OK) return st;
  const int nb = s->Nk / s->block;
  if (!block_table || num_pages < 1 || table_stride < nb) return BSA_ERR_INVALID_ARG;
  if (!idx || idx_stride < 1 || !(softmax_scale > 0.0f) || !workspace) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(num_pages) * s->Hkv * s->block >= (1ll << 31)) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  const int G = s->Hq / s->Hkv;
  const DecodePlan P = decode_plan(s->B * s->Hkv, idx_stride, sms);
  const size_t need = align256(static_cast<size_t>(s->B) * s->Hq * P.max_slots * (s->d + 4) * sizeof(float));
  if (workspace_bytes < need) return BSA_ERR_INVALID_ARG;
  const uint64_t pool_rows = static_cast<uint64_t>(num_pages) * s->Hkv * s->block;
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, q, static_cast<uint64_t>(s->B) * s->Hq, static_cast<uint32_t>(G)) ||
      !make_map_bf16(&mk, k_pool, pool_rows, 64) || !make_map_bf16(&mv, v_pool, pool_rows, 64))
    return BSA_ERR_CUDA;
  DecodeArgs a;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.Nk = s->Nk;
  a.bs = s->block;
  a.list = idx;
  a.list_stride = idx_stride;
  a.list_has_count = 0;
  a.expanded = nullptr;
  a.nc = 0;
  a.list_len = P.list_len;
  a.num_ctas = P.num_ctas;
  a.max_slots = P.max_slots;
  a.softmax_scale = softmax_scale;
  a.partial = static_cast<float*>(workspace);
  a.status = status;
  a.table = block_table;
  a.table_stride = table_stride;
  a.num_pages = num_pages;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_attn_decode_bf16(&mq, &mk, &mv, nullptr, nullptr, a, cs);
  if (e == cudaSuccess) e = launch_decode_combine(a.partial, a, s->d, true, o, lse, cs);
  return cuda_status(e);
}

bsa_status_t bsa_paged_append(const bsa_shape_t* s, const void* k_new, const void* v_new, const int* seq_lens,
                              const int* block_table, int table_stride, int num_pages, void* k_pool, void* v_pool,
                              float* pooled_k, void* stream) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (!k_new || !v_new || !seq_lens || !block_table || !k_pool || !v_pool) return BSA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool)) return BSA_ERR_INVALID_ARG;
  if (pooled_k && !aligned16(pooled_k)) return BSA_ERR_INVALID_ARG;
  if (table_stride < 1 || num_pages < 1) return BSA_ERR_INVALID_ARG;
  if (s->dtype != BSA_BF16 || s->block != 64 || s->d % 8 != 0 || s->d > 1024) return BSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(num_pages) * s->Hkv * s->block * s->d >= (1ll << 40)) return BSA_ERR_UNSUPPORTED;
  uint32_t* status = nullptr;
  if ((st = device_state(&status, nullptr)) != BSA_OK) return st;
  return cuda_status(launch_paged_append(k_new, v_new, s->B, s->Hkv, s->Nq, s->d, seq_lens, block_table,
                                         table_stride, num_pages, k_pool, v_pool, pooled_k, status,
                                         static_cast<cudaStream_t>(stream)));
}

bsa_status_t bsa_hssa_decode(const bsa_shape_t* s, const void* q, const void* k_cache, const void* v_cache,
                             const void* gist_k, const void* gist_v, const void* meta_k, const void* meta_v, int km,
                             int topk, int* meta_out, int* idx_out, float softmax_scale, void* workspace,
                             size_t workspace_bytes, void* o, float* lse, void* stream) {
  bsa_status_t st = decode_checks(s, q, k_cache, v_cache, o);
  if (st != BSA_OK) return st;
  const int nc = s->Nk / s->block;
  if (!gist_k || !gist_v || !meta_k || !meta_v) return BSA_ERR_INVALID_ARG;
  if (!aligned16(gist_k) || !aligned16(gist_v) || !aligned16(meta_k) || !aligned16(meta_v)) return BSA_ERR_INVALID_ARG;
  if (nc % 64 != 0 || nc / 64 > 64) return BSA_ERR_UNSUPPORTED;   // groups of 64 chunks, at most 64 groups
  const int nm = nc / 64;
  if (km < 1 || km > nm || topk < 0 || topk > km * 64 || !(softmax_scale > 0.0f) || !workspace)
    return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  const HssaLayout L = hssa_layout(s, km, topk, sms);
  if (workspace_bytes < L.total) return BSA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int G = s->Hq / s->Hkv;
  const int rows = s->B * s->Hq;
  const uint64_t bgs = static_cast<uint64_t>(s->B) * s->Hkv;
  CUtensorMap mq, mk, mv, mgk, mgv, mmk, mmv;
  if (!make_map_bf16(&mq, q, static_cast<uint64_t>(rows), static_cast<uint32_t>(G)) ||
      !make_map_bf16(&mk, k_cache, bgs * s->Nk, 64) || !make_map_bf16(&mv, v_cache, bgs * s->Nk, 64) ||
      !make_map_bf16(&mgk, gist_k, bgs * nc, 64) || !make_map_bf16(&mgv, gist_v, bgs * nc, 64) ||
      !make_map_bf16(&mmk, meta_k, bgs * nm, 64) || !make_map_bf16(&mmv, meta_v, bgs * nm, 64))
    return BSA_ERR_CUDA;
  const float scale = score_scale(s->d);
  float* meta_scores = reinterpret_cast<float*>(ws + L.meta_scores);
  int* meta_idx = meta_out ? meta_out : reinterpret_cast<int*>(ws + L.meta_idx);
  float* fine = reinterpret_cast<float*>(ws + L.fine);
  int* pos = reinterpret_cast<int*>(ws + L.pos);
  int* chunks = (idx_out && topk > 0) ? idx_out : reinterpret_cast<int*>(ws + L.chunks);
  uint32_t* expanded = reinterpret_cast<uint32_t*>(ws + L.expanded);
  uint32_t* allow = reinterpret_cast<uint32_t*>(ws + L.allow);
  int* ulist = reinterpret_cast<int*>(ws + L.union_list);
  // coarse: meta-gist scores and the km best groups per head
  cudaError_t e = launch_score_gist(&mmk, q, meta_k, true, s->B, s->Hq, s->Hkv, nm, s->d, scale, meta_scores, status,
                                    sms, cs);
  if (e == cudaSuccess) e = launch_topk(meta_scores, rows, nm, BSA_TOPK_PLAIN, km, meta_idx, km, nullptr, cs);
  // fine: the gists of the kept groups' chunks and the topk best per head
  // (with up to 32 kept groups the row's top-k runs in the scoring launch)
  const bool fuse_fine = gist_groups_select_fused_ok(km);
  if (e == cudaSuccess)
    e = launch_score_gist_groups(&mgk, q, meta_idx, km, s->B, s->Hq, s->Hkv, nc, scale, fine, topk,
                                 fuse_fine ? pos : nullptr, L.k_stride, status, cs);
  if (e == cudaSuccess && !fuse_fine)
    e = launch_topk(fine, rows, km * 64, BSA_TOPK_PLAIN, topk, pos, L.k_stride, nullptr, cs);
  if (e == cudaSuccess)
    e = launch_hssa_union(meta_idx, km, pos, L.k_stride, s->B, s->Hq, s->Hkv, nc, nm, chunks, expanded, allow, ulist,
                          L.union_stride, status, cs);
  DecodeArgs a;
  a.B = s->B;
  a.Hq = s->Hq;
  a.Hkv = s->Hkv;
  a.Nk = s->Nk;
  a.bs = s->block;
  a.list = ulist;
  a.list_stride = L.union_stride;
  a.list_has_count = 1;
  a.expanded = expanded;
  a.nc = nc;
  a.list_len = L.plan.list_len;
  a.num_ctas = L.plan.num_ctas;
  a.max_slots = L.plan.max_slots;
  a.softmax_scale = softmax_scale;
  a.partial = reinterpret_cast<float*>(ws + L.partial);
  a.status = status;
  a.gist_allow = allow;
  a.meta_rows = nm;
  if (e == cudaSuccess) e = launch_attn_decode_bf16(&mq, &mk, &mv, &mgk, &mgv, a, cs, &mmk, &mmv);
  if (e == cudaSuccess) e = launch_decode_combine(a.partial, a, s->d, true, o, lse, cs);
  return cuda_status(e);
}

size_t bsa_workspace_bytes_bwd(const bsa_shape_t* s, int idx_stride) {
  if (check_shape(s) != BSA_OK || idx_stride < 1 || s->Nq != s->Nk) return 0;
  return attn_bwd_workspace(s->B, s->Hq, s->Hkv, s->Nk, s->block, idx_stride);
}

bsa_status_t bsa_gated_attn_bwd(const bsa_shape_t* s, const void* q, const void* k, const void* v,
                                const float* lse, const void* d_o, const int* idx, int idx_stride,
                                const float* sel_scores, float softmax_scale, float* dq, float* dk, float* dv,
                                float* dsel, void* workspace, size_t workspace_bytes, void* stream) {
  bsa_status_t st = check_shape(s);
  if (st != BSA_OK) return st;
  if (s->Nq != s->Nk) return BSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !lse || !d_o || !idx || !dq || !dk || !dv || !workspace) return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return BSA_ERR_INVALID_ARG;
  if (dsel && !sel_scores) return BSA_ERR_INVALID_ARG;
  if (idx_stride < 1 || !(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  if (s->dtype != BSA_BF16 || s->d != 128 || (s->block != 64 && s->block != 128)) return BSA_ERR_UNSUPPORTED;
  if (idx_stride > 256) return BSA_ERR_UNSUPPORTED;   // the dQ pass keeps per-slot sums for 256 slots
  if (workspace_bytes < attn_bwd_workspace(s->B, s->Hq, s->Hkv, s->Nk, s->block, idx_stride))
    return BSA_ERR_INVALID_ARG;
  uint32_t* status = nullptr;
  int sms = 0;
  if ((st = device_state(&status, &sms)) != BSA_OK) return st;
  CUtensorMap mq, mdo, mk, mv;
  const uint64_t qrows = static_cast<uint64_t>(s->B) * s->Hq * s->Nk, kvrows = static_cast<uint64_t>(s->B) * s->Hkv * s->Nk;
  if (!make_map_bf16(&mq, q, qrows, 64) || !make_map_bf16(&mdo, d_o, qrows, 64) ||
      !make_map_bf16(&mk, k, kvrows, 64) || !make_map_bf16(&mv, v, kvrows, 64))
    return BSA_ERR_CUDA;
  return cuda_status(launch_attn_bwd(&mq, &mdo, &mk, &mv, lse, idx, idx_stride, sel_scores, softmax_scale, s->B,
                                     s->Hq, s->Hkv, s->Nk, s->block, dq, dk, dv, dsel, workspace, status, sms,
                                     static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
