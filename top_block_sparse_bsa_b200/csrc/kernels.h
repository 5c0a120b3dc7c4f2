// kernels.h -- internal launchers of libbsa (C++ linkage, not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace bsa {

// Identifier of the CUDA context current on the calling thread (unique for
// the life of the process: a context created after a device reset gets a new
// one); 0 if it cannot be read.  Per-device caches of device addresses and
// function attributes are keyed on it, because a device reset unloads the
// module they belong to.
uint64_t current_context_id();

// Opt kernel Fn into `bytes` of dynamic shared memory on the current device.
// The attribute belongs to the function in the current context and persists,
// so the driver call is made only when a context sees a larger request than
// before; launches after the first cost no extra driver call.
template <auto Fn>
inline cudaError_t ensure_dynamic_smem(size_t bytes) {
  static std::atomic<uint64_t> granted_ctx[32];
  static std::atomic<uint32_t> granted[32];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
  const uint64_t ctx = current_context_id();
  if (ctx != 0 && granted_ctx[dev].load(std::memory_order_acquire) == ctx &&
      granted[dev].load(std::memory_order_acquire) >= bytes)
    return cudaSuccess;
  e = cudaFuncSetAttribute(Fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  if (granted_ctx[dev].exchange(ctx, std::memory_order_acq_rel) != ctx) {
    granted[dev].store(static_cast<uint32_t>(bytes), std::memory_order_release);
  } else {
    uint32_t cur = granted[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !granted[dev].compare_exchange_weak(cur, static_cast<uint32_t>(bytes))) {
    }
  }
  return cudaSuccess;
}

// Launch a kernel that may start while the previous kernel on the stream is
// finishing (programmatic dependent launch): its launch and prologue overlap
// that kernel's tail, and it calls griddep_wait() before reading that
// kernel's output.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// selector.cu
cudaError_t launch_pool(const void* src, bool bf16, int B, int Hsrc, int Hgroups, int heads_sum, int N,
                        int d, int bs, float* out, cudaStream_t st);
cudaError_t launch_pool_prefill(const void* q, const void* k, bool bf16, int B, int Hq, int Hkv, int N, int d,
                                int bs, float* qbar, float* kbar, int num_sms, uint32_t* status, cudaStream_t st);
cudaError_t launch_score_prefill(const float* qbar, const float* kbar, int B, int Hkv, int nb, int d,
                                 float scale, float* s, cudaStream_t st);
cudaError_t launch_score_decode(const void* q, bool bf16, const float* kbar, int B, int Hq, int Hkv,
                                int nb, int d, float scale, float* s, float* qbar_out, cudaStream_t st);
// tmG: the gist keys as make_map_bf16 (rows B*Hkv*nc, box 64 rows), or null
// (then the generic kernel runs; bf16 with d = 128 uses the TMA kernel).
cudaError_t launch_score_gist(const CUtensorMap* tmG, const void* q, const void* gk, bool bf16, int B, int Hq,
                              int Hkv, int nc, int d, float scale, float* s, uint32_t* status, int num_sms,
                              cudaStream_t st);
cudaError_t launch_topk(const float* scores, int rows, int ncols, int mode, int kb, int* idx_out,
                        int idx_stride, int* count_out, cudaStream_t st);
cudaError_t launch_topk_pattern(const float* scores, int rows, int ncols, int sink, int local, int kb, int* idx_out,
                                int idx_stride, int* count_out, cudaStream_t st);
cudaError_t launch_score_heads(const void* q, bool bf16, const float* kbar, int B, int Hq, int Hkv, int nb, int d,
                               float scale, float* s, cudaStream_t st);
cudaError_t launch_topk_joint(const float* scores, int rows, int G, int nb, int kb_total, int* idx_out,
                              int idx_stride, int* count_out, cudaStream_t st);
// pos_out non-null: the row's top-k positions (topk of km*64, pos_stride apart) are
// selected in the same launch and the fine scores are not written (km*64 <= 2048)
bool gist_groups_select_fused_ok(int km);
cudaError_t launch_score_gist_groups(const CUtensorMap* tmG, const void* q, const int* meta_idx, int km, int B,
                                     int Hq, int Hkv, int nc, float scale, float* fine, int topk, int* pos_out,
                                     int pos_stride, uint32_t* status, cudaStream_t st);
// decode scores + top-k in one kernel (tmKbar: fp32 [rows, 128], box 32 x 128, 128-byte swizzle)
bool decode_select_fused_ok(int d, int nb);
cudaError_t launch_decode_select(const CUtensorMap* tmKbar, const void* q, bool bf16, int B, int Hq, int Hkv,
                                 int nb, float scale, int kb, float* scores, float* qbar_out, int* idx_out,
                                 int idx_stride, int* count_out, uint32_t* status, cudaStream_t st);

// attn_prefill.cu (bf16, d = 128, tcgen05)
struct PrefillArgs {
  int B, Hq, Hkv, N, bs;
  const int* idx;
  int idx_stride;
  const float* sel_scores;   // non-null: gated (SAS log-gate)
  float softmax_scale;
  void* o;
  float* lse;
  uint32_t* status;
  int num_sms;
  int kernel;                // 0: chosen by shape; 1 paired tiles; 2 one tile per item; 3 SM pair
};
cudaError_t launch_attn_prefill_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                     const PrefillArgs& a, cudaStream_t st);
// attn_prefill_split.cu (one tile per item; called for odd tile counts per unit)
cudaError_t launch_attn_prefill_split_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                           const PrefillArgs& a, cudaStream_t st);

// attn_prefill_pair.cu (two SMs per item, MMAs of M = 256)
cudaError_t launch_attn_prefill_pair_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                          const PrefillArgs& a, cudaStream_t st);

// attn_bwd.cu (backward of the sparse / gated prefill attention)
size_t attn_bwd_workspace(int B, int Hq, int Hkv, int N, int bs, int idx_stride);
cudaError_t launch_attn_bwd(const CUtensorMap* tmQ, const CUtensorMap* tmDO, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const float* lse, const int* idx, int idx_stride,
                            const float* sel, float scale, int B, int Hq, int Hkv, int N, int bs, float* dq,
                            float* dk, float* dv, float* dsel, void* workspace, uint32_t* status, int num_sms,
                            cudaStream_t st);

// paged.cu (paged cache upkeep)
cudaError_t launch_paged_append(const void* k_new, const void* v_new, int B, int Hkv, int T, int d,
                                const int* seq_lens, const int* table, int table_stride, int num_pages, void* k_pool,
                                void* v_pool, float* pooled_k, uint32_t* status, cudaStream_t st);

// attn_f32.cu (fp32 SIMT path)
cudaError_t launch_attn_prefill_f32(const float* q, const float* k, const float* v, const PrefillArgs& a,
                                    int d, cudaStream_t st);

// attn_decode.cu (bf16, d = 128, tcgen05, split-K + combine)
struct DecodeArgs {
  int B, Hq, Hkv, Nk, bs;
  // tile list: plain decode reads idx [B*Hkv][list_stride]; gist decode reads
  // the union list built in the workspace (count at [bg][0], entries after).
  const int* list;
  int list_stride;
  int list_has_count;        // 1: entry 0 is the count (gist union list)
  const uint32_t* expanded;  // gist: [B*Hq][nc/32] bitmap of expanded chunks; null for plain decode
  int nc;                    // gist: number of chunks
  int list_len;              // list positions per group row (split space = rows x list_len)
  int num_ctas;              // persistent CTAs sharing the split space
  int max_slots;             // partial records per output row
  float softmax_scale;
  float* partial;            // [B*Hq][max_slots][d+4]
  uint32_t* status;
  // paged cache (plain decode): logical block j of sequence b is physical block
  // table[b*table_stride + j] of pools [num_pages][Hkv][64][d]; null: contiguous
  const int* table = nullptr;
  int table_stride = 0, num_pages = 0;
  // two-level gists: per-head allowed gist / meta-gist rows; meta rows per (b, g)
  const uint32_t* gist_allow = nullptr;
  int meta_rows = 0;
  // gist decode with the union built inside the attention kernel (nc <= 2048,
  // G <= 16): the heads' kept chunk lists replace list / expanded
  const int* heads_idx = nullptr;
  int heads_topk = 0, heads_stride = 0;
};
cudaError_t launch_attn_decode_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                    const CUtensorMap* tmGK, const CUtensorMap* tmGV, const DecodeArgs& a,
                                    cudaStream_t st, const CUtensorMap* tmMK = nullptr,
                                    const CUtensorMap* tmMV = nullptr);
cudaError_t launch_hssa_union(const int* meta_idx, int km, const int* pos_idx, int k, int B, int Hq, int Hkv, int nc,
                              int nm, int* chunk_out, uint32_t* expanded, uint32_t* gist_allow, int* union_list,
                              int union_stride, uint32_t* status, cudaStream_t st);
cudaError_t launch_decode_combine(const float* partial, const DecodeArgs& a, int d, bool out_bf16, void* o,
                                  float* lse, cudaStream_t st);
int decode_slots_for(int rows, int list_len, int num_ctas);
cudaError_t launch_gist_union(const int* idx, int B, int Hq, int Hkv, int topk, int idx_stride, int nc,
                              uint32_t* expanded, int* union_list, int union_stride, bool with_gists,
                              uint32_t* status, cudaStream_t st);

}  // namespace bsa
