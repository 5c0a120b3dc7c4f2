// paged.cu -- upkeep of a paged KV cache: new tokens written into their
// physical blocks, and the block-mean summary the decode selector reads kept
// up to date block by block.
//
// PagedAttention ("稀疏注意力" tutorial §7): a sequence's logically
// contiguous KV cache is mapped onto physical blocks that need not be
// contiguous.  The pools are [P][Hkv][64][d] (bf16): physical block p of KV
// head g is the 64 rows starting at row (p * Hkv + g) * 64.  block_table
// [B][table_stride] maps sequence b's logical block j to its physical block.
// The selector of decode scores the query against one mean key per logical
// block (tutorial §4.6 coarse block scoring; §5 decode); with a retained
// cache (Sparse Frontier review §2.4.2) that summary is maintained as the
// cache grows: when an append completes a block, its mean is computed once,
// in the fixed order of the pooling kernel (tokens ascending, fp32 sums,
// one division), so it equals pooling the whole cache from scratch bit for
// bit.
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace paged {

// One thread per (sequence, KV head, new token, 16-byte piece of the row):
// token t of sequence b goes to logical position seq_lens[b] + t.
__global__ void paged_scatter_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
                                     int Hkv, int T, int d, const int* __restrict__ seq_lens,
                                     const int* __restrict__ table, int table_stride, int num_pages,
                                     __nv_bfloat16* __restrict__ k_pool, __nv_bfloat16* __restrict__ v_pool,
                                     int64_t total, uint32_t* __restrict__ status) {
  griddep_wait();
  const int pieces = d / 8;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int piece = static_cast<int>(e % pieces);
  const int64_t row = e / pieces;             // (b * Hkv + g) * T + t
  const int t = static_cast<int>(row % T);
  const int64_t bg = row / T;
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int pos = seq_lens[b] + t;
  const int j = pos >> 6, o = pos & 63;
  if (pos < 0 || j >= table_stride) {
    atomicOr(status, BSA_DEV_BAD_INDEX);
    return;
  }
  const int pg = table[static_cast<int64_t>(b) * table_stride + j];
  if (pg < 0 || pg >= num_pages) {
    atomicOr(status, BSA_DEV_BAD_INDEX);
    return;
  }
  const int64_t dst = ((static_cast<int64_t>(pg) * Hkv + g) * 64 + o) * d + piece * 8;
  const int64_t src = row * d + piece * 8;
  *reinterpret_cast<uint4*>(k_pool + dst) = __ldg(reinterpret_cast<const uint4*>(k_new + src));
  *reinterpret_cast<uint4*>(v_pool + dst) = __ldg(reinterpret_cast<const uint4*>(v_new + src));
}

// One thread per (sequence, KV head, completed block, 8 channels): the blocks
// j with seq_lens[b] < 64(j+1) <= seq_lens[b] + T were completed by this
// append.  Their mean key is summed over the block's 64 tokens ascending in
// fp32, then divided by 64 (the pooling kernel's arithmetic).
__global__ void paged_pool_kernel(const __nv_bfloat16* __restrict__ k_pool, int Hkv, int T, int d,
                                  const int* __restrict__ seq_lens, const int* __restrict__ table, int table_stride,
                                  int num_pages, int max_new, float* __restrict__ pooled_k, int64_t total) {
  griddep_wait();   // the new tokens are written by the kernel launched before
  const int groups = d / 8;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int cg = static_cast<int>(e % groups);
  const int64_t u = e / groups;               // ((b * Hkv + g) * max_new + n)
  const int n = static_cast<int>(u % max_new);
  const int64_t bg = u / max_new;
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int L = seq_lens[b];
  const int j = (L >> 6) + n;                 // candidate block
  if ((j + 1) * 64 > L + T || j >= table_stride) return;   // not completed by this append
  const int pg = table[static_cast<int64_t>(b) * table_stride + j];
  if (pg < 0 || pg >= num_pages) return;      // flagged by the scatter kernel
  const __nv_bfloat16* src = k_pool + (static_cast<int64_t>(pg) * Hkv + g) * 64 * d + cg * 8;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  for (int t = 0; t < 64; ++t) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(t) * d));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = __fadd_rn(acc[2 * i], __uint_as_float(ws[i] << 16));
      acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __uint_as_float(ws[i] & 0xFFFF0000u));
    }
  }
  float* out = pooled_k + (bg * table_stride + j) * d + cg * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) out[c] = __fdiv_rn(acc[c], 64.0f);
}

}  // namespace paged

cudaError_t launch_paged_append(const void* k_new, const void* v_new, int B, int Hkv, int T, int d,
                                const int* seq_lens, const int* table, int table_stride, int num_pages, void* k_pool,
                                void* v_pool, float* pooled_k, uint32_t* status, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(B) * Hkv * T * (d / 8);
  if (total > 0) {
    const unsigned grid = static_cast<unsigned>((total + 255) / 256);
    cudaError_t e = launch_dependent(paged::paged_scatter_kernel, dim3(grid), dim3(256), 0, st,
                                     static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
                                     Hkv, T, d, seq_lens, table, table_stride, num_pages,
                                     static_cast<__nv_bfloat16*>(k_pool), static_cast<__nv_bfloat16*>(v_pool), total,
                                     status);
    if (e != cudaSuccess) return e;
  }
  if (pooled_k == nullptr) return cudaSuccess;
  // a sequence completes at most T/64 + 1 blocks in one append
  const int max_new = T / 64 + 1;
  const int64_t ptotal = static_cast<int64_t>(B) * Hkv * max_new * (d / 8);
  const unsigned pgrid = static_cast<unsigned>((ptotal + 255) / 256);
  return launch_dependent(paged::paged_pool_kernel, dim3(pgrid), dim3(256), 0, st,
                          static_cast<const __nv_bfloat16*>(k_pool), Hkv, T, d, seq_lens, table, table_stride,
                          num_pages, max_new, pooled_k, ptotal);
}

}  // namespace bsa
