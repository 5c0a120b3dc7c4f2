// attn_f32.cu -- block-sparse causal attention (prefill) for fp32 inputs, on
// CUDA cores in fp32.  The tensor cores' fp32-input mode (TF32) keeps only 10
// mantissa bits, too coarse for fp32 parity, so this small-shape path stays
// in plain fp32 arithmetic.
//
// Same definition as the bf16 kernel: softmax(QK^T/sqrt(d) + M)V over the
// kept blocks with causality inside the current block ("稀疏注意力" tutorial
// §1-2, §4.5), optionally with the SAS log-gate log g_j on every key of kept
// block j (SAS page, 核心模块 2-3).
//
// One CTA per (query block i, query head h, batch b); four threads per query
// row, each holding a quarter of the channels (dot products finished with two
// shuffles).  Each kept K/V block is staged in shared memory; a row first
// scores all of the block's keys (independent dot products), then moves its
// running maximum once per block and accumulates the block's keys.
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace f32path {

constexpr int kMaxList = 256;

template <int D>
__global__ void attn_prefill_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                        const float* __restrict__ v, int Hq, int Hkv, int N, int bs,
                                        const int* __restrict__ idx, int idx_stride, const float* __restrict__ sel,
                                        float scale, float* __restrict__ o, float* __restrict__ lse,
                                        uint32_t* __restrict__ status) {
  extern __shared__ float sm[];
  float* ks = sm;                 // [bs][D]
  float* vs = sm + bs * D;        // [bs][D]
  __shared__ int s_list[kMaxList];
  __shared__ float s_bias[kMaxList];
  __shared__ int s_n;
  const int nb = N / bs;
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, g = h / G;
  const int t = threadIdx.x;
  const int64_t bg = static_cast<int64_t>(b) * Hkv + g;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int* src = idx + (bg * nb + i) * idx_stride;
    const unsigned lt = (1u << lane) - 1u;
    int count = 0, prev = -1;
    for (int base = 0; base < idx_stride; base += 32) {
      const int tt = base + lane;
      const int j = (tt < idx_stride) ? src[tt] : -1;
      const unsigned neg = __ballot_sync(0xffffffffu, j < 0);
      const int lim = neg ? __ffs(neg) - 1 : 32;
      int jprev = __shfl_up_sync(0xffffffffu, j, 1);
      if (lane == 0) jprev = prev;
      const bool in = lane < lim;
      const bool ok = in && j <= i && j > jprev && count + lim <= kMaxList;
      if (in && !ok) atomicOr(status, BSA_DEV_BAD_INDEX);
      const unsigned okm = __ballot_sync(0xffffffffu, ok);
      if (ok) s_list[count + __popc(okm & lt)] = j;
      count += __popc(okm);
      prev = __shfl_sync(0xffffffffu, j, 31);
      if (neg) break;
    }
    __syncwarp();
    // gate: natural-log weights log g_j = s_j - logsumexp over the kept blocks
    if (sel != nullptr && count > 0) {
      const float* srow = sel + (bg * nb + i) * nb;
      float mx = -INFINITY;
      for (int tt = lane; tt < count; tt += 32) mx = fmaxf(mx, srow[s_list[tt]]);
      for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      float sum = 0.0f;
      if (mx > -INFINITY)
        for (int tt = lane; tt < count; tt += 32) sum += expf(srow[s_list[tt]] - mx);
      for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const float lse_s = (mx > -INFINITY) ? mx + logf(sum) : 0.0f;
      for (int tt = lane; tt < count; tt += 32) s_bias[tt] = (mx > -INFINITY) ? srow[s_list[tt]] - lse_s : 0.0f;
    } else {
      for (int tt = lane; tt < count; tt += 32) s_bias[tt] = 0.0f;
    }
    if (lane == 0) s_n = count;
  }
  __syncthreads();
  constexpr int DQ = D / 4;           // channels per thread
  const int n = s_n;
  const int r = t >> 2, qt = t & 3;   // query row inside the block, channel quarter
  const int tpos = i * bs + r;
  const float* qrow = q + ((static_cast<int64_t>(b) * Hq + h) * N + tpos) * D + qt * DQ;
  float qr[DQ], acc[DQ];
#pragma unroll
  for (int c = 0; c < DQ; ++c) {
    qr[c] = qrow[c];
    acc[c] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  for (int e = 0; e < n; ++e) {
    const int j = s_list[e];
    const float bias = s_bias[e];
    __syncthreads();
    const float4* kb = reinterpret_cast<const float4*>(k + (bg * N + static_cast<int64_t>(j) * bs) * D);
    const float4* vb = reinterpret_cast<const float4*>(v + (bg * N + static_cast<int64_t>(j) * bs) * D);
    for (int x = threadIdx.x; x < bs * D / 4; x += blockDim.x) {
      reinterpret_cast<float4*>(ks)[x] = kb[x];
      reinterpret_cast<float4*>(vs)[x] = vb[x];
    }
    __syncthreads();
    const int umax = (j == i) ? r : bs - 1;   // causal inside the current block
    // the key loop runs to the warp's last row (r | 7: a warp holds 8 rows),
    // so every lane takes part in the shuffles; keys past umax are masked
    const int uend = (j == i) ? (r | 7) : bs - 1;
    // scores of the block's keys in chunks of 16, the chunk's maximum first
    for (int u0 = 0; u0 <= uend; u0 += 16) {
      float sc[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float* kr = ks + (u0 + x) * D + qt * DQ;
        float dot = 0.0f;
#pragma unroll
        for (int c = 0; c < DQ; ++c) dot = fmaf(qr[c], kr[c], dot);
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        sc[x] = (u0 + x <= umax) ? dot * scale + bias : -INFINITY;
      }
      float mb = sc[0];
#pragma unroll
      for (int x = 1; x < 16; ++x) mb = fmaxf(mb, sc[x]);
      if (mb > m) {
        const float rs = expf(m - mb);   // m = -inf -> 0
        l *= rs;
#pragma unroll
        for (int c = 0; c < DQ; ++c) acc[c] *= rs;
        m = mb;
      }
      if (m == -INFINITY) continue;   // every score so far is -inf (a -inf gate weight)
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float pw = expf(sc[x] - m);
        l += pw;
        const float* vr = vs + (u0 + x) * D + qt * DQ;
#pragma unroll
        for (int c = 0; c < DQ; ++c) acc[c] = fmaf(pw, vr[c], acc[c]);
      }
    }
  }
  float* orow = o + ((static_cast<int64_t>(b) * Hq + h) * N + tpos) * D + qt * DQ;
  const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
#pragma unroll
  for (int c = 0; c < DQ; ++c) orow[c] = acc[c] * inv;
  if (lse && qt == 0) lse[(static_cast<int64_t>(b) * Hq + h) * N + tpos] = (l > 0.0f) ? m + logf(l) : -INFINITY;
}

}  // namespace f32path

cudaError_t launch_attn_prefill_f32(const float* q, const float* k, const float* v, const PrefillArgs& a, int d,
                                    cudaStream_t st) {
  const int nb = a.N / a.bs;
  dim3 grid(nb, a.Hq, a.B);
  const size_t smem = 2ull * a.bs * d * sizeof(float);
  if (d == 64) {
    cudaError_t e = cudaFuncSetAttribute(f32path::attn_prefill_f32_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    f32path::attn_prefill_f32_kernel<64><<<grid, 4 * a.bs, smem, st>>>(q, k, v, a.Hq, a.Hkv, a.N, a.bs, a.idx,
                                                                   a.idx_stride, a.sel_scores, a.softmax_scale,
                                                                   static_cast<float*>(a.o), a.lse, a.status);
  } else {
    cudaError_t e = cudaFuncSetAttribute(f32path::attn_prefill_f32_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    f32path::attn_prefill_f32_kernel<128><<<grid, 4 * a.bs, smem, st>>>(q, k, v, a.Hq, a.Hkv, a.N, a.bs, a.idx,
                                                                    a.idx_stride, a.sel_scores, a.softmax_scale,
                                                                    static_cast<float*>(a.o), a.lse, a.status);
  }
  return cudaGetLastError();
}

}  // namespace bsa
