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
// One CTA per (query block i, query head h, batch b); one thread per query
// row.  Each kept K/V block is staged in shared memory and every thread runs
// an online softmax over its keys.
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
  const int n = s_n;
  const int tpos = i * bs + t;
  const float* qrow = q + ((static_cast<int64_t>(b) * Hq + h) * N + tpos) * D;
  float qr[D], acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    qr[c] = qrow[c];
    acc[c] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  for (int e = 0; e < n; ++e) {
    const int j = s_list[e];
    const float bias = s_bias[e];
    __syncthreads();
    const float* kb = k + (bg * N + static_cast<int64_t>(j) * bs) * D;
    const float* vb = v + (bg * N + static_cast<int64_t>(j) * bs) * D;
    for (int x = threadIdx.x; x < bs * D; x += blockDim.x) {
      ks[x] = kb[x];
      vs[x] = vb[x];
    }
    __syncthreads();
    const int umax = (j == i) ? t : bs - 1;   // causal inside the current block
    for (int u = 0; u <= umax; ++u) {
      float dot = 0.0f;
#pragma unroll
      for (int c = 0; c < D; ++c) dot = fmaf(qr[c], ks[u * D + c], dot);
      const float s = dot * scale + bias;
      if (s > m) {
        const float r = expf(m - s);   // m = -inf -> 0
        l *= r;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] *= r;
        m = s;
      }
      const float pw = expf(s - m);
      l += pw;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(pw, vs[u * D + c], acc[c]);
    }
  }
  float* orow = o + ((static_cast<int64_t>(b) * Hq + h) * N + tpos) * D;
  const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
#pragma unroll
  for (int c = 0; c < D; ++c) orow[c] = acc[c] * inv;
  if (lse) lse[(static_cast<int64_t>(b) * Hq + h) * N + tpos] = (l > 0.0f) ? m + logf(l) : -INFINITY;
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
    f32path::attn_prefill_f32_kernel<64><<<grid, a.bs, smem, st>>>(q, k, v, a.Hq, a.Hkv, a.N, a.bs, a.idx,
                                                                   a.idx_stride, a.sel_scores, a.softmax_scale,
                                                                   static_cast<float*>(a.o), a.lse, a.status);
  } else {
    cudaError_t e = cudaFuncSetAttribute(f32path::attn_prefill_f32_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    f32path::attn_prefill_f32_kernel<128><<<grid, a.bs, smem, st>>>(q, k, v, a.Hq, a.Hkv, a.N, a.bs, a.idx,
                                                                    a.idx_stride, a.sel_scores, a.softmax_scale,
                                                                    static_cast<float*>(a.o), a.lse, a.status);
  }
  return cudaGetLastError();
}

}  // namespace bsa
