// attn_bwd.cu -- backward of the block-sparse (and SAS gated) prefill
// attention, bf16 inputs, d = 128, fp32 arithmetic on the CUDA cores.
//
// What it computes (SAS page, 核心洞察 and 核心模块 2: the selector's
// continuous score sits inside the softmax logits in log form, so the
// language-modelling loss reaches it by ordinary back-propagation).  With the
// forward's P_{t,u} = exp(scale q_t.k_u + log g_{j(u)} - LSE_t) over the kept,
// causal keys of row t (LSE_t: the forward's natural-log row LSE) and the
// upstream gradient dO:
//   D_t      = dO_t . O_t
//   dl_{t,u} = P_{t,u} (dO_t . v_u - D_t)
//   dQ_t     = scale sum_u dl_{t,u} k_u           (query-block-major pass)
//   dK_u     = scale sum_t dl_{t,u} q_t,  dV_u = sum_t P_{t,u} dO_t
//                                                 (key-block-major pass)
//   for a unit (b, g, i) and its kept block l:
//   dsel_l   = dlogg_l - g_l sum_j dlogg_j,  dlogg_j = sum over the unit's
//              rows t and block j's keys u of dl_{t,u}.
// Both passes recompute P from Q, K and the saved LSE (no n x n storage);
// the key-block-major pass walks, for each key block, the query blocks that
// kept it (a transposed index built first), so no output is accumulated by
// atomics and every sum runs in a fixed order.
//
// Threads: four per row (dQ pass) or per key (dK/dV pass), each holding 32
// of the 128 channels; dot products are finished with two shuffles.
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace bwd {

constexpr int kD = 128;
constexpr int kRows = 64;          // rows (dQ pass) or keys (dK/dV pass) per CTA
constexpr int kThreads = 4 * kRows;

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&x)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint4 w = __ldg(p + e);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[8 * e + 2 * i] = __uint_as_float(ws[i] << 16);
      x[8 * e + 2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
    }
  }
}

// D_t = dO_t . O_t, one warp per row.
__global__ void rowdot_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                              int64_t rows, float* __restrict__ D) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const __nv_bfloat162 a0 = reinterpret_cast<const __nv_bfloat162*>(o + r * kD)[lane * 2];
  const __nv_bfloat162 a1 = reinterpret_cast<const __nv_bfloat162*>(o + r * kD)[lane * 2 + 1];
  const __nv_bfloat162 b0 = reinterpret_cast<const __nv_bfloat162*>(d_o + r * kD)[lane * 2];
  const __nv_bfloat162 b1 = reinterpret_cast<const __nv_bfloat162*>(d_o + r * kD)[lane * 2 + 1];
  const float2 fa0 = __bfloat1622float2(a0), fa1 = __bfloat1622float2(a1);
  const float2 fb0 = __bfloat1622float2(b0), fb1 = __bfloat1622float2(b1);
  float acc = fa0.x * fb0.x + fa0.y * fb0.y + fa1.x * fb1.x + fa1.y * fb1.y;
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) D[r] = acc;
}

// Per unit (b, g, i): its kept list (validated as the forward does) and, per
// kept slot, log g (natural log; 0 when ungated).  One warp per unit.
__global__ void gate_kernel(const int* __restrict__ idx, int idx_stride, const float* __restrict__ sel, int nb,
                            int64_t units, int* __restrict__ lists, int* __restrict__ counts,
                            float* __restrict__ logg, uint32_t* __restrict__ status) {
  const int64_t u = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= units) return;
  const int i = static_cast<int>(u % nb);
  const int* src = idx + u * idx_stride;
  int* dst = lists + u * idx_stride;
  int count = 0, prev = -1;
  for (int base = 0; base < idx_stride; base += 32) {
    const int t = base + lane;
    const int j = (t < idx_stride) ? src[t] : -1;
    const unsigned neg = __ballot_sync(0xffffffffu, j < 0);
    const int lim = neg ? __ffs(neg) - 1 : 32;
    int jprev = __shfl_up_sync(0xffffffffu, j, 1);
    if (lane == 0) jprev = prev;
    const bool in = lane < lim;
    const bool ok = in && j <= i && j > jprev;
    if (in && !ok) atomicOr(status, BSA_DEV_BAD_INDEX);
    const unsigned okm = __ballot_sync(0xffffffffu, ok);
    if (ok) dst[count + __popc(okm & ((1u << lane) - 1u))] = j;
    count += __popc(okm);
    prev = __shfl_sync(0xffffffffu, j, 31);
    if (neg) break;
  }
  __syncwarp();
  float* lg = logg + u * idx_stride;
  if (sel != nullptr && count > 0) {
    const float* srow = sel + u * nb;
    float mx = -INFINITY;
    for (int t = lane; t < count; t += 32) mx = fmaxf(mx, srow[dst[t]]);
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
    if (mx > -INFINITY)
      for (int t = lane; t < count; t += 32) sum += expf(srow[dst[t]] - mx);
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse_s = (mx > -INFINITY) ? mx + logf(sum) : 0.0f;
    for (int t = lane; t < count; t += 32) lg[t] = (mx > -INFINITY) ? srow[dst[t]] - lse_s : 0.0f;
  } else {
    for (int t = lane; t < count; t += 32) lg[t] = 0.0f;
  }
  if (lane == 0) counts[u] = count;
}

// For each (b, g): the query blocks i (ascending) that kept each key block j,
// with the slot of j in i's list.  One thread per (b, g), sequential, so the
// lists come out in a fixed order.
__global__ void transpose_kernel(const int* __restrict__ lists, const int* __restrict__ counts, int idx_stride,
                                 int nb, int bgs, int* __restrict__ toff, int2* __restrict__ tlist) {
  const int bg = blockIdx.x * blockDim.x + threadIdx.x;
  if (bg >= bgs) return;
  int* off = toff + static_cast<int64_t>(bg) * (nb + 1);
  const int64_t ubase = static_cast<int64_t>(bg) * nb;
  for (int j = 0; j <= nb; ++j) off[j] = 0;
  for (int i = 0; i < nb; ++i) {
    const int* l = lists + (ubase + i) * idx_stride;
    for (int s = 0; s < counts[ubase + i]; ++s) ++off[l[s] + 1];
  }
  for (int j = 0; j < nb; ++j) off[j + 1] += off[j];
  // fill, then restore the starts (each count was used as a cursor)
  int2* tl = tlist + ubase * idx_stride;
  for (int i = 0; i < nb; ++i) {
    const int* l = lists + (ubase + i) * idx_stride;
    for (int s = 0; s < counts[ubase + i]; ++s) tl[off[l[s]]++] = make_int2(i, s);
  }
  for (int j = nb; j > 0; --j) off[j] = off[j - 1];
  off[0] = 0;
}

struct Params {
  const __nv_bfloat16 *q, *k, *v, *d_o;
  const float *lse, *D, *logg;
  const int *lists, *counts, *toff;
  const int2* tlist;
  int B, Hq, Hkv, N, nb, G, bs, idx_stride, chunks;   // chunks: 64-row chunks per unit
  float scale;
  float *dq, *dk, *dv, *dlogg_part;                    // dlogg_part [units][idx_stride][chunks]
};

// dQ pass.  CTA = (unit, chunk of 64 of its G*bs stacked rows); thread
// (row, quarter).  Every kept block of the unit in list order; its keys are
// staged in shared memory as fp32, 64 at a time.
constexpr size_t kTileSmem = 2 * static_cast<size_t>(kRows) * (kD + 4) * sizeof(float);

__global__ void __launch_bounds__(kThreads) dq_kernel(const Params p) {
  extern __shared__ __align__(16) float dq_sm[];
  float (*ks)[kD + 4] = reinterpret_cast<float (*)[kD + 4]>(dq_sm);
  float (*vs)[kD + 4] = reinterpret_cast<float (*)[kD + 4]>(dq_sm + kRows * (kD + 4));
  __shared__ float red[kThreads / 32];
  const int64_t unit = blockIdx.x / p.chunks;
  const int chunk = static_cast<int>(blockIdx.x % p.chunks);
  const int64_t bg = unit / p.nb;
  const int i = static_cast<int>(unit % p.nb);
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int rl = threadIdx.x >> 2, qt = threadIdx.x & 3;
  const int R = chunk * kRows + rl;
  const bool valid = R < p.G * p.bs;
  const int h = g * p.G + (valid ? R / p.bs : 0);
  const int t = i * p.bs + R % p.bs;
  const int64_t row = (static_cast<int64_t>(b) * p.Hq + h) * p.N + t;
  float qv[32], dov[32], dq[32];
  if (valid) {
    load_bf16x32(p.q + row * kD + qt * 32, qv);
    load_bf16x32(p.d_o + row * kD + qt * 32, dov);
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) qv[c] = dov[c] = 0.0f;
  }
#pragma unroll
  for (int c = 0; c < 32; ++c) dq[c] = 0.0f;
  const float lse = valid ? p.lse[row] : -INFINITY;
  const float Dt = valid ? p.D[row] : 0.0f;
  const bool live = valid && lse > -INFINITY;
  const int count = p.counts[unit];
  const int* list = p.lists + unit * p.idx_stride;
  const float* lg = p.logg + unit * p.idx_stride;
  const int64_t kvbase = bg * static_cast<int64_t>(p.N);
  for (int s = 0; s < count; ++s) {
    const int j = list[s];
    const float bias = lg[s];
    float dlsum = 0.0f;
    for (int k0 = 0; k0 < p.bs; k0 += kRows) {
      __syncthreads();
      for (int e = threadIdx.x; e < kRows * (kD / 8); e += kThreads) {
        const int kr = e >> 4, c8 = e & 15;
        const int64_t src = (kvbase + j * p.bs + k0 + kr) * kD + c8 * 8;
        const uint4 wk = __ldg(reinterpret_cast<const uint4*>(p.k + src));
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(p.v + src));
        const uint32_t kk[4] = {wk.x, wk.y, wk.z, wk.w}, vv[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          ks[kr][c8 * 8 + 2 * x] = __uint_as_float(kk[x] << 16);
          ks[kr][c8 * 8 + 2 * x + 1] = __uint_as_float(kk[x] & 0xFFFF0000u);
          vs[kr][c8 * 8 + 2 * x] = __uint_as_float(vv[x] << 16);
          vs[kr][c8 * 8 + 2 * x + 1] = __uint_as_float(vv[x] & 0xFFFF0000u);
        }
      }
      __syncthreads();
      const int kend = (j == i) ? min(kRows, t - (j * p.bs + k0) + 1) : kRows;   // causal inside block i
      for (int u = 0; u < kRows; ++u) {
        const float* kr = &ks[u][qt * 32];
        const float* vr = &vs[u][qt * 32];
        float sdot = 0.0f, pdot = 0.0f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sdot = fmaf(qv[c], kr[c], sdot);
          pdot = fmaf(dov[c], vr[c], pdot);
        }
        sdot = quad_sum(sdot);
        pdot = quad_sum(pdot);
        const bool on = live && u < kend;
        const float P = on ? __expf(fmaf(sdot, p.scale, bias) - lse) : 0.0f;
        const float dl = P * (pdot - Dt);
        dlsum += dl;
        const float f = dl * p.scale;
#pragma unroll
        for (int c = 0; c < 32; ++c) dq[c] = fmaf(f, kr[c], dq[c]);
      }
    }
    // the chunk's rows' share of dlogg for this slot (quarter 0 of each row counts it)
    float x = (qt == 0) ? dlsum : 0.0f;
#pragma unroll
    for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
      float tot = 0.0f;
      for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
      p.dlogg_part[(unit * p.idx_stride + s) * p.chunks + chunk] = tot;
    }
  }
  if (valid) {
    float* dst = p.dq + row * kD + qt * 32;
#pragma unroll
    for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(dq[c], dq[c + 1], dq[c + 2], dq[c + 3]);
  }
}

// dK / dV pass.  CTA = (b, g, key block j, chunk of 64 of its keys); thread
// (key, quarter).  Every query block i that kept j (ascending), every head of
// the group, its rows staged 64 at a time.
__global__ void __launch_bounds__(kThreads) dkv_kernel(const Params p) {
  extern __shared__ __align__(16) float dkv_sm[];
  float (*qs)[kD + 4] = reinterpret_cast<float (*)[kD + 4]>(dkv_sm);
  float (*dos)[kD + 4] = reinterpret_cast<float (*)[kD + 4]>(dkv_sm + kRows * (kD + 4));
  __shared__ float ls[kRows], dsh[kRows];
  const int kchunks = p.bs / kRows;
  const int64_t blk = blockIdx.x / kchunks;           // (bg, j)
  const int k0 = static_cast<int>(blockIdx.x % kchunks) * kRows;
  const int64_t bg = blk / p.nb;
  const int j = static_cast<int>(blk % p.nb);
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int kl = threadIdx.x >> 2, qt = threadIdx.x & 3;
  const int u = j * p.bs + k0 + kl;                    // this thread's key position
  const int64_t krow = bg * static_cast<int64_t>(p.N) + u;
  float kv[32], vv[32], dk[32], dv[32];
  load_bf16x32(p.k + krow * kD + qt * 32, kv);
  load_bf16x32(p.v + krow * kD + qt * 32, vv);
#pragma unroll
  for (int c = 0; c < 32; ++c) dk[c] = dv[c] = 0.0f;
  const int* off = p.toff + bg * (p.nb + 1);
  const int2* tl = p.tlist + bg * static_cast<int64_t>(p.nb) * p.idx_stride;
  for (int e = off[j]; e < off[j + 1]; ++e) {
    const int i = tl[e].x, s = tl[e].y;
    const float bias = p.logg[(bg * p.nb + i) * p.idx_stride + s];
    for (int hh = 0; hh < p.G; ++hh) {
      const int h = g * p.G + hh;
      for (int r0 = 0; r0 < p.bs; r0 += kRows) {
        const int64_t rbase = (static_cast<int64_t>(b) * p.Hq + h) * p.N + i * p.bs + r0;
        __syncthreads();
        for (int x = threadIdx.x; x < kRows * (kD / 8); x += kThreads) {
          const int rr = x >> 4, c8 = x & 15;
          const int64_t src = (rbase + rr) * kD + c8 * 8;
          const uint4 wq = __ldg(reinterpret_cast<const uint4*>(p.q + src));
          const uint4 wd = __ldg(reinterpret_cast<const uint4*>(p.d_o + src));
          const uint32_t a[4] = {wq.x, wq.y, wq.z, wq.w}, d2[4] = {wd.x, wd.y, wd.z, wd.w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            qs[rr][c8 * 8 + 2 * y] = __uint_as_float(a[y] << 16);
            qs[rr][c8 * 8 + 2 * y + 1] = __uint_as_float(a[y] & 0xFFFF0000u);
            dos[rr][c8 * 8 + 2 * y] = __uint_as_float(d2[y] << 16);
            dos[rr][c8 * 8 + 2 * y + 1] = __uint_as_float(d2[y] & 0xFFFF0000u);
          }
        }
        if (threadIdx.x < kRows) {
          ls[threadIdx.x] = p.lse[rbase + threadIdx.x];
          dsh[threadIdx.x] = p.D[rbase + threadIdx.x];
        }
        __syncthreads();
        for (int rr = 0; rr < kRows; ++rr) {
          const float* qr = &qs[rr][qt * 32];
          const float* dr = &dos[rr][qt * 32];
          float sdot = 0.0f, pdot = 0.0f;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            sdot = fmaf(qr[c], kv[c], sdot);
            pdot = fmaf(dr[c], vv[c], pdot);
          }
          sdot = quad_sum(sdot);
          pdot = quad_sum(pdot);
          const int t = i * p.bs + r0 + rr;
          const float lse = ls[rr];
          const bool on = lse > -INFINITY && (i != j || u <= t);
          const float P = on ? __expf(fmaf(sdot, p.scale, bias) - lse) : 0.0f;
          const float f = P * (pdot - dsh[rr]) * p.scale;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            dv[c] = fmaf(P, dr[c], dv[c]);
            dk[c] = fmaf(f, qr[c], dk[c]);
          }
        }
      }
    }
  }
  float* dkd = p.dk + krow * kD + qt * 32;
  float* dvd = p.dv + krow * kD + qt * 32;
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    *reinterpret_cast<float4*>(dkd + c) = make_float4(dk[c], dk[c + 1], dk[c + 2], dk[c + 3]);
    *reinterpret_cast<float4*>(dvd + c) = make_float4(dv[c], dv[c + 1], dv[c + 2], dv[c + 3]);
  }
}

// dsel per unit: dlogg_l (the chunks' partials summed in order) minus
// g_l * (sum over the kept blocks of dlogg_j); zero off the kept blocks.
// One warp per unit.
__global__ void dsel_kernel(const Params p, int64_t units, float* __restrict__ dsel) {
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (unit >= units) return;
  float* row = dsel + unit * p.nb;
  for (int jj = lane; jj < p.nb; jj += 32) row[jj] = 0.0f;
  __syncwarp();
  const int count = p.counts[unit];
  const int* list = p.lists + unit * p.idx_stride;
  float tot = 0.0f;
  for (int s = lane; s < count; s += 32) {
    float x = 0.0f;
    for (int c = 0; c < p.chunks; ++c) x += p.dlogg_part[(unit * p.idx_stride + s) * p.chunks + c];
    tot += x;
  }
  for (int off = 16; off; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
  for (int s = lane; s < count; s += 32) {
    float x = 0.0f;
    for (int c = 0; c < p.chunks; ++c) x += p.dlogg_part[(unit * p.idx_stride + s) * p.chunks + c];
    row[list[s]] = x - __expf(p.logg[unit * p.idx_stride + s]) * tot;
  }
}

}  // namespace bwd

size_t attn_bwd_workspace(int B, int Hq, int Hkv, int N, int bs, int idx_stride) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int nb = N / bs;
  const int64_t units = static_cast<int64_t>(B) * Hkv * nb;
  const int chunks = (Hq / Hkv * bs + bwd::kRows - 1) / bwd::kRows;
  size_t off = 0;
  off = a256(off + static_cast<size_t>(B) * Hq * N * sizeof(float));            // D
  off = a256(off + units * idx_stride * sizeof(float));                          // logg
  off = a256(off + units * idx_stride * sizeof(int));                            // lists
  off = a256(off + units * sizeof(int));                                         // counts
  off = a256(off + static_cast<size_t>(B) * Hkv * (nb + 1) * sizeof(int));       // toff
  off = a256(off + units * idx_stride * sizeof(int2));                           // tlist
  off = a256(off + units * idx_stride * chunks * sizeof(float));                 // dlogg partials
  return off;
}

cudaError_t launch_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* d_o, const int* idx, int idx_stride, const float* sel, float scale, int B,
                            int Hq, int Hkv, int N, int bs, float* dq, float* dk, float* dv, float* dsel,
                            void* workspace, uint32_t* status, cudaStream_t st) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int nb = N / bs;
  const int64_t units = static_cast<int64_t>(B) * Hkv * nb;
  const int64_t rows = static_cast<int64_t>(B) * Hq * N;
  bwd::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.d_o = static_cast<const __nv_bfloat16*>(d_o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.nb = nb;
  p.G = Hq / Hkv;
  p.bs = bs;
  p.idx_stride = idx_stride;
  p.chunks = (p.G * bs + bwd::kRows - 1) / bwd::kRows;
  p.scale = scale;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  char* ws = static_cast<char*>(workspace);
  size_t off = 0;
  float* D = reinterpret_cast<float*>(ws + off);
  off = a256(off + rows * sizeof(float));
  float* logg = reinterpret_cast<float*>(ws + off);
  off = a256(off + units * idx_stride * sizeof(float));
  int* lists = reinterpret_cast<int*>(ws + off);
  off = a256(off + units * idx_stride * sizeof(int));
  int* counts = reinterpret_cast<int*>(ws + off);
  off = a256(off + units * sizeof(int));
  int* toff = reinterpret_cast<int*>(ws + off);
  off = a256(off + static_cast<size_t>(B) * Hkv * (nb + 1) * sizeof(int));
  int2* tlist = reinterpret_cast<int2*>(ws + off);
  off = a256(off + units * idx_stride * sizeof(int2));
  p.dlogg_part = reinterpret_cast<float*>(ws + off);
  p.D = D;
  p.logg = logg;
  p.lists = lists;
  p.counts = counts;
  p.toff = toff;
  p.tlist = tlist;
  bwd::rowdot_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                                             p.d_o, rows, D);
  bwd::gate_kernel<<<static_cast<unsigned>((units + 7) / 8), 256, 0, st>>>(idx, idx_stride, sel, nb, units, lists,
                                                                           counts, logg, status);
  const int bgs = B * Hkv;
  bwd::transpose_kernel<<<(bgs + 63) / 64, 64, 0, st>>>(lists, counts, idx_stride, nb, bgs, toff, tlist);
  cudaError_t e = ensure_dynamic_smem<bwd::dq_kernel>(bwd::kTileSmem);
  if (e == cudaSuccess) e = ensure_dynamic_smem<bwd::dkv_kernel>(bwd::kTileSmem);
  if (e != cudaSuccess) return e;
  bwd::dq_kernel<<<static_cast<unsigned>(units * p.chunks), bwd::kThreads, bwd::kTileSmem, st>>>(p);
  bwd::dkv_kernel<<<static_cast<unsigned>(static_cast<int64_t>(bgs) * nb * (bs / bwd::kRows)), bwd::kThreads,
                    bwd::kTileSmem, st>>>(p);
  if (dsel != nullptr)
    bwd::dsel_kernel<<<static_cast<unsigned>((units + 7) / 8), 256, 0, st>>>(p, units, dsel);
  return cudaGetLastError();
}

}  // namespace bsa
