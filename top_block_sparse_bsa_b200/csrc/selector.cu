// selector.cu -- the cheap selector of query-aware block-sparse attention:
// block pooling, block / gist scoring and hard top-k selection.
//
// Sources: "稀疏注意力" tutorial §4.5 (a block is a run of consecutive tokens)
// and §4.6 (coarse block scoring avoids the full QK^T); SAS page, 核心模块 1
// (a continuous score per context unit) and 推理 paragraph (each query keeps
// its k best units, the current block always kept); SSA page, 推理时的关键模块
// 1-2 (score the query against every gist, expand the top-k chunks, each
// query head choosing its own chunks under GQA).
//
// Arithmetic contract (kept identical on purpose to the plain definition, so
// selected indices are reproducible bit for bit): pooled means are fp32 sums
// in a fixed order (heads ascending, then tokens ascending) followed by one
// IEEE division; a score is an fp32 dot product over the channel index
// ascending with each product and each sum rounded separately (no FMA),
// then one multiply by fp32(1/sqrt(d)).  These kernels are bandwidth-bound,
// so the sequential order costs nothing that matters.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace bsa {

// ------------------------------------------------------------------ pooling
// One group of 8 channels per thread, 16-byte loads along d, every thread
// summing its channels over the unit's rows in order.
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// unit u = (b, g, j): rows base + hh*N + t for hh < heads_sum, t < bs,
// base = ((b*Hsrc + g*heads_sum)*N + j*bs).  out[u][c] = sum / (heads_sum*bs).
// One thread per (unit, 8-channel group).  Rows are read in batches of RB
// rows whose loads are all issued before the batch is summed in order, so a
// thread has RB 16-byte (bf16) loads in flight instead of one.
struct PoolJob {
  const void* src;
  int Hsrc, heads_sum;
  float* out;
};

template <typename T, int RB>
__global__ void __launch_bounds__(256) pool_kernel(PoolJob job0, PoolJob job1, int B, int Hgroups, int N, int d,
                                                   int bs) {
  const PoolJob job = blockIdx.y ? job1 : job0;
  if (job.src == nullptr) return;
  const T* src = static_cast<const T*>(job.src);
  const int lanes_per_unit = d / 8;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t unit = gtid / lanes_per_unit;
  const int cg = static_cast<int>(gtid % lanes_per_unit);
  const int nb = N / bs;
  const int64_t units = static_cast<int64_t>(B) * Hgroups * nb;
  if (unit >= units) return;
  const int64_t b = unit / (static_cast<int64_t>(Hgroups) * nb);
  const int64_t g = (unit / nb) % Hgroups;
  const int64_t j = unit % nb;
  const int64_t base = ((b * job.Hsrc + g * job.heads_sum) * N + j * bs) * d + cg * 8;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  for (int hh = 0; hh < job.heads_sum; ++hh) {
    const T* p = src + base + static_cast<int64_t>(hh) * N * d;
    for (int t0 = 0; t0 < bs; t0 += RB) {
      float x[RB][8];
#pragma unroll
      for (int t = 0; t < RB; ++t) Vec8<T>::load(p + static_cast<int64_t>(t0 + t) * d, x[t]);
#pragma unroll
      for (int t = 0; t < RB; ++t)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = __fadd_rn(acc[c], x[t][c]);
    }
  }
  const float div = static_cast<float>(job.heads_sum * bs);
  float* o = job.out + unit * d + cg * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) o[c] = __fdiv_rn(acc[c], div);
}

static cudaError_t launch_pool_jobs(const PoolJob& j0, const PoolJob& j1, bool bf16, int B, int Hgroups, int N, int d,
                                    int bs, cudaStream_t st) {
  const int64_t threads = static_cast<int64_t>(B) * Hgroups * (N / bs) * (d / 8);
  const int tpb = 256;
  const dim3 grid(static_cast<unsigned>((threads + tpb - 1) / tpb), j1.src ? 2u : 1u);
  if (bf16) {
    if (bs % 32 == 0)
      pool_kernel<__nv_bfloat16, 32><<<grid, tpb, 0, st>>>(j0, j1, B, Hgroups, N, d, bs);
    else
      pool_kernel<__nv_bfloat16, 1><<<grid, tpb, 0, st>>>(j0, j1, B, Hgroups, N, d, bs);
  } else {
    if (bs % 16 == 0)
      pool_kernel<float, 16><<<grid, tpb, 0, st>>>(j0, j1, B, Hgroups, N, d, bs);
    else
      pool_kernel<float, 1><<<grid, tpb, 0, st>>>(j0, j1, B, Hgroups, N, d, bs);
  }
  return cudaGetLastError();
}

// Streamed variant (persistent): a producer thread copies each unit's rows
// (heads_sum runs of bs*d contiguous elements) into kPoolStages shared-memory
// buffers with bulk copies, a chunk of whole runs per buffer, while 128
// threads sum earlier chunks, column c by thread c, rows in the fixed order
// (head, then row), the running sum carried from one chunk of a unit to the
// next.  Units of the query job come first, then those of the key job; a key
// unit is a single run and consecutive key units are contiguous in memory, so
// a buffer takes several of them in one copy, and their column sums (separate
// chains) advance together.  A column's sum over a unit is one dependent chain
// of additions, so the kernel runs two CTAs per SM with 32 KB chunks when a
// run fits (two summing warps per SM sub-partition), one with 64 KB chunks
// otherwise.
constexpr int kPoolStreamBytes = 64 * 1024;   // largest chunk
constexpr int kPoolSmallChunk = 32 * 1024;
constexpr int kPoolStages = 3;
constexpr int kPoolMaxGroup = 4;              // key units per chunk: 64 KB / 16 KB runs

template <typename T>
__global__ void __launch_bounds__(160, 2) pool_stream_kernel(PoolJob jq, PoolJob jk, int B, int Hgroups, int N, int d,
                                                             int bs, int chunk_bytes, uint32_t* status) {
  extern __shared__ uint8_t psmem_raw[];
  uint8_t* psmem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(psmem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t bars[2 * kPoolStages];
  __shared__ int abort_flag;
  const uint32_t sb = smem_u32(psmem);
  auto bar = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };
  const int nb = N / bs;
  const int64_t units_per_job = static_cast<int64_t>(B) * Hgroups * nb;
  const uint32_t run = static_cast<uint32_t>(bs) * d * sizeof(T);       // one head's rows of a unit
  const int runs_per_chunk = static_cast<int>(chunk_bytes / run);   // 1 .. kPoolMaxGroup (checked by the launcher)
  // key items: kgrp consecutive key units each (single-run units stored back
  // to back: unit u's rows start at u * bs * d)
  const int kgrp = (jk.src != nullptr && jk.heads_sum == 1 && jk.Hsrc == Hgroups) ? runs_per_chunk : 1;
  const int64_t kitems = jk.src ? (units_per_job + kgrp - 1) / kgrp : 0;
  const int64_t units = units_per_job + kitems;   // work items
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPoolStages; ++i) {
      mbar_init(bar(i), 1);
      mbar_init(bar(kPoolStages + i), 128);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  const int warp = threadIdx.x >> 5;
  if (warp == 4) {
    if ((threadIdx.x & 31) == 0) {
      int k = 0;   // chunks issued
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const bool isk = u >= units_per_job;
        if (isk && kgrp > 1) {
          const int64_t u0 = (u - units_per_job) * kgrp;
          const int nr = static_cast<int>(min(static_cast<int64_t>(kgrp), units_per_job - u0));
          const int buf = k % kPoolStages, use = k / kPoolStages;
          if (k >= kPoolStages && !(ok = mbar_wait(bar(kPoolStages + buf), (use - 1) & 1, ab, status))) break;
          mbar_arrive_expect_tx(bar(buf), run * nr);
          bulk_load(sb + buf * chunk_bytes, static_cast<const T*>(jk.src) + u0 * bs * d, run * nr, bar(buf));
          ++k;
          continue;
        }
        const PoolJob& job = isk ? jk : jq;
        const int64_t unit = isk ? u - units_per_job : u;
        const int64_t b = unit / (static_cast<int64_t>(Hgroups) * nb);
        const int64_t g = (unit / nb) % Hgroups;
        const int64_t j = unit % nb;
        const T* src = static_cast<const T*>(job.src);
        for (int h0 = 0; h0 < job.heads_sum; h0 += runs_per_chunk, ++k) {
          const int nr = min(runs_per_chunk, job.heads_sum - h0);
          const int buf = k % kPoolStages, use = k / kPoolStages;
          if (k >= kPoolStages && !(ok = mbar_wait(bar(kPoolStages + buf), (use - 1) & 1, ab, status))) break;
          mbar_arrive_expect_tx(bar(buf), run * nr);
          for (int hh = h0; hh < h0 + nr; ++hh)
            bulk_load(sb + buf * chunk_bytes + (hh - h0) * run,
                      src + ((b * job.Hsrc + g * job.heads_sum + hh) * static_cast<int64_t>(N) + j * bs) * d, run,
                      bar(buf));
        }
      }
      if (*ab) {   // let the copies still in flight land before the CTA exits
        for (int q = k > kPoolStages ? k - kPoolStages : 0; q < k; ++q)
          mbar_drain(bar(q % kPoolStages), (q / kPoolStages) & 1);
      }
    }
  } else {
    const int c = threadIdx.x;   // column
    int k = 0;   // chunks consumed
    bool ok = true;
    for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
      const bool isk = u >= units_per_job;
      if (isk && kgrp > 1) {
        const int64_t u0 = (u - units_per_job) * kgrp;
        const int nr = static_cast<int>(min(static_cast<int64_t>(kgrp), units_per_job - u0));
        const int buf = k % kPoolStages, use = k / kPoolStages;
        if (!(ok = mbar_wait(bar(buf), use & 1, ab, status))) break;
        const T* sv = reinterpret_cast<const T*>(psmem + buf * chunk_bytes);
        if (c < d) {
          // the nr units' column sums advance together (independent chains),
          // each over its own rows in ascending order
          float acc[kPoolMaxGroup] = {0.0f, 0.0f, 0.0f, 0.0f};
          for (int r = 0; r < bs; r += 16) {   // bs is a multiple of 16
#pragma unroll
            for (int x = 0; x < kPoolMaxGroup; ++x) {
              if (x < nr) {
                float xv[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) xv[t] = static_cast<float>(sv[(x * bs + r + t) * d + c]);
#pragma unroll
                for (int t = 0; t < 16; ++t) acc[x] = __fadd_rn(acc[x], xv[t]);
              }
            }
          }
#pragma unroll
          for (int x = 0; x < kPoolMaxGroup; ++x)
            if (x < nr) jk.out[(u0 + x) * d + c] = __fdiv_rn(acc[x], static_cast<float>(bs));
        }
        mbar_arrive(bar(kPoolStages + buf));
        ++k;
        continue;
      }
      const PoolJob& job = isk ? jk : jq;
      const int64_t unit = isk ? u - units_per_job : u;
      float acc = 0.0f;
      for (int h0 = 0; h0 < job.heads_sum; h0 += runs_per_chunk, ++k) {
        const int nr = min(runs_per_chunk, job.heads_sum - h0);
        const int buf = k % kPoolStages, use = k / kPoolStages;
        if (!(ok = mbar_wait(bar(buf), use & 1, ab, status))) break;
        const T* sv = reinterpret_cast<const T*>(psmem + buf * chunk_bytes);
        const int rows = nr * bs;   // a multiple of 16
        if (c < d) {
          for (int r = 0; r < rows; r += 16) {
            float x[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) x[t] = static_cast<float>(sv[(r + t) * d + c]);
#pragma unroll
            for (int t = 0; t < 16; ++t) acc = __fadd_rn(acc, x[t]);
          }
        }
        mbar_arrive(bar(kPoolStages + buf));
      }
      if (!ok) break;
      if (c < d) job.out[unit * d + c] = __fdiv_rn(acc, static_cast<float>(job.heads_sum * bs));
    }
  }
  __syncthreads();
}

cudaError_t launch_pool(const void* src, bool bf16, int B, int Hsrc, int Hgroups, int heads_sum, int N,
                        int d, int bs, float* out, cudaStream_t st) {
  const PoolJob j0{src, Hsrc, heads_sum, out};
  const PoolJob none{nullptr, 0, 0, nullptr};
  return launch_pool_jobs(j0, none, bf16, B, Hgroups, N, d, bs, st);
}

// Prefill: grouped queries (heads_sum G) and keys (heads_sum 1) in one launch
// of the streamed kernel when one head's rows of a unit fit a buffer and
// d <= 128.
cudaError_t launch_pool_prefill(const void* q, const void* k, bool bf16, int B, int Hq, int Hkv, int N, int d,
                                int bs, float* qbar, float* kbar, int num_sms, uint32_t* status, cudaStream_t st) {
  const PoolJob jq{q, Hq, Hq / Hkv, qbar};
  const PoolJob jk{k, Hkv, 1, kbar};
  const size_t esize = bf16 ? 2 : 4;
  const size_t run_bytes = static_cast<size_t>(bs) * d * esize;
  if (run_bytes > kPoolStreamBytes || d > 128 || bs % 16 != 0 || run_bytes % 16 != 0)
    return launch_pool_jobs(jq, jk, bf16, B, Hkv, N, d, bs, st);
  // a chunk holds 1 .. kPoolMaxGroup runs: runs of 8 KB to 32 KB take two
  // CTAs per SM with 32 KB chunks, runs above 32 KB one CTA per SM with 64 KB
  // chunks, and runs below 8 KB go to pool_kernel
  const bool small = run_bytes <= kPoolSmallChunk && kPoolSmallChunk / run_bytes <= kPoolMaxGroup;
  const int chunk = small ? kPoolSmallChunk : kPoolStreamBytes;
  if (static_cast<size_t>(chunk) / run_bytes > kPoolMaxGroup) return launch_pool_jobs(jq, jk, bf16, B, Hkv, N, d, bs, st);
  const size_t smem = static_cast<size_t>(kPoolStages) * chunk + 128;
  const int64_t units = 2ll * B * Hkv * (N / bs);
  const int64_t ctas = static_cast<int64_t>(num_sms) * (small ? 2 : 1);
  const unsigned grid = static_cast<unsigned>(units < ctas ? units : ctas);
  cudaError_t e;
  if (bf16) {
    e = ensure_dynamic_smem<pool_stream_kernel<__nv_bfloat16>>(smem);
    if (e != cudaSuccess) return e;
    pool_stream_kernel<__nv_bfloat16><<<grid, 160, smem, st>>>(jq, jk, B, Hkv, N, d, bs, chunk, status);
  } else {
    e = ensure_dynamic_smem<pool_stream_kernel<float>>(smem);
    if (e != cudaSuccess) return e;
    pool_stream_kernel<float><<<grid, 160, smem, st>>>(jq, jk, B, Hkv, N, d, bs, chunk, status);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ scores
__device__ __forceinline__ float dot_fixed_order(const float* a, const float* b, int d, int bstride) {
  float acc = 0.0f;
  for (int c = 0; c < d; ++c) acc = __fadd_rn(acc, __fmul_rn(a[c], b[c * bstride]));
  return acc;
}

// Prefill: one 64x64 (i, j) tile per CTA of 256 threads; each thread owns a
// 4x4 micro-tile (rows ty + 16a, columns tx + 16b), i.e. 16 independent
// fixed-order dot products advanced together over the channel index.  Rows
// of qbar/kbar are staged in shared memory with a pitch of d+4 floats.
constexpr int kScoreTile = 64;

__global__ void __launch_bounds__(256) score_prefill_kernel(const float* __restrict__ qbar,
                                                            const float* __restrict__ kbar, int nb, int d,
                                                            float scale, float* __restrict__ s) {
  extern __shared__ __align__(16) float sm[];
  const int pitch = d + 4;   // 16-byte aligned rows for the asynchronous copies
  float* qs = sm;
  float* ks = sm + kScoreTile * pitch;
  const int ti = blockIdx.y, tj = blockIdx.x;
  const int64_t bg = blockIdx.z;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16
  const int i0 = ti * kScoreTile, j0 = tj * kScoreTile;
  float* srow = s + bg * nb * static_cast<int64_t>(nb);
  if (j0 > i0 + kScoreTile - 1) {   // tile entirely above the diagonal
    for (int e = threadIdx.x; e < kScoreTile * kScoreTile; e += blockDim.x) {
      const int i = i0 + e / kScoreTile, j = j0 + e % kScoreTile;
      if (i < nb && j < nb) srow[static_cast<int64_t>(i) * nb + j] = -INFINITY;
    }
    return;
  }
  {
    // 64 rows x d floats per matrix with 16-byte asynchronous copies (every
    // copy of a thread in flight at once); rows past nb are zero-filled
    const int q4 = d / 4;
    for (int e = threadIdx.x; e < kScoreTile * q4; e += blockDim.x) {
      const int r = e / q4, c4 = e % q4;
      float* qd = qs + r * pitch + c4 * 4;
      float* kd = ks + r * pitch + c4 * 4;
      if (i0 + r < nb) cp_async16(smem_u32(qd), qbar + (bg * nb + i0 + r) * d + c4 * 4);
      else *reinterpret_cast<float4*>(qd) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < nb) cp_async16(smem_u32(kd), kbar + (bg * nb + j0 + r) * d + c4 * 4);
      else *reinterpret_cast<float4*>(kd) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_wait_all();
  }
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
  for (int c = 0; c < d; ++c) {
    float qv[4], kv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) qv[a] = qs[(ty + 16 * a) * pitch + c];
#pragma unroll
    for (int b = 0; b < 4; ++b) kv[b] = ks[(tx + 16 * b) * pitch + c];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(qv[a], kv[b]));
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= nb) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx + 16 * b;
      if (j >= nb) continue;
      srow[static_cast<int64_t>(i) * nb + j] = (j <= i) ? __fmul_rn(acc[a][b], scale) : -INFINITY;
    }
  }
}

cudaError_t launch_score_prefill(const float* qbar, const float* kbar, int B, int Hkv, int nb, int d,
                                 float scale, float* s, cudaStream_t st) {
  if (d % 4 != 0 || d > 128) return cudaErrorInvalidValue;
  dim3 grid((nb + kScoreTile - 1) / kScoreTile, (nb + kScoreTile - 1) / kScoreTile, B * Hkv);
  const size_t smem = 2 * kScoreTile * (d + 4) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_dynamic_smem<score_prefill_kernel>(smem);
    if (e != cudaSuccess) return e;
  }
  score_prefill_kernel<<<grid, 256, smem, st>>>(qbar, kbar, nb, d, scale, s);
  return cudaGetLastError();
}

// Decode: grid (tiles of 128 blocks, B*Hkv); one thread per block.  The
// CTA's 128 pooled-key rows are copied into shared memory with coalesced
// 16-byte cp.async (a warp moves 512 contiguous bytes per instruction) into
// rows padded to d+4 floats, so that the per-thread float4 reads of eight
// consecutive rows fall into distinct banks; each thread then runs the
// fixed-order dot product of its row.  The group query mean is formed in
// fixed order (heads ascending) per CTA.
template <typename T, int D>
__global__ void __launch_bounds__(128) score_decode_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                           int Hq, int Hkv, int nb, float scale,
                                                           float* __restrict__ s, float* __restrict__ qbar_out) {
  constexpr int kPitch = D + 4;
  constexpr int kChunks = D / 4;   // 16-byte chunks per row
  extern __shared__ __align__(16) float sm_dec[];
  float* ks = sm_dec;                 // [128][kPitch]
  float* qm = sm_dec + 128 * kPitch;  // [D]
  const int64_t bg = blockIdx.y;
  const int64_t b = bg / Hkv, g = bg % Hkv;
  const int G = Hq / Hkv;
  const int j0 = blockIdx.x * 128;
  const int rows = min(128, nb - j0);
  const float* src = kbar + (bg * nb + j0) * D;
  for (int e = threadIdx.x; e < rows * kChunks; e += 128) {
    const int r = e / kChunks, c = e % kChunks;
    cp_async16(smem_u32(ks + r * kPitch + 4 * c), src + static_cast<int64_t>(r) * D + 4 * c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.0f;
    for (int hh = 0; hh < G; ++hh) acc = __fadd_rn(acc, static_cast<float>(q[(b * Hq + g * G + hh) * D + c]));
    const float m = __fdiv_rn(acc, static_cast<float>(G));
    qm[c] = m;
    if (qbar_out && blockIdx.x == 0) qbar_out[bg * D + c] = m;
  }
  cp_async_wait_all();
  __syncthreads();
  const int r = threadIdx.x;
  if (r >= rows) return;
  const float4* row = reinterpret_cast<const float4*>(ks + r * kPitch);
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < kChunks; ++e) {
    const float4 kv = row[e];
    acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 0], kv.x));
    acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 1], kv.y));
    acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 2], kv.z));
    acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 3], kv.w));
  }
  s[bg * nb + j0 + r] = __fmul_rn(acc, scale);
}

// Generic-d fallback: rows staged through shared memory.
template <typename T>
__global__ void score_decode_generic_kernel(const T* __restrict__ q, const float* __restrict__ kbar, int Hq,
                                            int Hkv, int nb, int d, float scale, float* __restrict__ s,
                                            float* __restrict__ qbar_out) {
  extern __shared__ float sm[];
  const int pitch = d + 1;
  float* qm = sm;              // [d]
  float* ks = sm + d;          // [64][pitch]
  const int64_t bg = blockIdx.y;
  const int64_t b = bg / Hkv, g = bg % Hkv;
  const int G = Hq / Hkv;
  const int j0 = blockIdx.x * 64;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.0f;
    for (int hh = 0; hh < G; ++hh) acc = __fadd_rn(acc, static_cast<float>(q[(b * Hq + g * G + hh) * d + c]));
    const float m = __fdiv_rn(acc, static_cast<float>(G));
    qm[c] = m;
    if (qbar_out && blockIdx.x == 0) qbar_out[bg * d + c] = m;
  }
  const int rows = min(64, nb - j0);
  for (int e = threadIdx.x; e < rows * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    ks[r * pitch + c] = kbar[(bg * nb + j0 + r) * d + c];
  }
  __syncthreads();
  const int r = threadIdx.x;
  if (r < rows) s[bg * nb + j0 + r] = __fmul_rn(dot_fixed_order(qm, ks + r * pitch, d, 1), scale);
}

template <typename T, int D>
static cudaError_t launch_score_decode_d(dim3 grid, const void* q, const float* kbar, int Hq, int Hkv, int nb,
                                        float scale, float* s, float* qbar_out, cudaStream_t st) {
  constexpr size_t smem = (128 * (D + 4) + D) * sizeof(float);
  cudaError_t e = ensure_dynamic_smem<score_decode_kernel<T, D>>(smem);
  if (e != cudaSuccess) return e;
  score_decode_kernel<T, D><<<grid, 128, smem, st>>>(static_cast<const T*>(q), kbar, Hq, Hkv, nb, scale, s, qbar_out);
  return cudaGetLastError();
}

cudaError_t launch_score_decode(const void* q, bool bf16, const float* kbar, int B, int Hq, int Hkv,
                                int nb, int d, float scale, float* s, float* qbar_out,
                                cudaStream_t st) {
  if (d == 128 || d == 64) {
    dim3 grid((nb + 127) / 128, B * Hkv);
    if (bf16)
      return d == 128 ? launch_score_decode_d<__nv_bfloat16, 128>(grid, q, kbar, Hq, Hkv, nb, scale, s, qbar_out, st)
                      : launch_score_decode_d<__nv_bfloat16, 64>(grid, q, kbar, Hq, Hkv, nb, scale, s, qbar_out, st);
    return d == 128 ? launch_score_decode_d<float, 128>(grid, q, kbar, Hq, Hkv, nb, scale, s, qbar_out, st)
                    : launch_score_decode_d<float, 64>(grid, q, kbar, Hq, Hkv, nb, scale, s, qbar_out, st);
  }
  dim3 grid((nb + 63) / 64, B * Hkv);
  const size_t smem = (d + 64 * (d + 1)) * sizeof(float);
  if (bf16)
    score_decode_generic_kernel<__nv_bfloat16><<<grid, 64, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), kbar, Hq, Hkv, nb, d, scale, s, qbar_out);
  else
    score_decode_generic_kernel<float><<<grid, 64, smem, st>>>(static_cast<const float*>(q), kbar, Hq, Hkv,
                                                               nb, d, scale, s, qbar_out);
  return cudaGetLastError();
}

// Gist: grid (tiles of 64 gists, B*Hkv); threads (64 gists) x G heads.
template <typename T>
__global__ void score_gist_kernel(const T* __restrict__ q, const T* __restrict__ gk, int Hq, int Hkv,
                                  int nc, int d, float scale, float* __restrict__ s) {
  extern __shared__ float sm[];
  const int pitch = d + 1;
  const int G = Hq / Hkv;
  float* qs = sm;                 // [G][d]
  float* ks = sm + G * d;         // [64][pitch]
  const int64_t bg = blockIdx.y;
  const int64_t b = bg / Hkv, g = bg % Hkv;
  const int c0 = blockIdx.x * 64;
  const int rows = min(64, nc - c0);
  for (int e = threadIdx.x; e < G * d; e += blockDim.x)
    qs[e] = static_cast<float>(q[(b * Hq + g * G) * d + e]);
  for (int e = threadIdx.x; e < rows * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    ks[r * pitch + c] = static_cast<float>(gk[(bg * nc + c0 + r) * d + c]);
  }
  __syncthreads();
  const int hh = threadIdx.x / 64, r = threadIdx.x % 64;
  if (hh < G && r < rows)
    s[((b * Hq + g * G + hh) * nc) + c0 + r] =
        __fmul_rn(dot_fixed_order(qs + hh * d, ks + r * pitch, d, 1), scale);
}

// Gist, bf16, d = 128: persistent; a thread owns one gist row of a tile and
// a pair of the group's heads, so each widened gist value serves both heads'
// fixed-order dot products (channels ascending, each product and sum rounded
// on its own, as the generic kernel).  A
// tile is 64 consecutive gist keys of one (b, g); each CTA takes a contiguous
// range of tiles, R tiles at a time (R = threads / (64 x head pairs)), the
// tiles brought in by TMA (two 64-channel halves, 128-byte swizzle, so the
// same 16-byte chunk of eight consecutive rows sits in eight distinct bank
// groups) `stages` tiles ahead; the group's query rows are staged, as
// head-pair interleaved floats, only when a slot's (b, g) changes.
constexpr int kGistTileBytes = 64 * 128 * 2;
constexpr int kGistMaxStages = 8;

__global__ void __launch_bounds__(512) score_gist_bf16_d128_kernel(const __grid_constant__ CUtensorMap tmG,
                                                                  const __nv_bfloat16* __restrict__ q, int Hq,
                                                                  int Hkv, int nc, int64_t tiles, int stages,
                                                                  float scale, float* __restrict__ s,
                                                                  uint32_t* __restrict__ status) {
  constexpr int D = 128;
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm_gist = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kGistMaxStages];
  __shared__ __align__(16) float qs[16 * D];   // per round slot: head pairs x channels x 2
  __shared__ int abort_flag;
  const int G = Hq / Hkv, HP = (G + 1) / 2;
  const int tpt = 64 * HP;                     // threads per tile
  const int R = blockDim.x / tpt;              // tiles per round
  const int S = stages;                        // tile buffers (a multiple of R, at most kGistMaxStages)
  const int tpb = (nc + 63) / 64;              // tiles per (b, g)
  const uint32_t sbase = smem_u32(sm_gist);
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmG);
    for (int i = 0; i < S; ++i) mbar_init(smem_u32(&full[i]), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t per = (tiles + gridDim.x - 1) / gridDim.x;
  const int64_t t0 = min(tiles, static_cast<int64_t>(blockIdx.x) * per), t1 = min(tiles, t0 + per);
  auto issue = [&](int64_t tile) {
    const int k = static_cast<int>(tile - t0), stage = k % S;
    const int64_t bg = tile / tpb;
    const int c0 = static_cast<int>(tile % tpb) * 64;
    const uint32_t bar = smem_u32(&full[stage]);
    mbar_arrive_expect_tx(bar, kGistTileBytes);   // rows past the last gist are zero-filled
    const int y = static_cast<int>(bg * nc + c0);
    tma_load_2d(sbase + stage * kGistTileBytes, &tmG, bar, 0, y);
    tma_load_2d(sbase + stage * kGistTileBytes + kGistTileBytes / 2, &tmG, bar, 64, y);
  };
  if (threadIdx.x == 0)
    for (int64_t t = t0; t < t1 && t < t0 + S; ++t) issue(t);
  const int slot = threadIdx.x / tpt, within = threadIdx.x % tpt;
  const int pr = within / 64, r = within % 64;   // head pair, gist row
  const bool active = slot < R;
  float* qslot = qs + slot * (HP * 2 * D);
  int64_t qbg = -1, cur = t0;
  bool ok = true;
  for (int64_t base = t0; base < t1; base += R) {
    cur = base;
    const int64_t tile = base + slot;
    const bool mine = active && tile < t1;
    const int64_t bg = mine ? tile / tpb : -1;
    const int64_t b = bg / Hkv, g = bg % Hkv;
    // the slot's query rows, head pair interleaved: [pair][channel][2]
    if (mine && bg != qbg) {
      for (int e = within; e < HP * D; e += tpt) {
        const int p2 = e / D, c = e % D;
        const int h0 = 2 * p2, h1 = 2 * p2 + 1;
        qslot[(p2 * D + c) * 2] = __bfloat162float(q[(b * Hq + g * G + h0) * D + c]);
        qslot[(p2 * D + c) * 2 + 1] = (h1 < G) ? __bfloat162float(q[(b * Hq + g * G + h1) * D + c]) : 0.0f;
      }
      qbg = bg;
    }
    const int k = static_cast<int>(tile - t0), stage = k % S;
    if (mine) ok = mbar_wait(smem_u32(&full[stage]), (k / S) & 1, &abort_flag, status) && ok;
    __syncthreads();
    if (mine && ok) {
      const int c0 = static_cast<int>(tile % tpb) * 64;
      if (r < min(64, nc - c0)) {
        const uint8_t* tb = sm_gist + stage * kGistTileBytes + r * 128;
        const float4* q4 = reinterpret_cast<const float4*>(qslot + pr * 2 * D);
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          // chunk x (channels 8x .. 8x+7): half x / 8, 16-byte slot (x % 8) ^ (r % 8)
          const uint4 w = *reinterpret_cast<const uint4*>(tb + (x >> 3) * (kGistTileBytes / 2) + (((x & 7) ^ (r & 7)) << 4));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const float4 qq = q4[4 * x + y];   // channels 8x+2y, 8x+2y+1, both heads
            const float k0 = __uint_as_float(ws[y] << 16), k1 = __uint_as_float(ws[y] & 0xFFFF0000u);
            a0 = __fadd_rn(a0, __fmul_rn(qq.x, k0));
            a1 = __fadd_rn(a1, __fmul_rn(qq.y, k0));
            a0 = __fadd_rn(a0, __fmul_rn(qq.z, k1));
            a1 = __fadd_rn(a1, __fmul_rn(qq.w, k1));
          }
        }
        const int h0 = 2 * pr, h1 = 2 * pr + 1;
        s[((b * Hq + g * G + h0) * nc) + c0 + r] = __fmul_rn(a0, scale);
        if (h1 < G) s[((b * Hq + g * G + h1) * nc) + c0 + r] = __fmul_rn(a1, scale);
      }
    }
    // the round's stages are free again; so are the query rows of a slot
    // whose next tile belongs to another (b, g)
    __syncthreads();
    if (abort_flag) break;
    if (threadIdx.x == 0)
      for (int64_t t = base + S; t < t1 && t < base + S + R; ++t) issue(t);
  }
  if (threadIdx.x == 0 && abort_flag) {
    // let the copies in flight land before the CTA exits: the tiles of the
    // round that gave up and of the one issued ahead of it
    for (int64_t t = cur; t < t1 && t < cur + S; ++t) {
      const int k = static_cast<int>(t - t0);
      mbar_drain(smem_u32(&full[k % S]), (k / S) & 1);
    }
  }
}

cudaError_t launch_score_gist(const CUtensorMap* tmG, const void* q, const void* gk, bool bf16, int B, int Hq,
                              int Hkv, int nc, int d, float scale, float* s, uint32_t* status, int num_sms,
                              cudaStream_t st) {
  const int G = Hq / Hkv;
  dim3 grid((nc + 63) / 64, B * Hkv);
  if (tmG != nullptr && bf16 && d == 128 && G <= 16) {
    const int HP = (G + 1) / 2;
    const int threads = max(256, 64 * HP);
    const int R = threads / (64 * HP);
    const int64_t tiles = static_cast<int64_t>(B) * Hkv * ((nc + 63) / 64);
    // one round of R tiles per CTA while that keeps a few waves of small CTAs
    // (every tile's copy in flight at once); beyond that, persistent CTAs
    // with two rounds of buffers
    const int64_t need = (tiles + R - 1) / R;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    const unsigned ctas = static_cast<unsigned>(need < cap ? need : cap);
    const int stages = (need <= cap) ? R : 2 * R;
    if (ctas == 0) return cudaSuccess;
    const size_t smem2 = static_cast<size_t>(stages) * kGistTileBytes + 1024;   // + alignment slack
    cudaError_t e = ensure_dynamic_smem<score_gist_bf16_d128_kernel>(smem2);
    if (e != cudaSuccess) return e;
    score_gist_bf16_d128_kernel<<<ctas, threads, smem2, st>>>(*tmG, static_cast<const __nv_bfloat16*>(q), Hq, Hkv,
                                                              nc, tiles, stages, scale, s, status);
    return cudaGetLastError();
  }
  const size_t smem = (G * d + 64 * (d + 1)) * sizeof(float);
  if (bf16)
    score_gist_kernel<__nv_bfloat16><<<grid, 64 * G, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(gk), Hq, Hkv, nc, d,
        scale, s);
  else
    score_gist_kernel<float><<<grid, 64 * G, smem, st>>>(static_cast<const float*>(q),
                                                         static_cast<const float*>(gk), Hq, Hkv, nc,
                                                         d, scale, s);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ top-k

// One CTA per row.  Radix select (4 passes of 8 bits, most significant
// first) finds the key T of the k-th best candidate and how many candidates
// equal to T must be taken; warp 0 then walks the candidates in index order,
// taking every key > T and the lowest-index ties, which writes the kept list
// already ascending.  The forced block (current / last) is larger than every
// candidate, so it is appended at the end.
constexpr int kTopkThreads = 256;

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int ncols,
                                                            int mode, int kb, int* __restrict__ idx_out,
                                                            int idx_stride, int* __restrict__ count_out) {
  griddep_wait();   // the scores come from the kernel launched before
  extern __shared__ uint32_t skeys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit;
  __shared__ int s_remaining;
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int ncand, forced;
  if (mode == 0) {
    ncand = static_cast<int>(r % ncols);
    forced = ncand;
  } else if (mode == 1) {
    ncand = ncols - 1;
    forced = ncols - 1;
  } else {
    ncand = ncols;
    forced = -1;
  }
  const float* srow = scores + r * ncols;
  for (int j = tid; j < ncand; j += kTopkThreads) skeys[j] = order_key(srow[j]);
  const int take = min(kb, ncand);
  const bool take_all = (take == ncand);
  uint32_t thresh = 0;
  int remaining = take;
  __syncthreads();
  if (!take_all && take > 0) {
    uint32_t prefix = 0, pmask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < ncand; j += kTopkThreads) {
        const uint32_t k = skeys[j];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns digits 255-8l down to 248-8l (descending)
        uint32_t cnt[8];
        uint32_t mine = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = hist[255 - 8 * lane - e];
          mine += cnt[e];
        }
        uint32_t incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        const uint32_t excl = incl - mine;
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= static_cast<uint32_t>(remaining));
        const int first = __ffs(hit) - 1;   // always found: total >= remaining
        if (lane == first) {
          uint32_t cum = excl;
          for (int e = 0; e < 8; ++e) {
            if (cum + cnt[e] >= static_cast<uint32_t>(remaining)) {
              s_digit = 255 - 8 * lane - e;
              s_remaining = remaining - static_cast<int>(cum);
              break;
            }
            cum += cnt[e];
          }
        }
      }
      __syncthreads();
      remaining = s_remaining;
      prefix |= s_digit << shift;
      pmask |= 255u << shift;
      __syncthreads();
    }
    thresh = prefix;
  }
  if (warp != 0) return;
  int* out = idx_out + r * idx_stride;
  int run_sel = 0, run_tie = 0;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < ncand; base += 32) {
    const int j = base + lane;
    const bool valid = j < ncand;
    const uint32_t k = valid ? skeys[j] : 0u;
    bool gt, tie;
    if (take_all) {
      gt = valid;
      tie = false;
    } else if (take == 0) {
      gt = false;
      tie = false;
    } else {
      gt = valid && k > thresh;
      tie = valid && k == thresh;
    }
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    const int tie_rank = run_tie + __popc(tb & lt_mask);
    const bool sel = gt || (tie && tie_rank < remaining);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) out[run_sel + __popc(sb & lt_mask)] = j;
    run_sel += __popc(sb);
    run_tie += __popc(tb);
  }
  if (forced >= 0) {
    if (lane == 0) out[run_sel] = forced;
    ++run_sel;
  }
  for (int t = run_sel + lane; t < idx_stride; t += 32) out[t] = -1;
  if (count_out && lane == 0) count_out[r] = run_sel;
}

// Warp-per-row variant for rows of at most 32*KPL candidates: lane l holds
// candidates e*32 + l (e < KPL) in registers, loaded with coalesced reads.
// The key T of the k-th best candidate is found bit by bit from the most
// significant end (the largest T with at least k keys >= T), counting with
// warp reductions; then the warp walks e = 0, 1, ... (index order), taking
// every key > T and the lowest-index keys equal to T, and writes them at
// ballot prefix positions -- already ascending.
template <int KPL>
__global__ void __launch_bounds__(128) topk_warp_kernel(const float* __restrict__ scores, int rows, int ncols,
                                                        int mode, int kb, int* __restrict__ idx_out, int idx_stride,
                                                        int* __restrict__ count_out) {
  griddep_wait();   // the scores come from the kernel launched before
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  int ncand, forced;
  if (mode == 0) {
    ncand = static_cast<int>(r % ncols);
    forced = ncand;
  } else if (mode == 1) {
    ncand = ncols - 1;
    forced = ncols - 1;
  } else {
    ncand = ncols;
    forced = -1;
  }
  const float* srow = scores + r * ncols;
  uint32_t key[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = e * 32 + lane;
    key[e] = (j < ncand) ? order_key(__ldg(srow + j)) : 0u;
  }
  const int take = min(kb, ncand);
  const bool take_all = (take == ncand);
  uint32_t thresh = 0u;
  int remaining = take;     // how many keys equal to thresh are taken
  if (!take_all && take > 0) {
    // slots past the candidates hold key 0, and every threshold tried has a
    // bit set, so they never count: the counting loops need no bounds test
    uint32_t prefix = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int e = 0; e < KPL; ++e) cnt += (key[e] >= cand) ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= take) prefix = cand;
    }
    thresh = prefix;
    int gt = 0;
#pragma unroll
    for (int e = 0; e < KPL; ++e) gt += (e * 32 + lane < ncand && key[e] > thresh) ? 1 : 0;
    gt = __reduce_add_sync(0xffffffffu, gt);
    remaining = take - gt;
  }
  int* out = idx_out + r * idx_stride;
  const unsigned lt_mask = (1u << lane) - 1u;
  int run_sel = 0, run_tie = 0;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = e * 32 + lane;
    const bool valid = j < ncand;
    bool gt, tie;
    if (take_all) {
      gt = valid;
      tie = false;
    } else if (take == 0) {
      gt = false;
      tie = false;
    } else {
      gt = valid && key[e] > thresh;
      tie = valid && key[e] == thresh;
    }
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    const bool sel = gt || (tie && run_tie + __popc(tb & lt_mask) < remaining);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) out[run_sel + __popc(sb & lt_mask)] = j;
    run_sel += __popc(sb);
    run_tie += __popc(tb);
  }
  int n = run_sel;
  if (forced >= 0) {
    if (lane == 0) out[n] = forced;
    ++n;
  }
  for (int t = n + lane; t < idx_stride; t += 32) out[t] = -1;
  if (count_out && lane == 0) count_out[r] = n;
}

// CTA-per-row variant for rows of up to 256*KPT candidates.  Thread t holds
// candidates j = t*KPT .. t*KPT+KPT-1 (index order within the CTA).  Radix
// select in four 8-bit passes (most significant first): each pass builds a
// 256-bin shared histogram of the digit among the candidates that match the
// prefix found so far, and one warp's suffix scan over the bins picks the
// digit that holds the k-th best key.  The result is the key T of the k-th
// best candidate and the number of candidates equal to T still to be taken.
// A block-wide exclusive scan of each thread's (> T, == T) counts then gives
// every kept candidate its output slot directly: the number of kept
// candidates of lower index, i.e. all keys > T plus the lowest-index ties.
template <int KPT>
__global__ void __launch_bounds__(256) topk_cta_kernel(const float* __restrict__ scores, int ncols, int mode, int kb,
                                                       int* __restrict__ idx_out, int idx_stride,
                                                       int* __restrict__ count_out) {
  griddep_wait();   // the scores come from the kernel launched before
  const int tid = threadIdx.x;
  const int64_t r = blockIdx.x;
  int ncand, forced;
  if (mode == 0) {
    ncand = static_cast<int>(r % ncols);
    forced = ncand;
  } else if (mode == 1) {
    ncand = ncols - 1;
    forced = ncols - 1;
  } else {
    ncand = ncols;
    forced = -1;
  }
  const float* srow = scores + r * ncols;
  const int j0 = tid * KPT;
  uint32_t key[KPT];
#pragma unroll
  for (int e = 0; e < KPT; ++e) key[e] = (j0 + e < ncand) ? order_key(__ldg(srow + j0 + e)) : 0u;
  cta_topk_select<KPT>(key, ncand, kb, forced, idx_out + r * idx_stride, idx_stride,
                       count_out ? count_out + r : nullptr);
}

// ------------------------------------------------------- decode selector
// The decode selector in one kernel (d = 128, at most 2048 blocks): one CTA
// per (batch, KV group) row forms the group query mean, streams the row's
// pooled-key summary through shared memory and scores every block, then
// keeps the top-kb history blocks and the last block -- the work of
// score_decode_kernel followed by topk_cta_kernel<8>, with the scores held in
// shared memory between the two (tutorial §5: decode reads the history for
// one new query; SAS page, 推理: the k best units are kept, the last block
// always).  Same arithmetic, same order, so the same bits.
//
// The summary rows arrive by TMA in chunks of 128 rows: four boxes of 32
// channels (128 bytes) x 128 rows with the 128-byte swizzle, so the float4
// reads of eight consecutive rows at one channel offset fall in distinct
// banks.  Three chunks are in flight while threads 0..127 score the oldest
// (thread = row, channels ascending).
constexpr int kDsThreads = 256;
constexpr int kDsRows = 128;
constexpr int kDsStages = 3;
constexpr uint32_t kDsBox = 128u * 128u;             // 128 rows x 128 bytes
constexpr uint32_t kDsChunk = 4u * kDsBox;           // 128 rows x 128 floats
constexpr int kDsMaxBlocks = 256 * 8;                // the CTA select holds 8 keys per thread
constexpr uint32_t kDsScores = kDsStages * kDsChunk;                    // float[kDsMaxBlocks]
constexpr uint32_t kDsQm = kDsScores + kDsMaxBlocks * 4;                // float[128]
constexpr uint32_t kDsBar = kDsQm + 128 * 4;                            // kDsStages mbarriers
constexpr uint32_t kDsSmem = kDsBar + kDsStages * 8 + 1024;             // + alignment slack

template <typename T>
__global__ void __launch_bounds__(kDsThreads, 1)
    decode_select_kernel(const __grid_constant__ CUtensorMap tmKbar, const T* __restrict__ q, int Hq, int Hkv,
                         int nb, float scale, int kb, float* __restrict__ scores, float* __restrict__ qbar_out,
                         int* __restrict__ idx_out, int idx_stride, int* __restrict__ count_out,
                         uint32_t* __restrict__ status) {
  extern __shared__ uint8_t ds_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ds_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* sc = reinterpret_cast<float*>(sm + kDsScores);
  float* qm = reinterpret_cast<float*>(sm + kDsQm);
  __shared__ int abort_flag;
  const int tid = threadIdx.x;
  const int64_t bg = blockIdx.x;
  const int64_t b = bg / Hkv, g = bg % Hkv;
  const int G = Hq / Hkv;
  const int nchunks = (nb + kDsRows - 1) / kDsRows;
  auto bar = [&](int st) -> uint32_t { return sbase + kDsBar + 8u * st; };
  auto issue = [&](int c) {
    const int st = c % kDsStages;
    mbar_arrive_expect_tx(bar(st), kDsChunk);
    const int y = static_cast<int>(bg * nb) + c * kDsRows;   // rows past the tensor read the zero fill
    for (int k = 0; k < 4; ++k) tma_load_2d(sbase + st * kDsChunk + k * kDsBox, &tmKbar, bar(st), 32 * k, y);
  };
  if (tid == 0) {
    abort_flag = 0;
    for (int st = 0; st < kDsStages; ++st) mbar_init(bar(st), 1);
    fence_barrier_init();
    prefetch_tmap(&tmKbar);
  }
  __syncthreads();
  griddep_wait();   // the query may come from the kernel launched before
  int issued = 0;   // chunks whose copies thread 0 has started
  if (tid == 0)
    for (; issued < min(kDsStages, nchunks); ++issued) issue(issued);
  if (tid < 128) {
    // group query mean, heads ascending, one division (as score_decode_kernel)
    float acc = 0.0f;
    for (int hh = 0; hh < G; ++hh) acc = __fadd_rn(acc, static_cast<float>(q[(b * Hq + g * G + hh) * 128 + tid]));
    const float m = __fdiv_rn(acc, static_cast<float>(G));
    qm[tid] = m;
    if (qbar_out) qbar_out[bg * 128 + tid] = m;
  }
  __syncthreads();
  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % kDsStages;
    ok = mbar_wait(bar(st), (c / kDsStages) & 1, &abort_flag, status);
    if (ok && tid < kDsRows) {
      const int r = tid, row = c * kDsRows + r;
      if (row < nb) {
        const uint32_t rbase = sbase + st * kDsChunk + r * 128u;
        float acc = 0.0f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          // channels 4e..4e+3: box e/8, 16-byte chunk (e%8) XOR (row%8)
          const uint32_t a = rbase + (e >> 3) * kDsBox + ((((e & 7) ^ (r & 7)) & 7) << 4);
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(a));
          acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 0], v.x));
          acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 1], v.y));
          acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 2], v.z));
          acc = __fadd_rn(acc, __fmul_rn(qm[4 * e + 3], v.w));
        }
        const float sv = __fmul_rn(acc, scale);
        sc[row] = sv;
        scores[bg * nb + row] = sv;
      }
    }
    // every thread has passed the wait of chunk c (or given up) before its
    // stage is refilled
    if (!__syncthreads_and(ok)) break;
    if (tid == 0 && c + kDsStages < nchunks) issue(issued++);
  }
  if (abort_flag) {
    // an expired wait was recorded in the status word; let the copies in
    // flight land before the CTA exits
    if (tid == 0)
      for (int c = max(0, issued - kDsStages); c < issued; ++c) mbar_drain(bar(c % kDsStages), (c / kDsStages) & 1);
    return;
  }
  // top-k of blocks 0..nb-2, block nb-1 kept (the decode candidate rule)
  const int ncand = nb - 1;
  uint32_t key[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) key[e] = (tid * 8 + e < ncand) ? order_key(sc[tid * 8 + e]) : 0u;
  cta_topk_select<8>(key, ncand, kb, nb - 1, idx_out + bg * idx_stride, idx_stride,
                     count_out ? count_out + bg : nullptr);
}

bool decode_select_fused_ok(int d, int nb) { return d == 128 && nb >= 1 && nb <= kDsMaxBlocks; }

cudaError_t launch_decode_select(const CUtensorMap* tmKbar, const void* q, bool bf16, int B, int Hq, int Hkv,
                                 int nb, float scale, int kb, float* scores, float* qbar_out, int* idx_out,
                                 int idx_stride, int* count_out, uint32_t* status, cudaStream_t st) {
  const dim3 grid(B * Hkv);
  if (bf16) {
    cudaError_t e = ensure_dynamic_smem<decode_select_kernel<__nv_bfloat16>>(kDsSmem);
    if (e != cudaSuccess) return e;
    return launch_dependent(decode_select_kernel<__nv_bfloat16>, grid, dim3(kDsThreads), kDsSmem, st, *tmKbar,
                            static_cast<const __nv_bfloat16*>(q), Hq, Hkv, nb, scale, kb, scores, qbar_out, idx_out,
                            idx_stride, count_out, status);
  }
  cudaError_t e = ensure_dynamic_smem<decode_select_kernel<float>>(kDsSmem);
  if (e != cudaSuccess) return e;
  return launch_dependent(decode_select_kernel<float>, grid, dim3(kDsThreads), kDsSmem, st, *tmKbar,
                          static_cast<const float*>(q), Hq, Hkv, nb, scale, kb, scores, qbar_out, idx_out, idx_stride,
                          count_out, status);
}

// ------------------------------------------- fixed pattern + dynamic blocks
// Prefill selection with a fixed part (Sparse Frontier review §2.2.3,
// MInference block-sparse: the first blocks of the sequence, the local window,
// and a set of dynamically selected blocks per query block).  Row r is query
// block i = r % ncols.  Kept: the first `sink` blocks, the `local` most recent
// blocks (i included) and the kb best of the blocks between them.  The three
// sets are disjoint ranges in block order, [0, P) | candidates [P, S) | [S, i],
// so the list is written already ascending.  One CTA per row.
template <int KPT>
__global__ void __launch_bounds__(256) topk_pattern_kernel(const float* __restrict__ scores, int ncols, int sink,
                                                           int local, int kb, int* __restrict__ idx_out,
                                                           int idx_stride, int* __restrict__ count_out) {
  griddep_wait();   // the scores come from the kernel launched before
  __shared__ int s_nsel;
  const int tid = threadIdx.x;
  const int64_t r = blockIdx.x;
  const int i = static_cast<int>(r % ncols);
  const int P = min(sink, i + 1);
  const int S = max(P, i - local + 1);
  const int ncand = S - P;
  int* out = idx_out + r * idx_stride;
  const float* srow = scores + r * ncols + P;
  uint32_t key[KPT];
#pragma unroll
  for (int e = 0; e < KPT; ++e) key[e] = (tid * KPT + e < ncand) ? order_key(__ldg(srow + tid * KPT + e)) : 0u;
  for (int t = tid; t < P; t += 256) out[t] = t;
  cta_topk_select<KPT>(key, ncand, kb, -1, out + P, idx_stride - P, &s_nsel, P);
  __syncthreads();
  const int n0 = P + s_nsel;
  for (int t = tid; t <= i - S; t += 256) out[n0 + t] = S + t;
  if (tid == 0 && count_out) count_out[r] = n0 + (i + 1 - S);
}

cudaError_t launch_topk_pattern(const float* scores, int rows, int ncols, int sink, int local, int kb, int* idx_out,
                                int idx_stride, int* count_out, cudaStream_t st) {
  if (ncols <= 256 * 8)
    return launch_dependent(topk_pattern_kernel<8>, dim3(rows), dim3(256), 0, st, scores, ncols, sink, local, kb,
                            idx_out, idx_stride, count_out);
  return launch_dependent(topk_pattern_kernel<32>, dim3(rows), dim3(256), 0, st, scores, ncols, sink, local, kb,
                          idx_out, idx_stride, count_out);
}

// --------------------------------------------- per-head decode scores
// Each query head's decode scores against the pooled-key summary,
// s[b][h][j] = q_h . kbar_{g,j} / sqrt(d) in the fixed order (channels
// ascending, products and sums rounded separately) -- the per-head scores
// that a budget shared across the heads (Ada-KV) ranks.  Grid (tiles of 128
// blocks, B*Hkv); thread = block row; the CTA's pooled rows are staged as in
// score_decode_kernel, the G query rows as floats.
template <typename T, int D>
__global__ void __launch_bounds__(128) score_heads_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                          int Hq, int Hkv, int nb, float scale,
                                                          float* __restrict__ s) {
  constexpr int kPitch = D + 4;
  constexpr int kChunks = D / 4;
  extern __shared__ __align__(16) float sm_heads[];
  float* ks = sm_heads;                  // [128][kPitch]
  float* qs = sm_heads + 128 * kPitch;   // [G][D]
  const int64_t bg = blockIdx.y;
  const int64_t b = bg / Hkv, g = bg % Hkv;
  const int G = Hq / Hkv;
  const int j0 = blockIdx.x * 128;
  const int rows = min(128, nb - j0);
  const float* src = kbar + (bg * nb + j0) * D;
  for (int e = threadIdx.x; e < rows * kChunks; e += 128) {
    const int r = e / kChunks, c = e % kChunks;
    cp_async16(smem_u32(ks + r * kPitch + 4 * c), src + static_cast<int64_t>(r) * D + 4 * c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int e = threadIdx.x; e < G * D; e += 128) qs[e] = static_cast<float>(q[(b * Hq + g * G) * D + e]);
  cp_async_wait_all();
  __syncthreads();
  const int r = threadIdx.x;
  if (r >= rows) return;
  const float4* row = reinterpret_cast<const float4*>(ks + r * kPitch);
  for (int hh = 0; hh < G; ++hh) {
    const float* qr = qs + hh * D;
    float acc = 0.0f;
#pragma unroll
    for (int e = 0; e < kChunks; ++e) {
      const float4 kv = row[e];
      acc = __fadd_rn(acc, __fmul_rn(qr[4 * e + 0], kv.x));
      acc = __fadd_rn(acc, __fmul_rn(qr[4 * e + 1], kv.y));
      acc = __fadd_rn(acc, __fmul_rn(qr[4 * e + 2], kv.z));
      acc = __fadd_rn(acc, __fmul_rn(qr[4 * e + 3], kv.w));
    }
    s[((b * Hq + g * G + hh) * nb) + j0 + r] = __fmul_rn(acc, scale);
  }
}

template <typename T, int D>
static cudaError_t launch_score_heads_d(dim3 grid, int G, const void* q, const float* kbar, int Hq, int Hkv, int nb,
                                        float scale, float* s, cudaStream_t st) {
  const size_t smem = (128 * (D + 4) + G * D) * sizeof(float);
  cudaError_t e = ensure_dynamic_smem<score_heads_kernel<T, D>>(smem);
  if (e != cudaSuccess) return e;
  score_heads_kernel<T, D><<<grid, 128, smem, st>>>(static_cast<const T*>(q), kbar, Hq, Hkv, nb, scale, s);
  return cudaGetLastError();
}

cudaError_t launch_score_heads(const void* q, bool bf16, const float* kbar, int B, int Hq, int Hkv, int nb, int d,
                               float scale, float* s, cudaStream_t st) {
  const dim3 grid((nb + 127) / 128, B * Hkv);
  const int G = Hq / Hkv;
  if (d == 128)
    return bf16 ? launch_score_heads_d<__nv_bfloat16, 128>(grid, G, q, kbar, Hq, Hkv, nb, scale, s, st)
                : launch_score_heads_d<float, 128>(grid, G, q, kbar, Hq, Hkv, nb, scale, s, st);
  if (d == 64)
    return bf16 ? launch_score_heads_d<__nv_bfloat16, 64>(grid, G, q, kbar, Hq, Hkv, nb, scale, s, st)
                : launch_score_heads_d<float, 64>(grid, G, q, kbar, Hq, Hkv, nb, scale, s, st);
  return cudaErrorInvalidValue;
}

// ------------------------------------------ one budget across a group's heads
// Ada-KV (Sparse Frontier review §2.3.2): the group's G heads share one
// budget of kb_total (head, block) pairs, so an important head keeps more
// blocks and others fewer.  One CTA per (batch, KV group) row; candidate
// c = h*(nb-1) + j (j < nb-1: the last block is kept by every head) has the
// score s[b][g*G+h][j].  The CTA select takes the best kb_total candidates
// (equal scores: lower c first) and writes them ascending in c into shared
// memory, i.e. head by head with blocks ascending; each head's run then
// becomes its kept list, the last block appended.
template <int KPT>
__global__ void __launch_bounds__(256) topk_joint_kernel(const float* __restrict__ scores, int G, int nb,
                                                         int kb_total, int* __restrict__ idx_out, int idx_stride,
                                                         int* __restrict__ count_out) {
  griddep_wait();
  extern __shared__ int sl_joint[];   // [min(kb_total, G*(nb-1))]
  __shared__ int s_n;
  __shared__ int s_cnt[16], s_start[16];
  const int tid = threadIdx.x;
  const int64_t bg = blockIdx.x;
  const int per = nb - 1, ncand = G * per;
  const float* sbase = scores + bg * G * nb;
  uint32_t key[KPT];
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int c = tid * KPT + e;
    key[e] = (c < ncand) ? order_key(__ldg(sbase + (c / per) * nb + c % per)) : 0u;
  }
  if (tid < 16) s_cnt[tid] = 0;
  const int cap = min(kb_total, ncand);
  cta_topk_select<KPT>(key, ncand, kb_total, -1, sl_joint, cap, &s_n);
  __syncthreads();
  const int n = s_n;
  for (int t = tid; t < n; t += 256) atomicAdd(&s_cnt[sl_joint[t] / per], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int h = 0; h < G; ++h) {
      s_start[h] = run;
      run += s_cnt[h];
    }
  }
  __syncthreads();
  for (int t = tid; t < n; t += 256) {
    const int c = sl_joint[t], h = c / per;
    idx_out[(bg * G + h) * idx_stride + (t - s_start[h])] = c % per;
  }
  for (int e = tid; e < G * idx_stride; e += 256) {
    const int h = e / idx_stride, t = e % idx_stride;
    if (t == s_cnt[h]) idx_out[(bg * G + h) * idx_stride + t] = nb - 1;
    else if (t > s_cnt[h]) idx_out[(bg * G + h) * idx_stride + t] = -1;
  }
  if (count_out && tid < G) count_out[bg * G + tid] = s_cnt[tid] + 1;
}

cudaError_t launch_topk_joint(const float* scores, int rows, int G, int nb, int kb_total, int* idx_out,
                              int idx_stride, int* count_out, cudaStream_t st) {
  const int ncand = G * (nb - 1);
  const size_t smem = static_cast<size_t>(max(1, min(kb_total, ncand))) * sizeof(int);
  if (ncand <= 256 * 8)
    return launch_dependent(topk_joint_kernel<8>, dim3(rows), dim3(256), smem, st, scores, G, nb, kb_total, idx_out,
                            idx_stride, count_out);
  return launch_dependent(topk_joint_kernel<32>, dim3(rows), dim3(256), smem, st, scores, G, nb, kb_total, idx_out,
                          idx_stride, count_out);
}

// Two-level gists, fine stage: for row (b, h) and each of its km kept groups
// t (meta_idx), the scores of the group's 64 chunk gists.  One CTA per row,
// 256 threads = four groups at a time x 64 gists; the group tiles arrive by
// TMA (two 64-channel halves, 128-byte swizzle) in a four-stage ring, the
// next round's tiles loading while this round's dot products run.  Each
// thread runs the fixed-order dot product of its gist, channels ascending
// (as score_gist_bf16_d128_kernel).  fine [B*Hq][km*64]: position t*64 + x.
// A group slot past the kept ones gets NaN (never ranked above a number).
constexpr int kGroupStages = 4;

// The row's top-k over its km*64 fine scores held in shared memory (plain
// rule: every position a candidate, none forced; NaN scores of missing groups
// rank lowest), written as positions ascending.
constexpr int kGroupFuseMax = 256 * 8;   // positions the fused select holds (8 keys per thread)

template <int KPT>
__device__ __forceinline__ void group_row_select(const float* fsc, int ncand, int k, int* out, int stride) {
  uint32_t key[KPT];
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int j = static_cast<int>(threadIdx.x) * KPT + e;
    key[e] = (j < ncand) ? order_key(fsc[j]) : 0u;
  }
  cta_topk_select<KPT>(key, ncand, k, -1, out, stride, nullptr);
}

// pos_out != null: the row's fine scores stay in shared memory and the
// kernel also runs the row's top-k (the separate top-k launch is skipped).
__global__ void __launch_bounds__(256) score_gist_groups_kernel(const __grid_constant__ CUtensorMap tmG,
                                                                const __nv_bfloat16* __restrict__ q,
                                                                const int* __restrict__ meta_idx, int km, int Hq,
                                                                int Hkv, int nc, float scale,
                                                                float* __restrict__ fine, int topk,
                                                                int* __restrict__ pos_out, int pos_stride,
                                                                uint32_t* __restrict__ status) {
  constexpr int D = 128;
  extern __shared__ uint8_t sm_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kGroupStages];
  __shared__ float qs[D];
  __shared__ float fsc[kGroupFuseMax];
  __shared__ int abort_flag;
  const bool fused = pos_out != nullptr;
  const int64_t row = blockIdx.x;   // b * Hq + h
  const int64_t b = row / Hq;
  const int g = static_cast<int>(row % Hq) / (Hq / Hkv);
  const int grp = threadIdx.x >> 6, r = threadIdx.x & 63;
  const uint32_t sbase = smem_u32(tiles);
  const int nm = nc / 64;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmG);
    for (int i = 0; i < kGroupStages; ++i) mbar_init(smem_u32(&full[i]), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  griddep_wait();   // the kept groups come from the kernel launched before
  const int* mrow = meta_idx + row * km;
  // tile t into stage t % kGroupStages; a slot without a valid group still
  // completes its phase (an arrive without bytes), so the parities stay aligned
  auto issue = [&](int t) {
    const uint32_t bar = smem_u32(&full[t % kGroupStages]);
    const int m = mrow[t];
    if (m < 0 || m >= nm) {
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, 64 * D * 2);
    const int y = static_cast<int>((b * Hkv + g) * static_cast<int64_t>(nc) + m * 64);
    const uint32_t dst = sbase + (t % kGroupStages) * (64 * D * 2);
    tma_load_2d(dst, &tmG, bar, 0, y);
    tma_load_2d(dst + 64 * 128, &tmG, bar, 64, y);
  };
  int issued = 0;   // thread 0: tiles issued so far
  if (threadIdx.x == 0)
    for (; issued < km && issued < kGroupStages; ++issued) issue(issued);
  if (threadIdx.x < D) qs[threadIdx.x] = __bfloat162float(q[row * D + threadIdx.x]);
  __syncthreads();
  float* out = fine + row * (static_cast<int64_t>(km) * 64);
  bool ok = true;
  for (int base = 0; base < km; base += kGroupStages) {
    const int t = base + grp;
    if (t < km) {
      const int m = mrow[t];
      const bool valid = m >= 0 && m < nm;
      const bool got = mbar_wait(smem_u32(&full[t % kGroupStages]), (t / kGroupStages) & 1, &abort_flag, status);
      ok = ok && got;
      if (!valid) {
        if (fused) fsc[t * 64 + r] = __int_as_float(0x7fc00000);   // NaN
        else out[t * 64 + r] = __int_as_float(0x7fc00000);
      } else if (got) {
        const uint8_t* tb = tiles + (t % kGroupStages) * (64 * D * 2) + r * 128;
        float acc = 0.0f;
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          // chunk x (channels 8x .. 8x+7): half x / 8, 16-byte slot (x % 8) ^ (r % 8)
          const uint4 w = *reinterpret_cast<const uint4*>(tb + (x >> 3) * (64 * 128) + (((x & 7) ^ (r & 7)) << 4));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            acc = __fadd_rn(acc, __fmul_rn(qs[8 * x + 2 * y], __uint_as_float(ws[y] << 16)));
            acc = __fadd_rn(acc, __fmul_rn(qs[8 * x + 2 * y + 1], __uint_as_float(ws[y] & 0xFFFF0000u)));
          }
        }
        if (fused) fsc[t * 64 + r] = __fmul_rn(acc, scale);
        else out[t * 64 + r] = __fmul_rn(acc, scale);
      }
    }
    __syncthreads();   // this round's stages are free again
    if (abort_flag) break;
    if (threadIdx.x == 0)
      for (; issued < km && issued < base + 2 * kGroupStages; ++issued) issue(issued);
  }
  if (threadIdx.x == 0 && abort_flag) {
    // let the copies in flight land before the CTA exits
    for (int t = max(0, issued - kGroupStages); t < issued; ++t)
      mbar_drain(smem_u32(&full[t % kGroupStages]), (t / kGroupStages) & 1);
  }
  if (!fused || __syncthreads_or(abort_flag)) return;
  const int ncand = km * 64;
  int* prow = pos_out + row * pos_stride;
  if (ncand <= 256)
    group_row_select<1>(fsc, ncand, topk, prow, pos_stride);
  else if (ncand <= 512)
    group_row_select<2>(fsc, ncand, topk, prow, pos_stride);
  else if (ncand <= 1024)
    group_row_select<4>(fsc, ncand, topk, prow, pos_stride);
  else
    group_row_select<8>(fsc, ncand, topk, prow, pos_stride);
}

bool gist_groups_select_fused_ok(int km) { return km >= 1 && km * 64 <= kGroupFuseMax; }

cudaError_t launch_score_gist_groups(const CUtensorMap* tmG, const void* q, const int* meta_idx, int km, int B,
                                     int Hq, int Hkv, int nc, float scale, float* fine, int topk, int* pos_out,
                                     int pos_stride, uint32_t* status, cudaStream_t st) {
  if (pos_out != nullptr && !gist_groups_select_fused_ok(km)) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(kGroupStages) * 64 * 128 * 2 + 1024;   // + alignment slack
  cudaError_t e = ensure_dynamic_smem<score_gist_groups_kernel>(smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(score_gist_groups_kernel, dim3(B * Hq), dim3(256), smem, st, *tmG,
                          static_cast<const __nv_bfloat16*>(q), meta_idx, km, Hq, Hkv, nc, scale, fine, topk, pos_out,
                          pos_stride, status);
}

cudaError_t launch_topk(const float* scores, int rows, int ncols, int mode, int kb, int* idx_out,
                        int idx_stride, int* count_out, cudaStream_t st) {
  if (ncols <= 32 * 16) {
    const int warps = 4;
    const unsigned grid = static_cast<unsigned>((rows + warps - 1) / warps);
    return launch_dependent(topk_warp_kernel<16>, dim3(grid), dim3(32 * warps), 0, st, scores, rows, ncols, mode, kb,
                            idx_out, idx_stride, count_out);
  } else if (ncols <= 256 * 8) {
    return launch_dependent(topk_cta_kernel<8>, dim3(rows), dim3(256), 0, st, scores, ncols, mode, kb, idx_out,
                            idx_stride, count_out);
  } else {
    const size_t smem = static_cast<size_t>(ncols) * sizeof(uint32_t);
    return launch_dependent(topk_kernel, dim3(rows), dim3(kTopkThreads), smem, st, scores, ncols, mode, kb, idx_out,
                            idx_stride, count_out);
  }
  return cudaGetLastError();
}

}  // namespace bsa
