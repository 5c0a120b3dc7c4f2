// topk.cuh -- shared pieces of the hard top-k selection (SAS page, 推理
// paragraph: each query keeps its k best units): the order key of an fp32
// score and the CTA-wide selection of one row.
#pragma once

#include "common.cuh"

namespace bsa {

// Monotone unsigned key of an fp32 score: a larger score gives a larger key,
// -0 and +0 share one key, and every NaN gets key 0 (below -inf).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection of one row by a CTA of 256 threads (the algorithm is described at
// topk_cta_kernel in selector.cu):
// thread t holds the keys of candidates t*KPT .. t*KPT+KPT-1 (key 0 past
// ncand); writes the kept list (ascending, forced block last, -1 after it)
// to out and its length to *count_out (optional).  Candidate t is written as
// index_base + t.
template <int KPT>
__device__ __forceinline__ void cta_topk_select(const uint32_t (&key)[KPT], int ncand, int kb, int forced,
                                                int* __restrict__ out, int idx_stride, int* __restrict__ count_out,
                                                int index_base = 0) {
  __shared__ int hist[256];
  __shared__ uint32_t wsum[8];
  __shared__ int sel_digit, sel_above;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j0 = tid * KPT;
  const int take = min(kb, ncand);
  const bool take_all = (take == ncand);
  uint32_t thresh = 0u;
  int remaining = take;   // ties (== thresh) to keep
  if (!take_all && take > 0) {
    uint32_t prefix = 0u, pmask = 0u;
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[tid] = 0;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < KPT; ++e)
        if (j0 + e < ncand && (key[e] & pmask) == prefix) atomicAdd(&hist[(key[e] >> shift) & 255u], 1);
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 255-8l .. 248-8l (descending); suffix counts
        int c[8];
        int run = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          run += hist[255 - 8 * lane - i];
          c[i] = run;
        }
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const int excl = incl - run;   // keys in higher bins than this lane's
        // the digit is the first bin (from the top) whose suffix count reaches remaining
        int found = -1, above = 0;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          const int ge = excl + c[i];
          const int gt = excl + (i ? c[i - 1] : 0);
          if (ge >= remaining && gt < remaining) {
            found = 255 - 8 * lane - i;
            above = gt;
          }
        }
        const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(who) - 1;
        const int d = __shfl_sync(0xffffffffu, found, src);
        const int ab = __shfl_sync(0xffffffffu, above, src);
        if (lane == 0) {
          sel_digit = d;
          sel_above = ab;
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sel_digit) << shift;
      pmask |= 255u << shift;
      remaining -= sel_above;
      __syncthreads();   // hist and sel_* are rewritten by the next pass
    }
    thresh = prefix;
  }
  // this thread's kept candidates: every key > thresh, ties counted separately
  int ngt = 0, ntie = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const bool valid = j0 + e < ncand;
    if (take_all) {
      ngt += valid ? 1 : 0;
    } else if (take > 0) {
      ngt += (valid && key[e] > thresh) ? 1 : 0;
      ntie += (valid && key[e] == thresh) ? 1 : 0;
    }
  }
  // block exclusive scan of the packed (gt, tie) counts (each < 2^16)
  const uint32_t mine = static_cast<uint32_t>(ngt) | (static_cast<uint32_t>(ntie) << 16);
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t base = 0u, total = 0u;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    if (w < warp) base += wsum[w];
    total += wsum[w];
  }
  const uint32_t excl = base + incl - mine;
  int gt_before = static_cast<int>(excl & 0xFFFFu), tie_before = static_cast<int>(excl >> 16);
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const bool valid = j0 + e < ncand;
    const bool gt = take_all ? valid : (take > 0 && valid && key[e] > thresh);
    const bool tie = !take_all && take > 0 && valid && key[e] == thresh;
    if (gt || (tie && tie_before < remaining)) out[gt_before + min(tie_before, remaining)] = index_base + j0 + e;
    gt_before += gt ? 1 : 0;
    tie_before += tie ? 1 : 0;
  }
  int n = static_cast<int>(total & 0xFFFFu) + min(static_cast<int>(total >> 16), remaining);
  if (forced >= 0) {
    if (tid == 0) out[n] = forced;
    ++n;
  }
  for (int t = n + tid; t < idx_stride; t += 256) out[t] = -1;
  if (count_out && tid == 0) *count_out = n;
}


}  // namespace bsa
