// attn_prefill.cu -- block-sparse causal attention, prefill, bf16, d = 128,
// on sm_100a tensor cores (tcgen05 MMA into tensor memory, TMA tile loads).
//
// What it computes (source pages): softmax(QK^T/sqrt(d) + M)V with the
// additive mask M in {0,-inf} of the "稀疏注意力" tutorial (§1, §2), where
// M = 0 exactly on the keys of the kept blocks that are not in the query's
// future (§4.5 block-sparse pattern); the masked region is never computed
// (§2: real speed-up only if skipping happens at QK^T), using online softmax
// over the kept blocks (§7, Block-Sparse FlashAttention).  With a selector
// score matrix it computes the SAS gated variant (SAS page, 核心模块 2-3):
// every logit of kept block j gains log g_j, g = softmax of the group's
// selector scores over the kept blocks (current block included).
//
// Work decomposition.  A unit is (batch b, KV group g, query block i): the
// G heads of the group share one kept-block list, so their bs query rows
// each are stacked into G*bs rows that all read the same K/V tiles.  A CTA
// takes two 128-row tiles of one unit ("ping-pong": while one tile's
// softmax runs on CUDA cores, the tensor core works on the other tile), so
// each K/V tile is fetched into shared memory once for 256 query rows.
//
// Roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K and V of each step into a
//               two-stage ring, gathered by block index;
//   warp 1      TMEM owner + MMA issuer (one thread): S = Q K^T (SS form),
//               O += P V (TS form, P read from tensor memory);
//   warps 4-7   softmax of tile 0 (thread = query row = TMEM lane);
//   warps 8-11  softmax of tile 1.
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each; P (bf16
// pairs) is written over the first half of its S region.  tcgen05.mma
// instructions from one thread execute in issue order, so S(t, s+1), issued
// after O += P(t, s) V, never overwrites P before that MMA has read it.
//
// A step covers 128 keys: two 64-token blocks (bs = 64) or one 128-token
// block (bs = 128); the last step of an odd list holds one 64-token block.
//
// Softmax uses the base-2 exponent with the scale folded in, and a lazy
// rescale: the running maximum is only moved (and O rescaled in tensor
// memory) when a row's new maximum exceeds it by more than 8 (a factor 256),
// which keeps every P <= 256 and is exact after the final division.
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace prefill {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kStages = 2;
constexpr int kMaxList = 256;
constexpr uint32_t kHalfBytes = 128u * 128u;          // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kTileBytes = 2u * kHalfBytes;      // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + 2 * kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kTileBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kTileBytes;

enum {
  BAR_Q = 0,
  BAR_KF = 1,
  BAR_KE = BAR_KF + kStages,
  BAR_VF = BAR_KE + kStages,
  BAR_VE = BAR_VF + kStages,
  BAR_SF = BAR_VE + kStages,
  BAR_PF = BAR_SF + 2,
  BAR_OF = BAR_PF + 2,
  BAR_AB = BAR_OF + 1,
  NUM_BARS = BAR_AB + 1
};

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
  int n_list;
  int pad;
  int list[kMaxList];
  float bias[kMaxList];
};

constexpr uint32_t kSmemMisc = kSmemBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + sizeof(Misc) + 1024;   // + alignment slack

struct Params {
  int B, Hq, Hkv, N, nb, G;
  int rows_per_unit, tiles_per_unit, ctas_per_unit;
  const int* idx;
  int idx_stride;
  const float* sel;     // gated when non-null
  float scale_log2;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* status;
};

constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kRescaleThreshold = 8.0f;

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* ab, uint32_t* st) {
  bool ok = mbar_wait(bar, parity, ab, st);
  return __all_sync(0xffffffffu, ok);
}

// One softmax step for KEYS keys (64 or 128) of this thread's row.
template <int BS, int KEYS>
__device__ __forceinline__ void softmax_step(uint32_t t_s, uint32_t t_o, bool first, float scale_log2,
                                             float bias0, float bias1, bool diag0, bool diag1, int tb,
                                             float& m_run, float& l_run) {
  // pass 1: row maximum of the scaled, biased, masked logits
  float mx = -INFINITY;
#pragma unroll
  for (int ch = 0; ch < KEYS / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(t_s + ch * 32, v);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int c = ch * 32 + e;
      const bool second = (BS == 64) && (c >= 64);
      const int koff = (BS == 64) ? (c & 63) : c;
      float x = fmaf(__uint_as_float(v[e]), scale_log2, second ? bias1 : bias0);
      if ((second ? diag1 : diag0) && koff > tb) x = -INFINITY;
      mx = fmaxf(mx, x);
    }
  }
  const float m_new = fmaxf(m_run, mx);
  const bool need = m_new > m_run + kRescaleThreshold;
  const float m_use = need ? m_new : m_run;
  const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
  const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
  if (!first && __any_sync(0xffffffffu, need)) {
    // O row *= alpha (alpha == 1 for rows that keep their maximum)
#pragma unroll 1
    for (int ch = 0; ch < kD / 32; ++ch) {
      uint32_t v[32];
      tmem_ld32(t_o + ch * 32, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
      tmem_st32(t_o + ch * 32, v);
    }
  }
  l_run *= alpha;
  m_run = m_use;
  // pass 2: P = exp2(x - m), packed bf16 pairs written over S
  float sum = 0.0f;
#pragma unroll
  for (int ch = 0; ch < KEYS / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(t_s + ch * 32, v);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float p2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = ch * 32 + 2 * e + h;
        const bool second = (BS == 64) && (c >= 64);
        const int koff = (BS == 64) ? (c & 63) : c;
        float x = fmaf(__uint_as_float(v[2 * e + h]), scale_log2, second ? bias1 : bias0);
        if ((second ? diag1 : diag0) && koff > tb) x = -INFINITY;
        p2[h] = fast_exp2(x - m_sub);
        sum += p2[h];
      }
      pk[e] = pack_bf16x2(p2[0], p2[1]);
    }
    tmem_st16(t_s + ch * 16, pk);
  }
  l_run += sum;
  tmem_wait_st();
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + kSmemMisc);
  auto bar = [&](int b) -> uint32_t { return sbase + kSmemBar + 8u * b; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x / p.ctas_per_unit, pair = blockIdx.x % p.ctas_per_unit;
  const int bg = unit / p.nb;
  const int i = p.nb - 1 - unit % p.nb;   // heavy (late) query blocks first
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int tile0 = pair * 2;
  const int ntiles = min(2, p.tiles_per_unit - tile0);
  volatile int* abortp = &misc->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_KE + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(BAR_SF + t), 1);
      mbar_init(bar(BAR_PF + t), 128);
    }
    mbar_init(bar(BAR_OF), 1);
    mbar_init(bar(BAR_AB), 1);
    misc->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(sbase + kSmemMisc + offsetof(Misc, tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 2) {
    // kept-block list of this unit: ascending, ended by the first negative
    const int* src = p.idx + (static_cast<int64_t>(bg) * p.nb + i) * p.idx_stride;
    int count = 0, prev = -1;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < p.idx_stride; base += 32) {
      const int t = base + lane;
      const int j = (t < p.idx_stride) ? src[t] : -1;
      const unsigned neg = __ballot_sync(0xffffffffu, j < 0);
      const int lim = neg ? __ffs(neg) - 1 : 32;
      int jprev = __shfl_up_sync(0xffffffffu, j, 1);
      if (lane == 0) jprev = prev;
      const bool in = lane < lim;
      const bool ok = in && j <= i && j > jprev && count + lim <= kMaxList;
      if (in && !ok) atomicOr(p.status, BSA_DEV_BAD_INDEX);
      const unsigned okm = __ballot_sync(0xffffffffu, ok);
      if (ok) misc->list[count + __popc(okm & lt)] = j;
      count += __popc(okm);
      prev = __shfl_sync(0xffffffffu, j, 31);
      if (neg) break;
    }
    // gate: bias_t = log2(g_j) = (s_j - LSE_kept(s)) * log2(e)
    if (p.sel != nullptr && count > 0) {
      const float* srow = p.sel + (static_cast<int64_t>(bg) * p.nb + i) * p.nb;
      float mx = -INFINITY;
      for (int t = lane; t < count; t += 32) mx = fmaxf(mx, srow[misc->list[t]]);
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.0f;
      if (mx > -INFINITY)
        for (int t = lane; t < count; t += 32) sum += expf(srow[misc->list[t]] - mx);
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float lse_s = (mx > -INFINITY) ? mx + logf(sum) : 0.0f;
      for (int t = lane; t < count; t += 32)
        misc->bias[t] = (mx > -INFINITY) ? (srow[misc->list[t]] - lse_s) * kLog2e : 0.0f;
    } else {
      for (int t = lane; t < count; t += 32) misc->bias[t] = 0.0f;
    }
    if (lane == 0) misc->n_list = count;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = misc->tmem_base;
  const int n = misc->n_list;
  const int nsteps = (BS == 64) ? (n + 1) / 2 : n;

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------ TMA producer
      uint32_t qbytes = 0;
      for (int m = 0; m < ntiles; ++m)
        for (int pc = 0; pc < 2; ++pc)
          if ((tile0 + m) * 128 + pc * 64 < p.rows_per_unit) qbytes += 2 * 8192;
      mbar_arrive_expect_tx(bar(BAR_Q), qbytes);
      for (int m = 0; m < ntiles; ++m)
        for (int pc = 0; pc < 2; ++pc) {
          const int R0 = (tile0 + m) * 128 + pc * 64;
          if (R0 >= p.rows_per_unit) continue;
          const int h = g * p.G + R0 / BS;
          const int y = (b * p.Hq + h) * p.N + i * BS + R0 % BS;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(sbase + kSmemQ + m * kTileBytes + hf * kHalfBytes + pc * 8192, &tmQ, bar(BAR_Q),
                        hf * 64, y);
        }
      const int kvrow0 = bg * p.N;
      int k_issued = 0, v_issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const int slot = s % kStages, use = s / kStages;
        int jb[2];
        int nblk = 1;
        if (BS == 64) {
          jb[0] = misc->list[2 * s];
          nblk = (2 * s + 1 < n) ? 2 : 1;
          jb[1] = (nblk == 2) ? misc->list[2 * s + 1] : 0;
        } else {
          jb[0] = misc->list[s];
          jb[1] = 0;
        }
        const uint32_t bytes = static_cast<uint32_t>(nblk * BS) * 256u;
        // K
        if (s >= kStages && !mbar_wait(bar(BAR_KE + slot), (use - 1) & 1, abortp, p.status)) break;
        mbar_arrive_expect_tx(bar(BAR_KF + slot), bytes);
        for (int bl = 0; bl < nblk; ++bl)
          for (int r = 0; r < BS / 64; ++r) {
            const uint32_t rowoff = static_cast<uint32_t>(bl * BS + r * 64);
            const int y = kvrow0 + jb[bl] * BS + r * 64;
            for (int hf = 0; hf < 2; ++hf)
              tma_load_2d(sbase + kSmemK + slot * kTileBytes + hf * kHalfBytes + rowoff * 128u, &tmK,
                          bar(BAR_KF + slot), hf * 64, y);
          }
        ++k_issued;
        // V
        if (s >= kStages && !mbar_wait(bar(BAR_VE + slot), (use - 1) & 1, abortp, p.status)) break;
        mbar_arrive_expect_tx(bar(BAR_VF + slot), bytes);
        for (int bl = 0; bl < nblk; ++bl)
          for (int r = 0; r < BS / 64; ++r) {
            const uint32_t rowoff = static_cast<uint32_t>(bl * BS + r * 64);
            const int y = kvrow0 + jb[bl] * BS + r * 64;
            for (int hf = 0; hf < 2; ++hf)
              tma_load_2d(sbase + kSmemV + slot * kTileBytes + hf * kHalfBytes + rowoff * 128u, &tmV,
                          bar(BAR_VF + slot), hf * 64, y);
          }
        ++v_issued;
      }
      if (*abortp) {
        // let every copy this thread issued land before the CTA exits
        mbar_drain(bar(BAR_Q), 0);
        for (int s = max(0, k_issued - kStages); s < k_issued; ++s) mbar_drain(bar(BAR_KF + s % kStages), (s / kStages) & 1);
        for (int s = max(0, v_issued - kStages); s < v_issued; ++s) mbar_drain(bar(BAR_VF + s % kStages), (s / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s128 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s64 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
      auto keys_of = [&](int s) -> int { return (BS == 64) ? ((2 * s + 1 < n) ? 128 : 64) : 128; };
      auto issue_s = [&](int m, int slot, int keys) {
        const uint32_t qa = sbase + kSmemQ + m * kTileBytes;
        const uint32_t ka = sbase + kSmemK + slot * kTileBytes;
        const uint32_t id = (keys == 128) ? id_s128 : id_s64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem + m * 128, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), id,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int m, int slot, int keys, bool acc) {
        const uint32_t va = sbase + kSmemV + slot * kTileBytes;
        for (int kk = 0; kk < keys / 16; ++kk)
          mma_ts(tmem + 256 + m * 128, tmem + m * 128 + kk * 8,
                 smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(BAR_Q), 0, abortp, p.status);
      tc_fence_after();
      for (int s = 0; ok && s < nsteps; ++s) {
        const int slot = s % kStages, use = s / kStages;
        const int ps = s - 1, pslot = (s + kStages - 1) % kStages, puse = (s - 1) / kStages;
        if (!(ok = mbar_wait(bar(BAR_KF + slot), use & 1, abortp, p.status))) break;
        tc_fence_after();
        for (int m = 0; m < ntiles; ++m) {
          if (s > 0) {
            if (m == 0 && !(ok = mbar_wait(bar(BAR_VF + pslot), puse & 1, abortp, p.status))) break;
            if (!(ok = mbar_wait(bar(BAR_PF + m), ps & 1, abortp, p.status))) break;
            tc_fence_after();
            issue_pv(m, pslot, keys_of(ps), ps > 0);
          }
          issue_s(m, slot, keys_of(s));
          tc_commit(bar(BAR_SF + m));
        }
        if (!ok) break;
        if (s > 0) tc_commit(bar(BAR_VE + pslot));
        tc_commit(bar(BAR_KE + slot));
      }
      if (ok) {
        const int ls = nsteps - 1, lslot = ls % kStages;
        ok = mbar_wait(bar(BAR_VF + lslot), (ls / kStages) & 1, abortp, p.status);
        for (int m = 0; ok && m < ntiles; ++m) {
          if (!(ok = mbar_wait(bar(BAR_PF + m), ls & 1, abortp, p.status))) break;
          tc_fence_after();
          issue_pv(m, lslot, keys_of(ls), ls > 0);
        }
        if (ok) tc_commit(bar(BAR_OF));
      }
      if (!ok) {
        // every MMA issued so far must finish before tensor memory is freed
        tc_commit(bar(BAR_AB));
        mbar_drain(bar(BAR_AB), 0);
      }
    }
  } else if (warp >= 4 && (warp - 4) / 4 < ntiles) {
    // ------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) / 4;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int R = (tile0 + t) * 128 + r;
    const bool valid = R < p.rows_per_unit;
    const int hrow = g * p.G + (valid ? R / BS : 0);
    const int tb = R % BS;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t t_s = lane_addr + t * 128;
    const uint32_t t_o = lane_addr + 256 + t * 128;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      if (!(ok = warp_wait(bar(BAR_SF + t), s & 1, abortp, p.status))) break;
      tc_fence_after();
      int j0, j1 = -1, keys = 128;
      float b0, b1 = 0.0f;
      if (BS == 64) {
        j0 = misc->list[2 * s];
        b0 = misc->bias[2 * s];
        if (2 * s + 1 < n) {
          j1 = misc->list[2 * s + 1];
          b1 = misc->bias[2 * s + 1];
        } else {
          keys = 64;
        }
      } else {
        j0 = misc->list[s];
        b0 = misc->bias[s];
      }
      if (keys == 128)
        softmax_step<BS, 128>(t_s, t_o, s == 0, p.scale_log2, b0, b1, j0 == i, j1 == i, tb, m_run, l_run);
      else
        softmax_step<BS, 64>(t_s, t_o, s == 0, p.scale_log2, b0, b1, j0 == i, false, tb, m_run, l_run);
      tc_fence_before();
      mbar_arrive(bar(BAR_PF + t));
    }
    __nv_bfloat16* orow = p.o + ((static_cast<int64_t>(b) * p.Hq + hrow) * p.N + i * BS + tb) * kD;
    if (n == 0) {
      if (valid) {
        for (int c = 0; c < kD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[(static_cast<int64_t>(b) * p.Hq + hrow) * p.N + i * BS + tb] = -INFINITY;
      }
    } else if (ok && warp_wait(bar(BAR_OF), 0, abortp, p.status)) {
      tc_fence_after();
      const float inv = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
#pragma unroll 1
      for (int ch = 0; ch < kD / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(t_o + ch * 32, v);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (valid && p.lse)
        p.lse[(static_cast<int64_t>(b) * p.Hq + hrow) * p.N + i * BS + tb] =
            (l_run > 0.0f) ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BS>
static cudaError_t launch_bs(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const Params& p, unsigned grid, cudaStream_t st) {
  static bool configured = false;   // attribute is per-function; idempotent, so a race is harmless
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  attn_prefill_kernel<BS><<<grid, kThreads, kSmemBytes, st>>>(*tmQ, *tmK, *tmV, p);
  return cudaGetLastError();
}

}  // namespace prefill

cudaError_t launch_attn_prefill_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                     const PrefillArgs& a, cudaStream_t st) {
  prefill::Params p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.N = a.N;
  p.nb = a.N / a.bs;
  p.G = a.Hq / a.Hkv;
  p.rows_per_unit = p.G * a.bs;
  p.tiles_per_unit = (p.rows_per_unit + 127) / 128;
  p.ctas_per_unit = (p.tiles_per_unit + 1) / 2;
  p.idx = a.idx;
  p.idx_stride = a.idx_stride;
  p.sel = a.sel_scores;
  p.scale_log2 = a.softmax_scale * prefill::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.status = a.status;
  const int64_t grid = static_cast<int64_t>(a.B) * a.Hkv * p.nb * p.ctas_per_unit;
  if (grid <= 0) return cudaSuccess;
  if (a.bs == 64) return prefill::launch_bs<64>(tmQ, tmK, tmV, p, static_cast<unsigned>(grid), st);
  return prefill::launch_bs<128>(tmQ, tmK, tmV, p, static_cast<unsigned>(grid), st);
}

}  // namespace bsa
