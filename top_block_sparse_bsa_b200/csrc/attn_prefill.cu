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
// each are stacked into G*bs rows that all read the same K/V tiles.  An item
// is two 128-row tiles of one unit ("ping-pong": while one tile's softmax
// runs on CUDA cores, the tensor core works on the other tile), so each K/V
// tile is fetched into shared memory once for 256 query rows.  Units with an
// odd number of tiles go to the split-half kernel (attn_prefill_split.cu),
// which runs one tile per item with two S buffers.  The kernel is
// persistent: one CTA per SM walks items blockIdx.x, +gridDim.x, ... (heavy
// items first); the K/V ring, the item metadata and the Q buffer roll over
// from one item to the next, so the next item's loads and first MMAs overlap
// the previous item's tail and epilogue.
//
// Roles (384 threads, three warpgroups):
//   warp 0      TMA producer of Q (per item) and K (per step, two-stage
//               ring, gathered by block index);
//   warp 3      TMA producer of V (per step, two-stage ring): a separate
//               thread, because the K ring drains after S and the V ring
//               after O += P V;
//   warp 1      TMEM owner + MMA issuer (one thread): S = Q K^T (SS form),
//               O += P V (TS form, P read from tensor memory); per step it
//               issues O += P V of the previous step before S of this one,
//               tile by tile;
//   warp 2      item loader: kept-block list and gate biases into a
//               double-buffered metadata slot;
//   warps 4-7   softmax + epilogue of tile 0 (thread = query row = TMEM lane);
//   warps 8-11  softmax + epilogue of tile 1.
// The control warpgroup gives registers up (setmaxnreg) to the two softmax
// warpgroups, which hold a whole 128-column S row in registers.
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each; P (bf16
// pairs) is written over the first half of its S region.  tcgen05.mma
// instructions from one thread execute in issue order, so S(t, s+1), issued
// after O += P(t, s) V, never overwrites P before that MMA has read it.
//
// A step covers 128 keys: two 64-token blocks (bs = 64) or one 128-token
// block (bs = 128); the last step of an odd list holds one 64-token block.
//
// Softmax uses the base-2 exponent with the scale and the gate bias folded
// into one packed (f32x2) FMA per key pair, and a lazy rescale: the running maximum is only moved (and O
// rescaled in tensor memory) when a row's new maximum exceeds it by more than
// 8 (a factor 256), which keeps every P <= 256 and is exact after the final
// division.
#include "common.cuh"
#include "kernels.h"
#include "tmem_wide.cuh"

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
constexpr int kCtrlRegs = 96;       // warps 0-3 after setmaxnreg.dec
constexpr int kMathRegs = 200;      // warps 4-11 after setmaxnreg.inc (128*96 + 256*200 <= 384*168)

enum {
  BAR_QF = 0,
  BAR_QE,
  BAR_KF,
  BAR_KE = BAR_KF + kStages,
  BAR_VF = BAR_KE + kStages,
  BAR_VE = BAR_VF + kStages,
  BAR_SF = BAR_VE + kStages,   // per tile
  BAR_PF = BAR_SF + 2,         // per tile
  BAR_OF = BAR_PF + 2,         // per tile: final O of an item ready
  BAR_OE = BAR_OF + 2,         // per tile: O read back, free for the next item
  BAR_LF = BAR_OE + 2,         // per metadata slot: filled
  BAR_LE = BAR_LF + 2,         // per metadata slot: consumed by every role
  BAR_AB = BAR_LE + 2,
  NUM_BARS
};
constexpr uint32_t kListConsumers = 3 + 8;   // two producers, MMA, one lane per softmax warp

struct ItemInfo {
  int n, ntiles, b, g, i, tile0, pad0, pad1;
  int list[kMaxList];
  float bias[kMaxList];
};

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
  int pad[2];
  ItemInfo info[2];
};

constexpr uint32_t kSmemMisc = kSmemBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + sizeof(Misc) + 1024;   // + alignment slack

struct Params {
  int B, Hq, Hkv, N, nb, G;
  int rows_per_unit, tiles_per_unit, ctas_per_unit, num_items;
  const int* idx;
  int idx_stride;
  const float* sel;     // gated when non-null
  float scale_log2;
  __nv_bfloat16* o;
  int o_v8;             // o is 32-byte aligned: 256-bit row stores
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

template <int N>
__device__ __forceinline__ void set_regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void set_regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// One softmax step over KEYS keys (64 or 128) of this thread's row.  MASK:
// the step holds the query block itself (causal mask inside it).
template <int BS, int KEYS, bool MASK>
__device__ __forceinline__ void softmax_step(uint32_t t_s, uint32_t t_o, bool first, float scale_log2, float bias0,
                                             float bias1, bool diag0, bool diag1, int tb, float& m_run,
                                             float& l_run) {
  uint32_t v[KEYS];
  constexpr int H0 = (BS == 64 && KEYS == 128) ? 64 : KEYS;
  auto mask_range = [&](int c0, int c1) {
    if constexpr (MASK) {
#pragma unroll
      for (int c = c0; c < c1; ++c) {
        const bool second = (BS == 64) && (c >= 64);
        const int koff = (BS == 64) ? (c & 63) : c;
        if ((second ? diag1 : diag0) && koff > tb) v[c] = 0xFF800000u;   // -inf
      }
    }
  };
  // row maximum of the raw scores per block (the scale is positive and the
  // bias is constant over a block, so the maximum commutes with both);
  // three-input maxima in 8 independent chains
  float m8[8];
  auto max_init = [&]() {
#pragma unroll
    for (int a = 0; a < 8; ++a) m8[a] = -INFINITY;
  };
  auto max_acc = [&](int c0, int c1) {
#pragma unroll
    for (int c = c0; c < c1; c += 2)
      m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
  };
  auto max_fin = [&]() {
    return fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
  };
  float mx0, mx1 = -INFINITY;
  if constexpr (KEYS == 128) {
    // first 64 columns, then the second 64 in flight while the first are reduced
    uint32_t(&lo)[64] = *reinterpret_cast<uint32_t(*)[64]>(&v[0]);
    uint32_t(&hi)[64] = *reinterpret_cast<uint32_t(*)[64]>(&v[64]);
    tmem_ld64(t_s, lo);
    tmem_ld64_nowait(t_s + 64, hi);
    mask_range(0, 64);
    max_init();
    max_acc(0, 64);
    if constexpr (H0 < KEYS) {
      mx0 = max_fin();
      max_init();
    }
    tmem_wait_ld_tied64(hi);
    mask_range(64, 128);
    max_acc(64, 128);
    if constexpr (H0 < KEYS) mx1 = max_fin();
    else mx0 = max_fin();
  } else {
    tmem_ld64(t_s, reinterpret_cast<uint32_t(&)[64]>(v));
    mask_range(0, KEYS);
    max_init();
    max_acc(0, KEYS);
    mx0 = max_fin();
  }
  float mx = fmaf(mx0, scale_log2, bias0);
  if constexpr (H0 < KEYS) mx = fmaxf(mx, fmaf(mx1, scale_log2, bias1));
  const float m_new = fmaxf(m_run, mx);
  const bool need = m_new > m_run + kRescaleThreshold;
  const float m_use = need ? m_new : m_run;
  const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
  const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
  if (!first && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
    for (int ch = 0; ch < kD / 32; ++ch) {
      uint32_t o[32];
      tmem_ld32(t_o + ch * 32, o);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      tmem_st32(t_o + ch * 32, o);
    }
  }
  l_run *= alpha;
  m_run = m_use;
  // p = 2^(s * scale*log2(e) + bias - m), two keys per packed FMA; packed
  // partial row sums
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t off0 = f2_pack(bias0 - m_sub, bias0 - m_sub), off1 = f2_pack(bias1 - m_sub, bias1 - m_sub);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // independent packed partial row sums (+0.0f pairs)
#pragma unroll
  for (int half = 0; half < KEYS / 64; ++half) {
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int c = half * 64 + 2 * e;
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2,
                                (c < H0) ? off0 : off1);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
      acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
      pk[e] = pack_bf16x2(p0, p1);
    }
    tmem_st32(t_s + half * 32, pk);
  }
  float a0, a1, a2, a3;
  f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
  f2_unpack(f2_add(acc[2], acc[3]), a2, a3);
  l_run += (a0 + a1) + (a2 + a3);
  tmem_wait_st();
}

template <int BS>
__device__ __forceinline__ void softmax_dispatch(int keys, bool has_diag, uint32_t t_s, uint32_t t_o, bool first,
                                                 float scale_log2, float b0, float b1, bool d0, bool d1, int tb,
                                                 float& m_run, float& l_run) {
  if (keys == 128) {
    if (has_diag)
      softmax_step<BS, 128, true>(t_s, t_o, first, scale_log2, b0, b1, d0, d1, tb, m_run, l_run);
    else
      softmax_step<BS, 128, false>(t_s, t_o, first, scale_log2, b0, b1, d0, d1, tb, m_run, l_run);
  } else {
    if (has_diag)
      softmax_step<BS, 64, true>(t_s, t_o, first, scale_log2, b0, b1, d0, false, tb, m_run, l_run);
    else
      softmax_step<BS, 64, false>(t_s, t_o, first, scale_log2, b0, b1, d0, false, tb, m_run, l_run);
  }
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
  volatile int* abortp = &misc->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_QF), 1);
    mbar_init(bar(BAR_QE), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_KE + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(BAR_SF + t), 1);
      mbar_init(bar(BAR_PF + t), 4);    // one arrive per softmax warp
      mbar_init(bar(BAR_OF + t), 1);
      mbar_init(bar(BAR_OE + t), 4);
      mbar_init(bar(BAR_LF + t), 1);
      mbar_init(bar(BAR_LE + t), kListConsumers);
    }
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;

  if (warp < 4) {
  set_regs_dec<kCtrlRegs>();
  if (warp == 2) {
    // ------------------------------------------------ item loader
    const unsigned lt = (1u << lane) - 1u;
    for (int k = 0;; ++k) {
      const int item = blockIdx.x + k * gridDim.x;
      if (item >= p.num_items) break;
      const int buf = k & 1;
      if (k >= 2 && !warp_wait(bar(BAR_LE + buf), ((k >> 1) - 1) & 1, abortp, p.status)) break;
      ItemInfo* inf = &misc->info[buf];
      const int unit = item / p.ctas_per_unit, pair = item % p.ctas_per_unit;
      const int bg = unit / p.nb;
      const int i = p.nb - 1 - unit % p.nb;   // heavy (late) query blocks first
      const int* src = p.idx + (static_cast<int64_t>(bg) * p.nb + i) * p.idx_stride;
      int count = 0, prev = -1;
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
        if (ok) inf->list[count + __popc(okm & lt)] = j;
        count += __popc(okm);
        prev = __shfl_sync(0xffffffffu, j, 31);
        if (neg) break;
      }
      __syncwarp();
      // gate: bias_t = log2(g_j) = (s_j - LSE_kept(s)) * log2(e)
      if (p.sel != nullptr && count > 0) {
        const float* srow = p.sel + (static_cast<int64_t>(bg) * p.nb + i) * p.nb;
        float mx = -INFINITY;
        for (int t = lane; t < count; t += 32) mx = fmaxf(mx, srow[inf->list[t]]);
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.0f;
        if (mx > -INFINITY)
          for (int t = lane; t < count; t += 32) sum += expf(srow[inf->list[t]] - mx);
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float lse_s = (mx > -INFINITY) ? mx + logf(sum) : 0.0f;
        for (int t = lane; t < count; t += 32)
          inf->bias[t] = (mx > -INFINITY) ? (srow[inf->list[t]] - lse_s) * kLog2e : 0.0f;
      } else {
        for (int t = lane; t < count; t += 32) inf->bias[t] = 0.0f;
      }
      if (lane == 0) {
        inf->n = count;
        inf->ntiles = min(2, p.tiles_per_unit - pair * 2);
        inf->b = bg / p.Hkv;
        inf->g = bg % p.Hkv;
        inf->i = i;
        inf->tile0 = pair * 2;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LF + buf));
    }
  } else if (warp == 0 || warp == 3) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producers
      // warp 0 loads Q and K, warp 3 loads V: the two rings drain at
      // different points of the MMA order (K after S, V after O += P V), so
      // separate threads keep a late V slot from holding back the next K.
      const int kv = (warp == 3) ? 1 : 0;
      const int full = kv ? BAR_VF : BAR_KF, empty = kv ? BAR_VE : BAR_KE;
      const CUtensorMap* map = kv ? &tmV : &tmK;
      const uint32_t ring = sbase + (kv ? kSmemV : kSmemK);
      int gs = 0, qcount = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int ntiles = inf->ntiles, tile0 = inf->tile0, b = inf->b, g = inf->g, i = inf->i;
          if (kv == 0) {
            if (qcount > 0 && !(ok = mbar_wait(bar(BAR_QE), (qcount - 1) & 1, abortp, p.status))) break;
            uint32_t qbytes = 0;
            for (int m = 0; m < ntiles; ++m)
              for (int pc = 0; pc < 2; ++pc)
                if ((tile0 + m) * 128 + pc * 64 < p.rows_per_unit) qbytes += 2 * 8192;
            mbar_arrive_expect_tx(bar(BAR_QF), qbytes);
            for (int m = 0; m < ntiles; ++m)
              for (int pc = 0; pc < 2; ++pc) {
                const int R0 = (tile0 + m) * 128 + pc * 64;
                if (R0 >= p.rows_per_unit) continue;
                const int h = g * p.G + R0 / BS;
                const int y = (b * p.Hq + h) * p.N + i * BS + R0 % BS;
                for (int hf = 0; hf < 2; ++hf)
                  tma_load_2d(sbase + kSmemQ + m * kTileBytes + hf * kHalfBytes + pc * 8192, &tmQ, bar(BAR_QF),
                              hf * 64, y);
              }
            ++qcount;
          }
          const int kvrow0 = (b * p.Hkv + g) * p.N;
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int slot = gs % kStages, use = gs / kStages;
            int jb[2];
            int nblk = 1;
            if (BS == 64) {
              jb[0] = inf->list[2 * s];
              nblk = (2 * s + 1 < n) ? 2 : 1;
              jb[1] = (nblk == 2) ? inf->list[2 * s + 1] : 0;
            } else {
              jb[0] = inf->list[s];
              jb[1] = 0;
            }
            if (gs >= kStages && !(ok = mbar_wait(bar(empty + slot), (use - 1) & 1, abortp, p.status))) break;
            mbar_arrive_expect_tx(bar(full + slot), static_cast<uint32_t>(nblk * BS) * 256u);
            const uint32_t dst0 = ring + slot * kTileBytes;
            for (int bl = 0; bl < nblk; ++bl)
              for (int r = 0; r < BS / 64; ++r) {
                const uint32_t rowoff = static_cast<uint32_t>(bl * BS + r * 64);
                const int y = kvrow0 + jb[bl] * BS + r * 64;
                for (int hf = 0; hf < 2; ++hf)
                  tma_load_2d(dst0 + hf * kHalfBytes + rowoff * 128u, map, bar(full + slot), hf * 64, y);
              }
          }
          if (!ok) break;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (*abortp) {
        // let every copy this thread issued land before the CTA exits
        if (qcount > 0) mbar_drain(bar(BAR_QF), (qcount - 1) & 1);
        for (int s = max(0, gs - kStages); s < gs; ++s) mbar_drain(bar(full + s % kStages), (s / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s128 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s64 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
      // Descriptors are built once; a k-step only adds its byte offset (>> 4)
      // to the start-address field, so issuing an MMA is one add and the MMA.
      const uint64_t q_desc0 = smem_desc_sw128(sbase + kSmemQ, 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(sbase + kSmemK, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(sbase + kSmemV, kHalfBytes, 1024);
      auto issue_s = [&](int m, int slot, int keys) {
        const uint64_t qd = q_desc0 + ((m * kTileBytes) >> 4);
        const uint64_t kd = k_desc0 + ((slot * kTileBytes) >> 4);
        const uint32_t id = (keys == 128) ? id_s128 : id_s64;
        const uint32_t d_tmem = tmem + m * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss(d_tmem, qd + off, kd + off, id, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int m, int slot, int keys, bool acc) {
        const uint64_t vd = v_desc0 + ((slot * kTileBytes) >> 4);
        const uint32_t d_tmem = tmem + 256 + m * 128;
        const uint32_t a_tmem = tmem + m * 128;
        if (keys == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(d_tmem, a_tmem + kk * 8, vd + ((kk * 2048) >> 4), id_pv, (acc || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(d_tmem, a_tmem + kk * 8, vd + ((kk * 2048) >> 4), id_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      int gs = 0, qcount = 0;
      int st[2] = {0, 0};        // completed S/P steps per tile
      int pv_items[2] = {0, 0};  // items whose O has been produced, per tile
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int ntiles = inf->ntiles;
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          auto keys_of = [&](int s) -> int { return (BS == 64) ? ((2 * s + 1 < n) ? 128 : 64) : 128; };
          if (!(ok = mbar_wait(bar(BAR_QF), qcount & 1, abortp, p.status))) break;
          ++qcount;
          tc_fence_after();
          for (int s = 0; ok && s < nsteps; ++s, ++gs) {
            const int slot = gs % kStages, use = gs / kStages;
            const int pslot = (gs + kStages - 1) % kStages, puse = (gs - 1) / kStages;
            bool have_k = false;
            for (int m = 0; m < ntiles; ++m) {
              if (s > 0) {
                // O += P V of the previous step first: it needs V and P, not K
                if (m == 0 && !(ok = mbar_wait(bar(BAR_VF + pslot), puse & 1, abortp, p.status))) break;
                if (!(ok = mbar_wait(bar(BAR_PF + m), (st[m] - 1) & 1, abortp, p.status))) break;
                if (s == 1 && pv_items[m] > 0 &&
                    !(ok = mbar_wait(bar(BAR_OE + m), (pv_items[m] - 1) & 1, abortp, p.status)))
                  break;
                tc_fence_after();
                issue_pv(m, pslot, keys_of(s - 1), s - 1 > 0);
                // the V slot is free as soon as the last tile's O += P V is done
                if (m == ntiles - 1) tc_commit(bar(BAR_VE + pslot));
              }
              if (!have_k) {
                if (!(ok = mbar_wait(bar(BAR_KF + slot), use & 1, abortp, p.status))) break;
                tc_fence_after();
                have_k = true;
              }
              issue_s(m, slot, keys_of(s));
              tc_commit(bar(BAR_SF + m));
              ++st[m];
            }
            if (!ok) break;
            tc_commit(bar(BAR_KE + slot));
          }
          if (!ok) break;
          tc_commit(bar(BAR_QE));   // Q is free once this item's S MMAs complete
          const int ls = nsteps - 1, lg = gs - 1, lslot = lg % kStages;
          if (!(ok = mbar_wait(bar(BAR_VF + lslot), (lg / kStages) & 1, abortp, p.status))) break;
          for (int m = 0; ok && m < ntiles; ++m) {
            if (!(ok = mbar_wait(bar(BAR_PF + m), (st[m] - 1) & 1, abortp, p.status))) break;
            if (ls == 0 && pv_items[m] > 0 &&
                !(ok = mbar_wait(bar(BAR_OE + m), (pv_items[m] - 1) & 1, abortp, p.status)))
              break;
            tc_fence_after();
            issue_pv(m, lslot, keys_of(ls), ls > 0);
            tc_commit(bar(BAR_OF + m));
            ++pv_items[m];
          }
          if (!ok) break;
          tc_commit(bar(BAR_VE + lslot));
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (!ok) {
        // every MMA issued so far must finish before tensor memory is freed
        tc_commit(bar(BAR_AB));
        mbar_drain(bar(BAR_AB), 0);
      }
    }
  }
  } else {
    set_regs_inc<kMathRegs>();
    // ------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) / 4;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t t_s = lane_addr + t * 128;
    const uint32_t t_o = lane_addr + 256 + t * 128;
    int st = 0, oc = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = blockIdx.x + k * gridDim.x;
      if (item >= p.num_items) break;
      const int buf = k & 1;
      if (!(ok = warp_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
      const ItemInfo* inf = &misc->info[buf];
      const int n = inf->n, ntiles = inf->ntiles;
      const int b = inf->b, g = inf->g, i = inf->i;
      const int R = (inf->tile0 + t) * 128 + r;
      const bool valid = (t < ntiles) && R < p.rows_per_unit;
      const int hrow = g * p.G + (valid ? R / BS : 0);
      const int tb = R % BS;
      const int64_t orow_idx = (static_cast<int64_t>(b) * p.Hq + hrow) * p.N + i * BS + tb;
      if (t < ntiles && n == 0) {
        if (valid) {
          __nv_bfloat16* orow = p.o + orow_idx * kD;
          for (int c = 0; c < kD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[orow_idx] = -INFINITY;
        }
      } else if (t < ntiles) {
        const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
        float m_run = -INFINITY, l_run = 0.0f;
        for (int s = 0; s < nsteps; ++s, ++st) {
          if (!(ok = warp_wait(bar(BAR_SF + t), st & 1, abortp, p.status))) break;
          tc_fence_after();
          int j0, j1 = -1, keys = 128;
          float b0, b1 = 0.0f;
          if (BS == 64) {
            j0 = inf->list[2 * s];
            b0 = inf->bias[2 * s];
            if (2 * s + 1 < n) {
              j1 = inf->list[2 * s + 1];
              b1 = inf->bias[2 * s + 1];
            } else {
              keys = 64;
            }
          } else {
            j0 = inf->list[s];
            b0 = inf->bias[s];
          }
          softmax_dispatch<BS>(keys, j0 == i || j1 == i, t_s, t_o, s == 0, p.scale_log2, b0, b1, j0 == i, j1 == i,
                               tb, m_run, l_run);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_PF + t));
        }
        if (!ok) break;
        if (!(ok = warp_wait(bar(BAR_OF + t), oc & 1, abortp, p.status))) break;
        ++oc;
        tc_fence_after();
        // read O back (packed to bf16 pairs right away), then free O for the next item
        const float inv = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
        uint32_t ob[64];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          tmem_ld32(t_o + ch * 32, v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            ob[ch * 16 + e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_OE + t));   // O may be overwritten by the next item from here on
        if (valid) {
          if (p.o_v8) {   // whole 32-byte sectors per store
#pragma unroll
            for (int e = 0; e < 8; ++e) st_global_v8(p.o + orow_idx * kD + 16 * e, ob + 8 * e);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.o + orow_idx * kD);
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2], ob[4 * e + 3]);
          }
          if (p.lse) p.lse[orow_idx] = (l_run > 0.0f) ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LE + buf));
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
  cudaError_t e = ensure_dynamic_smem<attn_prefill_kernel<BS>>(kSmemBytes);
  if (e != cudaSuccess) return e;
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
  if (a.kernel == 3) return launch_attn_prefill_pair_bf16(tmQ, tmK, tmV, a, st);
  // an odd tile count would leave one tile per unit without a partner
  if (a.kernel == 2 || (a.kernel == 0 && p.tiles_per_unit % 2 == 1))
    return launch_attn_prefill_split_bf16(tmQ, tmK, tmV, a, st);
  p.ctas_per_unit = (p.tiles_per_unit + 1) / 2;
  const int64_t items = static_cast<int64_t>(a.B) * a.Hkv * p.nb * p.ctas_per_unit;
  if (items <= 0) return cudaSuccess;
  p.num_items = static_cast<int>(items);
  p.idx = a.idx;
  p.idx_stride = a.idx_stride;
  p.sel = a.sel_scores;
  p.scale_log2 = a.softmax_scale * prefill::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) & 31u) == 0 ? 1 : 0;
  p.lse = a.lse;
  p.status = a.status;
  const unsigned grid = static_cast<unsigned>(items < a.num_sms ? items : a.num_sms);
  if (a.bs == 64) return prefill::launch_bs<64>(tmQ, tmK, tmV, p, grid, st);
  return prefill::launch_bs<128>(tmQ, tmK, tmV, p, grid, st);
}

}  // namespace bsa
