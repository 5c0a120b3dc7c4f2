// attn_decode.cu -- sparse decode attention over a retained KV cache, and the
// SSA gist-expansion decode, bf16, d = 128, on sm_100a tensor cores.
//
// What it computes (source pages): for one new query token per sequence,
// softmax(q K^T/sqrt(d)) V over the tokens of the kept blocks only ("稀疏注意力"
// tutorial §5: decode reads the history; Sparse Frontier review §2.4.2: the
// full cache is retained and only the selected pages are loaded).  In gist
// mode (SSA page, 推理时的关键模块 2-3) the key set of query head h is the
// tokens of the chunks h expanded plus the gist key/value of every chunk it
// did not expand.
//
// Work decomposition.  All G query heads of a KV group read the same kept
// blocks (decode) or the union of their expanded chunks (gist), so each
// 64-token tile is gathered once for the whole group.  The MMAs are "swapped":
// the 128 keys of a step are the M dimension and the group's heads (padded to
// 16) the N dimension, S^T = K Q^T and O^T += V^T P^T, so one softmax thread
// owns one key and evaluates only G exponentials per step.  Split-K: the
// groups' tile lists are laid end to end and cut into equal contiguous
// ranges, one per persistent CTA (about one per SM), so every CTA streams the
// same number of tiles through its TMA ring; a CTA's range covers one to a few
// row segments, and each segment writes an unnormalised partial (running max
// m, sum l, O) per head; a second kernel merges a row's segments.
//
// Roles (256 threads): warps 0-3 softmax (TMEM lanes 0-127 = the step's keys)
// and epilogue (lanes = channels of O^T), warp 4 TMA producer, warp 5 TMEM
// owner + MMA issuer, warp 6 slice loader.  Tensor memory: two S^T buffers
// (16 columns each) and O^T (16 columns).  The four softmax warps exchange
// per-head maxima through shared memory with mbarrier hand-offs (bounded
// waits, never bar.sync, so an abort cannot strand a warp).
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace decode {

constexpr int kD = 128;
constexpr int kNH = 16;                 // query heads of a group, padded (MMA N)
constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kMaxItemTiles = 128;      // tiles one item may own
constexpr uint32_t kHalfBytes = 128u * 128u;          // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2u * kHalfBytes;      // 128 rows x 128 bf16 (one step of K or V)
constexpr uint32_t kSmallHalf = 16u * 128u;           // 16 rows x 64 bf16
constexpr uint32_t kSmallBytes = 2u * kSmallHalf;     // Q^T or P^T buffer
constexpr uint32_t kSmemK = 0;
constexpr uint32_t kSmemV = kSmemK + kStages * kTileBytes;
constexpr uint32_t kSmemQ = kSmemV + kStages * kTileBytes;   // 2 buffers
constexpr uint32_t kSmemP = kSmemQ + 2 * kSmallBytes;        // 2 buffers
constexpr uint32_t kSmemBar = kSmemP + 2 * kSmallBytes;

enum {
  BAR_KF = 0,
  BAR_KE = BAR_KF + kStages,
  BAR_VF = BAR_KE + kStages,
  BAR_VE = BAR_VF + kStages,
  BAR_QF = BAR_VE + kStages,   // per Q buffer
  BAR_QE = BAR_QF + 2,
  BAR_SF = BAR_QE + 2,         // per S buffer
  BAR_SE = BAR_SF + 2,
  BAR_PF = BAR_SE + 2,         // per P buffer
  BAR_PE = BAR_PF + 2,
  BAR_OD = BAR_PE + 2,         // one completion per O += V^T P^T
  BAR_OF = BAR_OD + 1,         // per item: O complete
  BAR_OE = BAR_OF + 1,         // per item: O read back
  BAR_LF = BAR_OE + 1,         // per metadata slot
  BAR_LE = BAR_LF + 2,
  BAR_RX = BAR_LE + 2,         // cross-warp tile-maximum exchange, by step parity
  BAR_LX = BAR_RX + 2,         // cross-warp row-sum exchange, by epilogue parity
  BAR_AB = BAR_LX + 2,
  NUM_BARS
};
constexpr uint32_t kListConsumers = 2 + 4;   // producer, MMA, one lane per softmax warp

constexpr int kUnionWords = 64;         // fused gist union: up to 2048 chunks per row
struct ItemInfo {
  int n, b, g, bg, slot, pad0, pad1, pad2;
  int tiles[kMaxItemTiles];
  uint32_t bits[kNH + 1][kUnionWords];   // fused gist union: heads' expanded chunks, then the union
};

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
  int pad[2];
  float red[2][4][kNH];    // per-warp tile maxima, double-buffered by step parity
  float lred[2][4][kNH];   // per-warp row sums at the end of an item, by epilogue parity
  ItemInfo info[2];
};
constexpr uint32_t kSmemMisc = kSmemBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + sizeof(Misc) + 1024;
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the sm_100 per-CTA limit");

constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kRescaleThreshold = 8.0f;
// partial record per (row, split): m, l, 2 pad, then O (16-byte aligned)
constexpr int kRec = kD + 4;

struct Params {
  int B, Hq, Hkv, Nk, G, nc;
  const int* list;
  int list_stride;
  int list_has_count;
  const uint32_t* expanded;
  int list_len;        // positions per group row (the split space is rows x list_len)
  int64_t total;       // rows * list_len
  int num_ctas;        // CTAs sharing the split space
  int max_slots;       // partial records per head
  float scale_log2;
  float* partial;
  uint32_t* status;
  // paged cache (plain decode only): logical block j of sequence b lives in
  // physical block table[b * table_stride + j] of the pools [P][Hkv][64][d]
  const int* table;
  int table_stride, num_pages;
  // gist decode with the union built in the kernel (nc <= 2048): the heads'
  // kept chunk lists [B*Hq][heads_stride] (heads_topk entries, -1 = none);
  // null: list/expanded hold a union built by gist_union_kernel
  const int* heads_idx;
  int heads_topk, heads_stride;
  // two-level gists (H-SSA): gist tiles at or past nc/64 are meta-gist tiles
  // (rows bg*meta_rows + ..., of the meta maps); gist_allow [B*Hq][(nc+64)/32]
  // says per head which gist / meta-gist rows it attends (null: SSA's rule,
  // the gist of every chunk the head did not expand)
  const uint32_t* gist_allow;
  int meta_rows;
};

// The split space is every group row's list positions laid end to end; CTA c
// owns positions [c*total/C, (c+1)*total/C).  cta_of(x) is the CTA owning x.
__host__ __device__ __forceinline__ int cta_of(int64_t x, int64_t total, int C) {
  return static_cast<int>(((x + 1) * C + total - 1) / total) - 1;
}

// Number of row segments (work items) of this CTA, and its first row.
__device__ __forceinline__ int cta_items(const Params& p, int c, int* r0) {
  const int64_t lo = static_cast<int64_t>(c) * p.total / p.num_ctas;
  const int64_t hi = static_cast<int64_t>(c + 1) * p.total / p.num_ctas;
  if (lo >= hi) return 0;
  *r0 = static_cast<int>(lo / p.list_len);
  return static_cast<int>((hi - 1) / p.list_len) - *r0 + 1;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* ab, uint32_t* st) {
  bool ok = mbar_wait(bar, parity, ab, st);
  return __all_sync(0xffffffffu, ok);
}

// Softmax role (warps 0-3), specialised on GH >= G query heads per group:
// only GH columns of S^T and O^T are read, reduced and written.
template <int GH>
__device__ __forceinline__ void softmax_role(const Params& p, Misc* misc, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                                             volatile int* abortp, int warp, int lane, bool gist) {
  auto bar = [&](int b) -> uint32_t { return sbase + kSmemBar + 8u * b; };
    const int r = warp * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    int s_read = 0, p_written = 0, od_seen = 0, items_done = 0, rx = 0;
    bool ok = true;
    int r0 = 0;
    const int nitems = cta_items(p, blockIdx.x, &r0);
    for (int k = 0; ok && k < nitems; ++k) {
      const int buf = k & 1;
      if (!(ok = warp_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
      const ItemInfo* inf = &misc->info[buf];
      const int n = inf->n, G = p.G;
      const int b = inf->b, g = inf->g;
      float* part_base = p.partial + (static_cast<int64_t>(inf->bg) * G * p.max_slots + inf->slot) * kRec;
      const int64_t head_stride = static_cast<int64_t>(p.max_slots) * kRec;
      if (n == 0) {
        // empty slice: m = -inf, l = 0, O = 0
        for (int h = 0; h < G; ++h) {
          float* part = part_base + h * head_stride;
          if (r == 0) {
            part[0] = -INFINITY;
            part[1] = 0.0f;
          }
          part[4 + r] = 0.0f;
        }
      } else {
        const bool fused = p.heads_idx != nullptr;
        const uint32_t* bits_base =
            fused ? &inf->bits[0][0]
                  : (gist ? p.expanded + (static_cast<int64_t>(b) * p.Hq + g * G) * (p.nc / 32) : nullptr);
        const bool two_level = p.gist_allow != nullptr;
        const int words_g = (p.nc + 64) / 32;
        const uint32_t* allow_base =
            two_level ? p.gist_allow + (static_cast<int64_t>(b) * p.Hq + g * G) * words_g : nullptr;
        float m_run[GH], l_part[GH];
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          m_run[h] = -INFINITY;
          l_part[h] = 0.0f;
        }
        const int nsteps = (n + 1) / 2;
        const int words = p.nc / 32;
        for (int s = 0; s < nsteps; ++s) {
          const int sb = s_read & 1;
          // this thread's key r lies in one tile of the step; in gist mode
          // its allowance per head is one bit of that head's expanded-chunk
          // bitmap, loaded here so the load overlaps the wait for S
          const int ta = inf->tiles[2 * s];
          const bool has_b = 2 * s + 1 < n;
          const int tbv = has_b ? inf->tiles[2 * s + 1] : 0;
          const bool has_mine = (r < 64) || has_b;
          const int mytile = (r < 64) ? ta : tbv;
          const int bitpos = (mytile >= 0) ? mytile : (-(mytile + 1)) * 64 + (r & 63);
          uint32_t word[GH];
#pragma unroll
          for (int h = 0; h < GH; ++h)
            word[h] = (gist && h < G && has_mine)
                          ? ((two_level && mytile < 0)
                                 ? __ldg(allow_base + h * words_g + (bitpos >> 5))
                                 : (fused ? bits_base[h * kUnionWords + (bitpos >> 5)]
                                          : __ldg(bits_base + h * words + (bitpos >> 5))))
                          : 0u;
          if (!(ok = warp_wait(bar(BAR_SF + sb), (s_read >> 1) & 1, abortp, p.status))) break;
          tc_fence_after();
          uint32_t sv[GH];
          tmem_ldn<GH>(lane_addr + sb * 16, sv);
          tc_fence_before();
          mbar_arrive(bar(BAR_SE + sb));   // S buffer may be rewritten
          ++s_read;
          float x[GH];
#pragma unroll
          for (int h = 0; h < GH; ++h) {
            bool allowed = h < G && has_mine;
            if (allowed && gist) {
              const bool bit = (word[h] >> (bitpos & 31)) & 1u;
              // an expanded chunk's tokens, or the gist of a chunk not expanded;
              // with two-level gists, a gist or meta-gist row the head attends
              allowed = (mytile >= 0 || two_level) ? bit : !bit;
            }
            x[h] = allowed ? __uint_as_float(sv[h]) * p.scale_log2 : -INFINITY;
          }
          // tile maximum per head across the 128 keys
          float tm[GH];
#pragma unroll
          for (int h = 0; h < GH; ++h) {
            float v = x[h];
            if (h < G) {
#pragma unroll
              for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            }
            tm[h] = v;
          }
          // exchange the four warps' maxima (bounded mbarrier wait, double-buffered)
          const int xb = rx & 1;
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < GH; ++h) misc->red[xb][warp][h] = tm[h];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_RX + xb));
          if (!(ok = warp_wait(bar(BAR_RX + xb), (rx >> 1) & 1, abortp, p.status))) break;
          ++rx;
          bool any_need = false;
          float alpha[GH], msub[GH];
#pragma unroll
          for (int h = 0; h < GH; ++h) {
            float t = -INFINITY;
            if (h < G) {
#pragma unroll
              for (int w2 = 0; w2 < 4; ++w2) t = fmaxf(t, misc->red[xb][w2][h]);
            }
            const float m_new = fmaxf(m_run[h], t);
            const bool need = m_new > m_run[h] + kRescaleThreshold;
            const float m_use = need ? m_new : m_run[h];
            alpha[h] = need ? fast_exp2(m_run[h] - m_use) : 1.0f;
            any_need |= need && s > 0;
            m_run[h] = m_use;
            msub[h] = (m_use == -INFINITY) ? 0.0f : m_use;
            l_part[h] *= alpha[h];
          }
          if (any_need) {
            // rescale O^T (this thread's lane = channel r): the previous PV must be done
            if (!(ok = warp_wait(bar(BAR_OD), (od_seen + s - 1) & 1, abortp, p.status))) break;
            tc_fence_after();
            uint32_t ov[GH];
            tmem_ldn<GH>(lane_addr + 32, ov);
#pragma unroll
            for (int h = 0; h < GH; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
            tmem_stn<GH>(lane_addr + 32, ov);
            tmem_wait_st();
          }
          // P^T[h][key] = exp2(x - m), written into the swizzled B operand
          const int pb = p_written & 1;
          if (p_written >= 2 && !(ok = warp_wait(bar(BAR_PE + pb), ((p_written >> 1) - 1) & 1, abortp, p.status))) break;
          uint8_t* pbase = smem + kSmemP + pb * kSmallBytes + (r >> 6) * kSmallHalf;
          const int kr = r & 63;
#pragma unroll
          for (int h = 0; h < GH; ++h) {
            const float pv = (h < G) ? fast_exp2(x[h] - msub[h]) : 0.0f;
            l_part[h] += pv;
            const uint32_t off = h * 128 + ((((kr >> 3) ^ (h & 7)) & 7) << 4) + (kr & 7) * 2;
            *reinterpret_cast<__nv_bfloat16*>(pbase + off) = __float2bfloat16_rn(pv);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar(BAR_PF + pb));
          ++p_written;
        }
        if (!ok) break;
        od_seen += nsteps;
        // ---- epilogue: row sums across the 128 keys, then O^T row r = channel r
        const int lb = items_done & 1;
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          float v = l_part[h];
          if (h < G) {
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          }
          if (lane == 0) misc->lred[lb][warp][h] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_LX + lb));
        if (!(ok = warp_wait(bar(BAR_OF), items_done & 1, abortp, p.status))) break;
        tc_fence_after();
        uint32_t ov[GH];
        tmem_ldn<GH>(lane_addr + 32, ov);
        tc_fence_before();
        mbar_arrive(bar(BAR_OE));
        if (!(ok = warp_wait(bar(BAR_LX + lb), (items_done >> 1) & 1, abortp, p.status))) break;
        ++items_done;
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          if (h >= G) continue;
          float* part = part_base + h * head_stride;
          part[4 + r] = __uint_as_float(ov[h]);
          if (r == 0) {
            part[0] = m_run[h];
            part[1] = misc->lred[lb][0][h] + misc->lred[lb][1][h] + misc->lred[lb][2][h] + misc->lred[lb][3][h];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LE + buf));
    }
  }

__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmGK,
                       const __grid_constant__ CUtensorMap tmGV, const __grid_constant__ CUtensorMap tmMK,
                       const __grid_constant__ CUtensorMap tmMV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + kSmemMisc);
  auto bar = [&](int b) -> uint32_t { return sbase + kSmemBar + 8u * b; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abortp = &misc->abort_flag;
  const bool gist = p.expanded != nullptr || p.heads_idx != nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_KE + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(BAR_QF + t), 1);
      mbar_init(bar(BAR_QE + t), 1);
      mbar_init(bar(BAR_SF + t), 1);
      mbar_init(bar(BAR_SE + t), 128);
      mbar_init(bar(BAR_PF + t), 128);
      mbar_init(bar(BAR_PE + t), 1);
      mbar_init(bar(BAR_LF + t), 1);
      mbar_init(bar(BAR_LE + t), kListConsumers);
      mbar_init(bar(BAR_RX + t), 4);
      mbar_init(bar(BAR_LX + t), 4);
    }
    mbar_init(bar(BAR_OD), 1);
    mbar_init(bar(BAR_OF), 1);
    mbar_init(bar(BAR_OE), 128);
    mbar_init(bar(BAR_AB), 1);
    misc->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (gist) {
      prefetch_tmap(&tmGK);
      prefetch_tmap(&tmGV);
      if (p.meta_rows > 0) {
        prefetch_tmap(&tmMK);
        prefetch_tmap(&tmMV);
      }
    }
  }
  if (warp == 5) {
    tmem_alloc(sbase + kSmemMisc + offsetof(Misc, tmem_base), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();   // kept lists / union lists come from the kernel launched before
  const uint32_t tmem = misc->tmem_base;   // S^T buffers at columns 0 / 16, O^T at 32

  if (warp == 6) {
    // ------------------------------------------------ item loader
    const int nb_cache = p.Nk / 64, ngist = p.nc / 64 + (p.meta_rows > 0 ? 1 : 0);
    int r0 = 0;
    const int nitems = cta_items(p, blockIdx.x, &r0);
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * p.total / p.num_ctas;
    const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * p.total / p.num_ctas;
    const unsigned lt = (1u << lane) - 1u;
    for (int k = 0; k < nitems; ++k) {
      const int buf = k & 1;
      if (k >= 2 && !warp_wait(bar(BAR_LE + buf), ((k >> 1) - 1) & 1, abortp, p.status)) break;
      ItemInfo* inf = &misc->info[buf];
      const int bg = r0 + k;
      const int64_t row0 = static_cast<int64_t>(bg) * p.list_len;
      const int a = static_cast<int>(max(lo, row0) - row0);
      const int e = static_cast<int>(min(hi, row0 + p.list_len) - row0);
      int stop, w = 0;
      if (p.heads_idx != nullptr) {
        // gist decode, union built here: each head's expanded chunks and
        // their union as bitmaps in the item slot, then the row's list =
        // union chunks ascending followed by every gist tile -(t+1)
        const int G = p.G, words = p.nc / 32, topk = p.heads_topk;
        uint32_t* ub = &inf->bits[0][0];
        for (int t = lane; t < (G + 1) * kUnionWords; t += 32) ub[t] = 0u;
        __syncwarp();
        const int* hsrc = p.heads_idx + (static_cast<int64_t>(bg / p.Hkv) * p.Hq + (bg % p.Hkv) * G) *
                                            static_cast<int64_t>(p.heads_stride);
        // the entries in rounds of 8 per lane, each round's loads issued together
        for (int t0 = 0; t0 < G * topk; t0 += 32 * 8) {
          int cv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int t = t0 + 32 * u + lane;
            const int hh = t / topk;
            cv[u] = (t < G * topk) ? __ldg(hsrc + static_cast<int64_t>(hh) * p.heads_stride + (t - hh * topk)) : -1;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int c = cv[u];
            if (c < 0) continue;
            if (c >= p.nc) {
              atomicOr(p.status, BSA_DEV_BAD_INDEX);
              continue;
            }
            const int hh = (t0 + 32 * u + lane) / topk;
            atomicOr(&ub[hh * kUnionWords + (c >> 5)], 1u << (c & 31));
            atomicOr(&ub[G * kUnionWords + (c >> 5)], 1u << (c & 31));
          }
        }
        __syncwarp();
        const uint32_t w0 = (2 * lane < words) ? ub[G * kUnionWords + 2 * lane] : 0u;
        const uint32_t w1 = (2 * lane + 1 < words) ? ub[G * kUnionWords + 2 * lane + 1] : 0u;
        const int cnt = __popc(w0) + __popc(w1);
        int incl = cnt;
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        const int U = __shfl_sync(0xffffffffu, incl, 31);
        stop = min(e, min(U + ngist, p.list_len));
        const int lim = min(stop, a + kMaxItemTiles);
        int pos = incl - cnt;
        for (int hw = 0; hw < 2; ++hw) {
          uint32_t m = hw ? w1 : w0;
          while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1;
            if (pos >= a && pos < lim) inf->tiles[pos - a] = (2 * lane + hw) * 32 + bit;
            ++pos;
          }
        }
        for (int t = lane; t < ngist; t += 32)
          if (U + t >= a && U + t < lim) inf->tiles[U + t - a] = -(t + 1);
        w = max(0, lim - a);
        __syncwarp();
      } else {
        const int* src = p.list + static_cast<int64_t>(bg) * p.list_stride;
        int count;
        if (p.list_has_count) {
          count = min(src[0], p.list_len);
          src += 1;
        } else {
          count = e;   // the first negative entry ends the list
          for (int base = 0; base < e; base += 32) {
            const int t = base + lane;
            const int v = (t < e) ? src[t] : 0;
            const unsigned neg = __ballot_sync(0xffffffffu, v < 0);
            if (neg) {
              count = base + __ffs(neg) - 1;
              break;
            }
          }
        }
        stop = min(e, count);
        for (int base = a; base < stop; base += 32) {
          const int t = base + lane;
          const int v = (t < stop) ? src[t] : 0;
          bool bad = (t < stop) && (gist ? (v >= nb_cache || v < -ngist) : (v < 0 || v >= nb_cache));
          int tile = v;
          if (p.table != nullptr && t < stop && !bad) {
            // paged cache: the kept logical block's physical block
            tile = __ldg(p.table + static_cast<int64_t>(bg / p.Hkv) * p.table_stride + v);
            bad = tile < 0 || tile >= p.num_pages;
          }
          if (bad) atomicOr(p.status, BSA_DEV_BAD_INDEX);
          const bool keep = (t < stop) && !bad && (w + (t - base) < kMaxItemTiles);
          const unsigned km = __ballot_sync(0xffffffffu, keep);
          if (keep) inf->tiles[w + __popc(km & lt)] = tile;
          w += __popc(km);
        }
      }
      if (lane == 0) {
        if (stop - a > kMaxItemTiles) atomicOr(p.status, BSA_DEV_BAD_SHAPE);
        inf->n = w;
        inf->bg = bg;
        inf->b = bg / p.Hkv;
        inf->g = bg % p.Hkv;
        inf->slot = static_cast<int>(blockIdx.x) - cta_of(row0, p.total, p.num_ctas);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LF + buf));
    }
  } else if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int gs = 0, qcount = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      int r0 = 0;
      const int nitems = cta_items(p, blockIdx.x, &r0);
      for (int k = 0; ok && k < nitems; ++k) {
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int qb = qcount & 1;
          if (qcount >= 2 && !(ok = mbar_wait(bar(BAR_QE + qb), ((qcount >> 1) - 1) & 1, abortp, p.status))) break;
          mbar_arrive_expect_tx(bar(BAR_QF + qb), static_cast<uint32_t>(p.G) * 256u);
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(sbase + kSmemQ + qb * kSmallBytes + hf * kSmallHalf, &tmQ, bar(BAR_QF + qb), hf * 64,
                        inf->b * p.Hq + inf->g * p.G);
          ++qcount;
          const int nsteps = (n + 1) / 2;
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int slot = gs % kStages, use = gs / kStages;
            const int nt = (2 * s + 1 < n) ? 2 : 1;
            const uint32_t bytes = static_cast<uint32_t>(nt) * 64u * 256u;
            for (int kv = 0; kv < 2; ++kv) {
              const int full = kv ? BAR_VF : BAR_KF, empty = kv ? BAR_VE : BAR_KE;
              const uint32_t dst0 = sbase + (kv ? kSmemV : kSmemK) + slot * kTileBytes;
              if (gs >= kStages && !(ok = mbar_wait(bar(empty + slot), (use - 1) & 1, abortp, p.status))) break;
              mbar_arrive_expect_tx(bar(full + slot), bytes);
              for (int tt = 0; tt < nt; ++tt) {
                const int tile = inf->tiles[2 * s + tt];
                const CUtensorMap* map;
                int y;
                if (tile >= 0) {
                  map = kv ? &tmV : &tmK;
                  y = (p.table != nullptr) ? (tile * p.Hkv + inf->g) * 64 : inf->bg * p.Nk + tile * 64;
                } else if (-(tile + 1) < p.nc / 64) {
                  map = kv ? &tmGV : &tmGK;
                  y = inf->bg * p.nc + (-(tile + 1)) * 64;
                } else {   // the meta-gist tile (two-level gists)
                  map = kv ? &tmMV : &tmMK;
                  y = inf->bg * p.meta_rows + (-(tile + 1) - p.nc / 64) * 64;
                }
                for (int hf = 0; hf < 2; ++hf)
                  tma_load_2d(dst0 + hf * kHalfBytes + tt * 8192u, map, bar(full + slot), hf * 64, y);
              }
              if (kv) ++v_issued; else ++k_issued;
            }
            if (!ok) break;
          }
          if (!ok) break;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (*abortp) {
        for (int q = max(0, qcount - 2); q < qcount; ++q) mbar_drain(bar(BAR_QF + (q & 1)), (q >> 1) & 1);
        for (int s = max(0, k_issued - kStages); s < k_issued; ++s) mbar_drain(bar(BAR_KF + s % kStages), (s / kStages) & 1);
        for (int s = max(0, v_issued - kStages); s < v_issued; ++s) mbar_drain(bar(BAR_VF + s % kStages), (s / kStages) & 1);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16_f32(128, kNH, 0, 0);    // S^T = K Q^T, both K-major
      const uint32_t id_pv = idesc_bf16_f32(128, kNH, 1, 0);   // O^T = V^T P^T, V^T MN-major
      int gs = 0, qcount = 0, items_done = 0;
      int s_issued = 0, p_used = 0;   // S buffers written / P buffers consumed (global counts)
      bool ok = true;
      auto issue_s = [&](int slot, int qb, int sbuf) {
        const uint32_t ka = sbase + kSmemK + slot * kTileBytes;
        const uint32_t qa = sbase + kSmemQ + qb * kSmallBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t offk = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint32_t offq = (kk >> 2) * kSmallHalf + (kk & 3) * 32;
          mma_ss(tmem + sbuf * 16, smem_desc_sw128(ka + offk, 16, 1024), smem_desc_sw128(qa + offq, 16, 1024),
                 id_s, kk > 0 ? 1u : 0u);
        }
      };
      int r0 = 0;
      const int nitems = cta_items(p, blockIdx.x, &r0);
      for (int k = 0; ok && k < nitems; ++k) {
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const int n = misc->info[buf].n;
        if (n > 0) {
          const int nsteps = (n + 1) / 2;
          const int qb = qcount & 1;
          if (!(ok = mbar_wait(bar(BAR_QF + qb), (qcount >> 1) & 1, abortp, p.status))) break;
          ++qcount;
          tc_fence_after();
          const int gs0 = gs;
          // S for the first step of the item
          for (int s = 0; ok && s < nsteps; ++s) {
            // issue S(s) (the softmax must have read the S buffer two steps back)
            {
              const int g_s = gs0 + s, slot = g_s % kStages, sb = s_issued & 1;
              if (!(ok = mbar_wait(bar(BAR_KF + slot), (g_s / kStages) & 1, abortp, p.status))) break;
              if (s_issued >= 2 && !(ok = mbar_wait(bar(BAR_SE + sb), ((s_issued >> 1) - 1) & 1, abortp, p.status)))
                break;
              tc_fence_after();
              issue_s(slot, qb, sb);
              tc_commit(bar(BAR_SF + sb));
              tc_commit(bar(BAR_KE + slot));
              ++s_issued;
            }
            // O^T += V^T P^T for step s-1 (one step behind, so S(s) overlaps the softmax of s-1)
            if (s > 0) {
              const int ps = s - 1, g_p = gs0 + ps, slot = g_p % kStages, pb = p_used & 1;
              if (!(ok = mbar_wait(bar(BAR_PF + pb), (p_used >> 1) & 1, abortp, p.status))) break;
              if (!(ok = mbar_wait(bar(BAR_VF + slot), (g_p / kStages) & 1, abortp, p.status))) break;
              if (ps == 0 && items_done > 0 &&
                  !(ok = mbar_wait(bar(BAR_OE), (items_done - 1) & 1, abortp, p.status)))
                break;
              tc_fence_after();
              const int keys = (2 * ps + 1 < n) ? 128 : 64;
              const uint32_t va = sbase + kSmemV + slot * kTileBytes;
              const uint32_t pa = sbase + kSmemP + pb * kSmallBytes;
              for (int kk = 0; kk < keys / 16; ++kk)
                mma_ss(tmem + 32, smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024),
                       smem_desc_sw128(pa + (kk >> 2) * kSmallHalf + (kk & 3) * 32, 16, 1024), id_pv,
                       (ps > 0 || kk > 0) ? 1u : 0u);
              tc_commit(bar(BAR_OD));
              tc_commit(bar(BAR_VE + slot));
              tc_commit(bar(BAR_PE + pb));
              ++p_used;
            }
          }
          if (!ok) break;
          tc_commit(bar(BAR_QE + qb));
          {
            const int ps = nsteps - 1, g_p = gs0 + ps, slot = g_p % kStages, pb = p_used & 1;
            if (!(ok = mbar_wait(bar(BAR_PF + pb), (p_used >> 1) & 1, abortp, p.status))) break;
            if (!(ok = mbar_wait(bar(BAR_VF + slot), (g_p / kStages) & 1, abortp, p.status))) break;
            if (ps == 0 && items_done > 0 && !(ok = mbar_wait(bar(BAR_OE), (items_done - 1) & 1, abortp, p.status)))
              break;
            tc_fence_after();
            const int keys = (2 * ps + 1 < n) ? 128 : 64;
            const uint32_t va = sbase + kSmemV + slot * kTileBytes;
            const uint32_t pa = sbase + kSmemP + pb * kSmallBytes;
            for (int kk = 0; kk < keys / 16; ++kk)
              mma_ss(tmem + 32, smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024),
                     smem_desc_sw128(pa + (kk >> 2) * kSmallHalf + (kk & 3) * 32, 16, 1024), id_pv,
                     (ps > 0 || kk > 0) ? 1u : 0u);
            tc_commit(bar(BAR_OD));
            tc_commit(bar(BAR_VE + slot));
            tc_commit(bar(BAR_PE + pb));
            ++p_used;
          }
          tc_commit(bar(BAR_OF));
          ++items_done;
          gs += nsteps;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (!ok) {
        tc_commit(bar(BAR_AB));
        mbar_drain(bar(BAR_AB), 0);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------ softmax (thread = key) + epilogue (thread = d)
    if (p.G <= 4)
      softmax_role<4>(p, misc, smem, sbase, tmem, abortp, warp, lane, gist);
    else if (p.G <= 8)
      softmax_role<8>(p, misc, smem, sbase, tmem, abortp, warp, lane, gist);
    else
      softmax_role<16>(p, misc, smem, sbase, tmem, abortp, warp, lane, gist);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// Merge the partial records of one output row (b, h) (one warp per row):
// the row's group was cut into nseg segments, one record each.  Up to four
// records are read in one round (every load issued before any is used), so
// a row costs one memory round trip rather than one per segment.
__global__ void combine_kernel(const float* __restrict__ partial, int rows, int G, int list_len, int64_t total,
                               int num_ctas, int max_slots, int d, int out_bf16, void* __restrict__ o,
                               float* __restrict__ lse) {
  griddep_wait();
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t bg = row / G;
  const int first = cta_of(bg * list_len, total, num_ctas);
  const int last = cta_of((bg + 1) * list_len - 1, total, num_ctas);
  const int nseg = min(max_slots, last - first + 1);
  const int rec = d + 4;
  const float* pr = partial + static_cast<int64_t>(row) * max_slots * rec;
  float M = -INFINITY;
  float L = 0.0f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = 0; s0 < nseg; s0 += 4) {
    float ms[4], ls[4], ov[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool in = s0 + k < nseg;
      const float* r = pr + (s0 + k) * rec;
      ms[k] = in ? r[0] : -INFINITY;
      ls[k] = in ? r[1] : 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        ov[k][e] = (in && c < d) ? r[4 + c] : 0.0f;
      }
    }
    // fold this round into the running (M, L, acc), segments in order
    float Mn = M;
#pragma unroll
    for (int k = 0; k < 4; ++k) Mn = fmaxf(Mn, ms[k]);
    if (Mn == -INFINITY) continue;
    const float a = (M == -INFINITY) ? 0.0f : exp2f(M - Mn);
    L *= a;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] *= a;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (ms[k] == -INFINITY) continue;
      const float w = exp2f(ms[k] - Mn);
      L += w * ls[k];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] += w * ov[k][e];
    }
    M = Mn;
  }
  const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
  for (int e = 0; e < 4; ++e) {
    const int c = lane + 32 * e;
    if (c >= d) continue;
    const float val = acc[e] * inv;
    if (out_bf16)
      static_cast<__nv_bfloat16*>(o)[static_cast<int64_t>(row) * d + c] = __float2bfloat16_rn(val);
    else
      static_cast<float*>(o)[static_cast<int64_t>(row) * d + c] = val;
  }
  if (lse && lane == 0) lse[row] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
}

// Gist: per (b, g) build each head's expanded-chunk bitmap and the ascending
// union of expanded chunks followed by every gist block (-(gb+1)) when
// with_gists is set.  Without gists (per-head decode, where chunk = block)
// the union lists only the heads' kept blocks.
__global__ void gist_union_kernel(const int* __restrict__ idx, int Hq, int Hkv, int topk, int idx_stride, int nc,
                                  uint32_t* __restrict__ expanded, int* __restrict__ union_list, int union_stride,
                                  int with_gists, uint32_t* __restrict__ status) {
  griddep_wait();
  extern __shared__ uint32_t sbits[];   // [G+1][nc/32]; row G = union
  const int G = Hq / Hkv;
  const int words = nc / 32;
  const int bg = blockIdx.x;
  const int b = bg / Hkv, g = bg % Hkv;
  for (int e = threadIdx.x; e < (G + 1) * words; e += blockDim.x) sbits[e] = 0u;
  __syncthreads();
  for (int e = threadIdx.x; e < G * topk; e += blockDim.x) {
    const int hh = e / topk, t = e % topk;
    const int c = idx[(static_cast<int64_t>(b) * Hq + g * G + hh) * idx_stride + t];
    if (c < 0) continue;
    if (c >= nc) {
      atomicOr(status, BSA_DEV_BAD_INDEX);
      continue;
    }
    atomicOr(&sbits[hh * words + (c >> 5)], 1u << (c & 31));
    atomicOr(&sbits[G * words + (c >> 5)], 1u << (c & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * words; e += blockDim.x) {
    const int hh = e / words, w = e % words;
    expanded[(static_cast<int64_t>(b) * Hq + g * G + hh) * words + w] = sbits[e];
  }
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int* out = union_list + static_cast<int64_t>(bg) * union_stride;
    int run = 0;
    for (int base = 0; base < words; base += 32) {
      const int w = base + lane;
      const uint32_t bitsw = (w < words) ? sbits[G * words + w] : 0u;
      const int cnt = __popc(bitsw);
      int incl = cnt;
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = run + incl - cnt;
      uint32_t m = bitsw;
      while (m) {
        const int bit = __ffs(m) - 1;
        m &= m - 1;
        out[1 + pos++] = w * 32 + bit;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int ngb = with_gists ? nc / 64 : 0;
    for (int t = lane; t < ngb; t += 32) out[1 + run + t] = -(t + 1);
    if (lane == 0) out[0] = run + ngb;
  }
}

// Two-level gists (H-SSA): per (b, g) from each head's kept groups (meta_idx
// [B*Hq][km], ascending) and chosen positions among its kept groups' chunks
// (pos_idx [B*Hq][k]: position t*64 + x = chunk x of its t-th kept group,
// ascending): each head's chunk list (chunk_out), its expanded-chunk bitmap,
// its gist-allowed bitmap over the rows [gists 0..nc) | [meta-gists nm..)
// (a gist of a kept group not expanded; a meta-gist of a group not kept),
// and the group's tile list: expanded chunks ascending, the gist tiles of the
// groups any head kept, then the meta-gist tile.  Groups are 64 chunks, so a
// kept group's gists are one gist tile.
__global__ void hssa_union_kernel(const int* __restrict__ meta_idx, int km, const int* __restrict__ pos_idx, int k,
                                  int Hq, int Hkv, int nc, int nm, int* __restrict__ chunk_out,
                                  uint32_t* __restrict__ expanded, uint32_t* __restrict__ gist_allow,
                                  int* __restrict__ union_list, int union_stride, uint32_t* __restrict__ status) {
  griddep_wait();
  extern __shared__ uint32_t sb[];
  const int G = Hq / Hkv;
  const int words = nc / 32, words_g = (nc + 64) / 32;
  uint32_t* ex = sb;                       // [G+1][words]: heads' expanded chunks, then the union
  uint32_t* al = sb + (G + 1) * words;     // [G][words_g]: heads' allowed gist / meta rows
  uint32_t* kg = al + G * words_g;         // [G+1][2]: heads' kept groups (nm <= 64), then the union
  const int bg = blockIdx.x;
  const int b = bg / Hkv, g = bg % Hkv;
  const int total = (G + 1) * words + G * words_g + (G + 1) * 2;
  for (int e = threadIdx.x; e < total; e += blockDim.x) sb[e] = 0u;
  __syncthreads();
  const int64_t row0 = static_cast<int64_t>(b) * Hq + g * G;
  for (int e = threadIdx.x; e < G * km; e += blockDim.x) {
    const int hh = e / km, t = e % km;
    const int m = meta_idx[(row0 + hh) * km + t];
    if (m < 0) continue;
    if (m >= nm) {
      atomicOr(status, BSA_DEV_BAD_INDEX);
      continue;
    }
    atomicOr(&kg[hh * 2 + (m >> 5)], 1u << (m & 31));
    atomicOr(&kg[G * 2 + (m >> 5)], 1u << (m & 31));
  }
  for (int e = threadIdx.x; e < G * k; e += blockDim.x) {
    const int hh = e / k, t = e % k;
    const int pos = pos_idx[(row0 + hh) * k + t];
    int c = -1;
    if (pos >= 0) {
      const int grp = pos >> 6;
      const int m = (grp < km) ? meta_idx[(row0 + hh) * km + grp] : -1;
      c = (m >= 0 && m < nm) ? m * 64 + (pos & 63) : -1;
      if (c < 0 || c >= nc) {
        atomicOr(status, BSA_DEV_BAD_INDEX);
        c = -1;
      }
    }
    chunk_out[(row0 + hh) * k + t] = c;
    if (c < 0) continue;
    atomicOr(&ex[hh * words + (c >> 5)], 1u << (c & 31));
    atomicOr(&ex[G * words + (c >> 5)], 1u << (c & 31));
  }
  __syncthreads();
  // allowed rows: gist c of a kept group not expanded; meta-gist m of a group not kept
  for (int e = threadIdx.x; e < G * words_g; e += blockDim.x) {
    const int hh = e / words_g, w = e % words_g;
    uint32_t bits = 0u;
    if (w < words) {
      const int m = (w * 32) >> 6;   // 32 consecutive chunks lie in one group of 64
      if ((kg[hh * 2 + (m >> 5)] >> (m & 31)) & 1u) bits = ~ex[hh * words + w];
    } else {
      for (int x = 0; x < 32; ++x) {
        const int m = (w - words) * 32 + x;
        if (m < nm && !((kg[hh * 2 + (m >> 5)] >> (m & 31)) & 1u)) bits |= 1u << x;
      }
    }
    al[e] = bits;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * words; e += blockDim.x) expanded[row0 * words + e] = ex[e];
  for (int e = threadIdx.x; e < G * words_g; e += blockDim.x) gist_allow[row0 * words_g + e] = al[e];
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int* out = union_list + static_cast<int64_t>(bg) * union_stride;
    int run = 0;
    for (int base = 0; base < words; base += 32) {
      const int w = base + lane;
      const uint32_t bitsw = (w < words) ? ex[G * words + w] : 0u;
      const int cnt = __popc(bitsw);
      int incl = cnt;
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = run + incl - cnt;
      uint32_t mm = bitsw;
      while (mm) {
        const int bit = __ffs(mm) - 1;
        mm &= mm - 1;
        out[1 + pos++] = w * 32 + bit;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    // the gist tiles of kept groups (tile -(m+1) holds the 64 gists of group m), then the meta tile
    if (lane == 0) {
      for (int m = 0; m < nm; ++m)
        if ((kg[G * 2 + (m >> 5)] >> (m & 31)) & 1u) out[1 + run++] = -(m + 1);
      out[1 + run++] = -(nc / 64 + 1);
      out[0] = run;
    }
  }
}

}  // namespace decode

cudaError_t launch_attn_decode_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                    const CUtensorMap* tmGK, const CUtensorMap* tmGV, const DecodeArgs& a,
                                    cudaStream_t st, const CUtensorMap* tmMK, const CUtensorMap* tmMV) {
  cudaError_t e = ensure_dynamic_smem<decode::attn_decode_kernel>(decode::kSmemBytes);
  if (e != cudaSuccess) return e;
  decode::Params p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Nk = a.Nk;
  p.G = a.Hq / a.Hkv;
  p.nc = a.nc;
  p.list = a.list;
  p.list_stride = a.list_stride;
  p.list_has_count = a.list_has_count;
  p.expanded = a.expanded;
  p.list_len = a.list_len;
  p.total = static_cast<int64_t>(a.B) * a.Hkv * a.list_len;
  p.num_ctas = a.num_ctas;
  p.max_slots = a.max_slots;
  p.scale_log2 = a.softmax_scale * decode::kLog2e;
  p.partial = a.partial;
  p.status = a.status;
  p.table = a.table;
  p.table_stride = a.table_stride;
  p.num_pages = a.num_pages;
  p.gist_allow = a.gist_allow;
  p.meta_rows = (tmMK != nullptr) ? a.meta_rows : 0;
  p.heads_idx = a.heads_idx;
  p.heads_topk = a.heads_topk;
  p.heads_stride = a.heads_stride;
  if (p.heads_idx != nullptr && (p.nc > 32 * decode::kUnionWords || p.G > decode::kNH || p.gist_allow != nullptr))
    return cudaErrorInvalidValue;
  const int grid = a.num_ctas;
  return launch_dependent(decode::attn_decode_kernel, dim3(grid), dim3(decode::kThreads), decode::kSmemBytes, st, *tmQ,
                          *tmK, *tmV, tmGK ? *tmGK : *tmK, tmGV ? *tmGV : *tmV, tmMK ? *tmMK : *tmK,
                          tmMV ? *tmMV : *tmV, p);
}

cudaError_t launch_decode_combine(const float* partial, const DecodeArgs& a, int d, bool out_bf16, void* o,
                                  float* lse, cudaStream_t st) {
  const int warps = 8;
  const int rows = a.B * a.Hq;
  const int64_t total = static_cast<int64_t>(a.B) * a.Hkv * a.list_len;
  return launch_dependent(decode::combine_kernel, dim3((rows + warps - 1) / warps), dim3(warps * 32), 0, st, partial,
                          rows, a.Hq / a.Hkv, a.list_len, total, a.num_ctas, a.max_slots, d, out_bf16 ? 1 : 0, o, lse);
}

int decode_slots_for(int rows, int list_len, int num_ctas) {
  // the largest number of CTAs that can share one row's positions
  const int64_t total = static_cast<int64_t>(rows) * list_len;
  int best = 1;
  for (int r = 0; r < rows; ++r) {
    const int first = decode::cta_of(static_cast<int64_t>(r) * list_len, total, num_ctas);
    const int last = decode::cta_of(static_cast<int64_t>(r + 1) * list_len - 1, total, num_ctas);
    if (last - first + 1 > best) best = last - first + 1;
  }
  return best;
}

cudaError_t launch_gist_union(const int* idx, int B, int Hq, int Hkv, int topk, int idx_stride, int nc,
                              uint32_t* expanded, int* union_list, int union_stride, bool with_gists,
                              uint32_t* status, cudaStream_t st) {
  const int G = Hq / Hkv;
  const size_t smem = static_cast<size_t>(G + 1) * (nc / 32) * sizeof(uint32_t);
  return launch_dependent(decode::gist_union_kernel, dim3(B * Hkv), dim3(256), smem, st, idx, Hq, Hkv, topk, idx_stride,
                          nc, expanded, union_list, union_stride, with_gists ? 1 : 0, status);
}

cudaError_t launch_hssa_union(const int* meta_idx, int km, const int* pos_idx, int k, int B, int Hq, int Hkv, int nc,
                              int nm, int* chunk_out, uint32_t* expanded, uint32_t* gist_allow, int* union_list,
                              int union_stride, uint32_t* status, cudaStream_t st) {
  const int G = Hq / Hkv;
  const size_t smem = (static_cast<size_t>(G + 1) * (nc / 32) + static_cast<size_t>(G) * ((nc + 64) / 32) +
                       static_cast<size_t>(G + 1) * 2) *
                      sizeof(uint32_t);
  return launch_dependent(decode::hssa_union_kernel, dim3(B * Hkv), dim3(256), smem, st, meta_idx, km, pos_idx, k, Hq,
                          Hkv, nc, nm, chunk_out, expanded, gist_allow, union_list, union_stride, status);
}

}  // namespace bsa
