// attn_prefill_pair.cu -- block-sparse causal attention, prefill, bf16,
// d = 128, on a pair of SMs: tcgen05 MMAs of M = 256 issued for two CTAs of
// a cluster (cta_group::2), TMA tile loads, accumulators in tensor memory.
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
// is two consecutive 128-row tiles of a unit, run by the two CTAs of a
// cluster: CTA r holds tile 2*pair + r (its Q rows, its S and O
// accumulators), and the pair computes S = Q K^T and O += P V as MMAs of
// M = 256.  B operands are split along N between the CTAs: for S each CTA
// loads half of the step's keys (N = keys), for O += P V half of the value
// channels (N = d), so each K/V tile is fetched once per 256 query rows and
// each SM stages and reads only half of it.  The kernel is persistent: the
// clusters walk items cluster_id, +num_clusters, ... (heavy items first).
//
// A step covers 128 keys: two 64-token blocks (bs = 64: CTA r loads block
// r of the step for S) or one 128-token block (CTA r loads its rows
// 64r..64r+63); the last step of an odd bs = 64 list holds one block of 64
// keys (N = 64: CTA r loads its keys 32r..32r+31).  Each step is split into
// two key halves of 64 keys; half h has its own softmax warps, its own
// running maximum and sum per row and its own output accumulator O_h, and
// the two partials of a row are merged once, in the epilogue.
//
// Roles (384 threads per CTA, three warpgroups):
//   warp 0      TMA producer of Q (per item, two slots) and K (per step,
//               four-stage ring of this CTA's halves);
//   warp 3      TMA producer of V (per step, four-stage ring);
//   warp 1      tensor-memory owner (both CTAs, allocating together) and, in
//               the even CTA, the MMA issuer (one thread): S(s) into S buffer
//               s mod 2, then O_h += P_h(s-1) V for the previous step;
//   warp 2      item loader: kept-block list and gate biases;
//   warps 4-7   softmax of key half 0 (thread = query row = TMEM lane);
//   warps 8-11  softmax of key half 1; the epilogue is shared.
// Tensor memory per CTA (512 columns): S buffer 0 | S buffer 1 | O_0 | O_1.
//
// Cross-CTA signalling.  Barriers that the issuer waits on live in the even
// CTA: the loads of both CTAs count their bytes on its full barriers, and
// the softmax and epilogue warps of both CTAs arrive on its P-ready and
// O-read barriers.  The issuer's commits arrive on the barrier at the same
// offset in both CTAs (S ready, K / V / Q slot free).  No load uses cluster
// multicast: every CTA copies into its own shared memory only.
#include "common.cuh"
#include "kernels.h"
#include "tmem_wide.cuh"

namespace bsa {
namespace prefill_pair {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kStages = 4;
constexpr int kMaxList = 256;
constexpr uint32_t kQHalf = 128u * 128u;      // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kQBytes = 2u * kQHalf;     // this CTA's 128 query rows x 128 channels
constexpr uint32_t kKHalf = 64u * 128u;       // 64 keys x 64 bf16
constexpr uint32_t kKBytes = 2u * kKHalf;     // this CTA's keys of a step x 128 channels
constexpr uint32_t kVBytes = 128u * 128u;     // 128 keys x this CTA's 64 channels
constexpr uint32_t kSmemQ = 0;                // two Q slots
constexpr uint32_t kSmemK = kSmemQ + 2 * kQBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kKBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kVBytes;
constexpr uint32_t kColO = 256;     // O_0 at 256, O_1 at 384; S buffers at 0 and 128
constexpr int kCtrlRegs = 120;      // warps 0-3 after setmaxnreg.dec
constexpr int kMathRegs = 184;      // warps 4-11 after setmaxnreg.inc
static_assert(128 * kCtrlRegs + 256 * kMathRegs <= kThreads * 168, "register split exceeds the launch pool");
constexpr uint16_t kBoth = 0x3;     // multicast mask: both CTAs of the pair

enum {
  BAR_QF = 0,                  // per Q slot: both CTAs' rows loaded (even CTA)
  BAR_QE = BAR_QF + 2,         // per Q slot: the item's last S has completed (both)
  BAR_KF = BAR_QE + 2,         // per K stage: both halves loaded (even CTA)
  BAR_KE = BAR_KF + kStages,   // per K stage: S of its step completed (both)
  BAR_VF = BAR_KE + kStages,   // per V stage: both halves loaded (even CTA)
  BAR_VE = BAR_VF + kStages,   // per V stage: O += P V of its step completed (both)
  BAR_SF = BAR_VE + kStages,   // per S buffer: S complete (both)
  BAR_PF = BAR_SF + 2,         // per (half, S buffer): P written by both CTAs (even CTA)
  BAR_OE = BAR_PF + 4,         // O_0 and O_1 read back by both CTAs (even CTA)
  BAR_ML = BAR_OE + 1,         // both halves' (m, l) of an item published (local)
  BAR_LF = BAR_ML + 1,         // per metadata slot: filled (local)
  BAR_LE = BAR_LF + 2,         // per metadata slot: consumed by every local role
  BAR_AB = BAR_LE + 2,
  NUM_BARS
};

struct ItemInfo {
  int n, b, g, i, tile, pad0, pad1, pad2;
  int list[kMaxList];
  float bias[kMaxList];
};

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
  int pad[2];
  float2 ml[2][2][128];   // [item parity][half][row]: running (max, sum) at the end of an item
  ItemInfo info[2];
};

constexpr uint32_t kSmemMisc = kSmemBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + sizeof(Misc) + 1024;   // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Params {
  int B, Hq, Hkv, N, nb, G;
  int rows_per_unit, tiles_per_unit, pairs_per_unit, num_items;
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

template <int N>
__device__ __forceinline__ void set_regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void set_regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Per-CTA context of the bounded waits: a wait that gives up also raises
// the peer CTA's abort flag, so both CTAs of the pair leave their loops.
struct Ctx {
  volatile int* abortp;
  uint32_t peer_abort;   // cluster address of the peer's abort flag
  uint32_t* status;
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    if (mbar_wait_cluster(bar, parity, abortp, status)) return true;
    st_shared_cluster_u32(peer_abort, 1u);
    return false;
  }
  __device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) const {
    const bool ok = wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
  }
};

// One softmax step of one key half (64 keys of this thread's row), as in the
// one-tile-per-item kernel: t_s the half's 64 S columns, t_o its O_h.
template <bool MASK>
__device__ __forceinline__ bool softmax_half(uint32_t t_s, uint32_t t_o, bool first, float scale_log2, float bias,
                                             int koff0, int tb, float& m_run, float& l_run, uint32_t ve_bar,
                                             uint32_t ve_par, const Ctx& cx) {
  uint32_t v[64];
  tmem_ld64(t_s, v);
  if constexpr (MASK) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (koff0 + c > tb) v[c] = 0xFF800000u;   // -inf
  }
  float m8[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) m8[a] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 2)
    m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
  const float mraw = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
  const float mx = fmaf(mraw, scale_log2, bias);
  const float m_new = fmaxf(m_run, mx);
  const bool need = m_new > m_run + kRescaleThreshold;
  const float m_use = need ? m_new : m_run;
  const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
  const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
  if (!first && __any_sync(0xffffffffu, need)) {
    // O_h may still be accumulating the previous step's P V
    if (!cx.warp_wait(ve_bar, ve_par)) return false;
    tc_fence_after();
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
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t off = f2_pack(bias - m_sub, bias - m_sub);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  uint32_t pk[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sc2, off);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    acc[e & 3] = f2_add(acc[e & 3], f2_pack(p0, p1));
    pk[e] = pack_bf16x2(p0, p1);
  }
  tmem_st32(t_s, pk);
  float a0, a1, a2, a3;
  f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
  f2_unpack(f2_add(acc[2], acc[3]), a2, a3);
  l_run += (a0 + a1) + (a2 + a3);
  tmem_wait_st();
  return true;
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + kSmemMisc);
  auto bar = [&](int b) -> uint32_t { return sbase + kSmemBar + 8u * b; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = static_cast<int>(cluster_id_x());
  const int nclusters = static_cast<int>(cluster_count_x());
  // barrier of the even CTA at this CTA's offset of barrier b
  auto lead = [&](int b) -> uint32_t { return mapa_shared(bar(b), 0); };
  Ctx cx;
  cx.abortp = &misc->abort_flag;
  cx.peer_abort = mapa_shared(smem_u32(&misc->abort_flag), rank ^ 1u);
  cx.status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BAR_QF + s), 1);
      mbar_init(bar(BAR_QE + s), 1);
      mbar_init(bar(BAR_SF + s), 1);
      mbar_init(bar(BAR_PF + s), 8);       // 4 softmax warps of half 0 in each CTA
      mbar_init(bar(BAR_PF + 2 + s), 8);   // ... of half 1
      mbar_init(bar(BAR_LF + s), 1);
      // producers (2) + softmax warps (8) + the issuer (even CTA only)
      mbar_init(bar(BAR_LE + s), rank == 0 ? 11 : 10);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_KE + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
    }
    mbar_init(bar(BAR_OE), 16);
    mbar_init(bar(BAR_ML), 8);
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
    tmem_alloc_pair(sbase + kSmemMisc + offsetof(Misc, tmem_base), 512);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;

  if (warp < 4) {
  set_regs_dec<kCtrlRegs>();
  if (warp == 2) {
    // ------------------------------------------------ item loader
    const unsigned lt = (1u << lane) - 1u;
    for (int k = 0;; ++k) {
      const int item = cluster + k * nclusters;
      if (item >= p.num_items) break;
      const int buf = k & 1;
      if (k >= 2 && !cx.warp_wait(bar(BAR_LE + buf), ((k >> 1) - 1) & 1)) break;
      ItemInfo* inf = &misc->info[buf];
      const int unit = item / p.pairs_per_unit, pair = item % p.pairs_per_unit;
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
        if (in && !ok && rank == 0) atomicOr(p.status, BSA_DEV_BAD_INDEX);
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
        inf->b = bg / p.Hkv;
        inf->g = bg % p.Hkv;
        inf->i = i;
        inf->tile = 2 * pair + static_cast<int>(rank);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LF + buf));
    }
  } else if (warp == 0 || warp == 3) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producers
      // warp 0 loads Q and this CTA's half of K, warp 3 this CTA's half of V.
      // The even CTA's producer announces both CTAs' bytes on its full
      // barrier; both CTAs' copies count their bytes there.
      const int kv = (warp == 3) ? 1 : 0;
      const int full = kv ? BAR_VF : BAR_KF, empty = kv ? BAR_VE : BAR_KE;
      const CUtensorMap* map = kv ? &tmV : &tmK;
      const uint32_t ring = sbase + (kv ? kSmemV : kSmemK);
      const uint32_t stage_bytes = kv ? kVBytes : kKBytes;
      int gs = 0, qc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = cluster + k * nclusters;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = cx.wait(bar(BAR_LF + buf), (k >> 1) & 1))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int tile = inf->tile, b = inf->b, g = inf->g, i = inf->i;
          if (kv == 0) {
            const int qslot = qc & 1;
            if (qc >= 2 && !(ok = cx.wait(bar(BAR_QE + qslot), ((qc >> 1) - 1) & 1))) break;
            // rows past the unit (an odd tile count) load other rows or the
            // zero fill past the tensor; their results are never stored
            if (rank == 0) mbar_arrive_expect_tx(bar(BAR_QF + qslot), 2u * kQBytes);
            const uint32_t qbar = lead(BAR_QF + qslot);
            for (int pc = 0; pc < 2; ++pc) {
              const int R0 = tile * 128 + pc * 64;
              const int h = g * p.G + R0 / BS;
              const int y = (b * p.Hq + h) * p.N + i * BS + R0 % BS;
              for (int hf = 0; hf < 2; ++hf)
                tma_load_2d_pair(sbase + kSmemQ + qslot * kQBytes + hf * kQHalf + pc * 8192, &tmQ, qbar, hf * 64,
                                 y);
            }
            ++qc;
          }
          const int kvrow0 = (b * p.Hkv + g) * p.N;
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int slot = gs % kStages;
            if (gs >= kStages && !(ok = cx.wait(bar(empty + slot), ((gs / kStages) - 1) & 1))) break;
            const uint32_t dst0 = ring + slot * stage_bytes;
            const uint32_t fbar = lead(full + slot);
            if (kv == 0) {
              // K: this CTA's N half of the step's keys, both 64-channel halves
              int y;
              if (BS == 64) {
                const bool two = 2 * s + 1 < n;
                y = two ? kvrow0 + inf->list[2 * s + rank] * 64 : kvrow0 + inf->list[2 * s] * 64 + rank * 32;
              } else {
                y = kvrow0 + inf->list[s] * 128 + rank * 64;
              }
              if (rank == 0) mbar_arrive_expect_tx(bar(full + slot), 2u * kKBytes);
              for (int hf = 0; hf < 2; ++hf) tma_load_2d_pair(dst0 + hf * kKHalf, map, fbar, hf * 64, y);
            } else {
              // V: all keys of the step, this CTA's 64 channels
              const int nrow = (BS == 64) ? ((2 * s + 1 < n) ? 2 : 1) : 2;
              if (rank == 0) mbar_arrive_expect_tx(bar(full + slot), 2u * static_cast<uint32_t>(nrow) * 8192u);
              for (int r = 0; r < nrow; ++r) {
                const int y = (BS == 64) ? kvrow0 + inf->list[2 * s + r] * 64 : kvrow0 + inf->list[s] * 128 + r * 64;
                tma_load_2d_pair(dst0 + r * 8192u, map, fbar, static_cast<int>(rank) * 64, y);
              }
            }
          }
          if (!ok) break;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (*cx.abortp && rank == 0) {
        // let the copies of both CTAs counted on this CTA's barriers land
        for (int c = max(0, qc - 2); c < qc; ++c) mbar_drain_cluster(bar(BAR_QF + (c & 1)), (c >> 1) & 1);
        for (int s = max(0, gs - kStages); s < gs; ++s) mbar_drain_cluster(bar(full + s % kStages), (s / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (even CTA)
      const uint32_t id_s128 = idesc_bf16_f32(256, 128, 0, 0);
      const uint32_t id_s64 = idesc_bf16_f32(256, 64, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(256, 128, 0, 1);
      const uint64_t q_desc0 = smem_desc_sw128(sbase + kSmemQ, 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(sbase + kSmemK, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(sbase + kSmemV, kVBytes, 1024);
      auto issue_s = [&](int qslot, int kslot, int sbuf, int keys) {
        const uint64_t qd = q_desc0 + ((qslot * kQBytes) >> 4);
        const uint64_t kd = k_desc0 + ((kslot * kKBytes) >> 4);
        const uint32_t id = (keys == 128) ? id_s128 : id_s64;
        const uint32_t d_tmem = tmem + sbuf * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * kKHalf + (kk & 3) * 32) >> 4;
          mma2_ss(d_tmem, qd + qoff, kd + koff, id, kk > 0 ? 1u : 0u);
        }
      };
      // O_h += P_h V: the 64 keys of half h, P from its S buffer columns
      auto issue_pv_half = [&](int h, int vslot, int sbuf, bool acc) {
        const uint64_t vd = v_desc0 + ((vslot * kVBytes) >> 4);
        const uint32_t d_tmem = tmem + kColO + h * 128;
        const uint32_t a_tmem = tmem + sbuf * 128 + h * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma2_ts(d_tmem, a_tmem + kk * 8, vd + (((h * 4 + kk) * 2048) >> 4), id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      int gs = 0, qc = 0, items_pv = 0;
      int pend_g = -1, pend_keys = 0;   // the step whose O += P V is still to be issued
      bool pend_first = false;
      auto issue_pv = [&]() -> bool {
        const int g = pend_g, vslot = g % kStages, sb = g & 1;
        if (!cx.wait(bar(BAR_VF + vslot), (g / kStages) & 1)) return false;
        if (pend_first) {
          // both CTAs' epilogues must have read the previous item's O_0 and O_1
          if (items_pv > 0 && !cx.wait(bar(BAR_OE), (items_pv - 1) & 1)) return false;
          ++items_pv;
        }
        if (!cx.wait(bar(BAR_PF + sb), (g >> 1) & 1)) return false;
        tc_fence_after();
        issue_pv_half(0, vslot, sb, !pend_first);
        if (pend_keys == 128) {
          if (!cx.wait(bar(BAR_PF + 2 + sb), (g >> 1) & 1)) return false;
          tc_fence_after();
          issue_pv_half(1, vslot, sb, !pend_first);
        }
        tc_commit_pair_mc(bar(BAR_VE + vslot), kBoth);
        return true;
      };
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = cluster + k * nclusters;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = cx.wait(bar(BAR_LF + buf), (k >> 1) & 1))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          const int qslot = qc & 1;
          if (!(ok = cx.wait(bar(BAR_QF + qslot), (qc >> 1) & 1))) break;
          ++qc;
          tc_fence_after();
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int kslot = gs % kStages;
            const int keys = (BS == 64) ? ((2 * s + 1 < n) ? 128 : 64) : 128;
            if (!(ok = cx.wait(bar(BAR_KF + kslot), (gs / kStages) & 1))) break;
            tc_fence_after();
            issue_s(qslot, kslot, gs & 1, keys);
            tc_commit_pair_mc(bar(BAR_SF + (gs & 1)), kBoth);
            tc_commit_pair_mc(bar(BAR_KE + kslot), kBoth);
            if (s == nsteps - 1) tc_commit_pair_mc(bar(BAR_QE + qslot), kBoth);
            if (pend_g >= 0 && !(ok = issue_pv())) break;
            pend_g = gs;
            pend_keys = keys;
            pend_first = (s == 0);
          }
          if (!ok) break;
        } else if (pend_g >= 0) {
          // an item without keys: issue the pending O += P V now (the next
          // item's metadata slot is only refilled after that item's epilogue)
          if (!(ok = issue_pv())) break;
          pend_g = -1;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (ok && pend_g >= 0) ok = issue_pv();
      if (!ok) {
        // every MMA issued so far must finish before tensor memory is freed
        tc_commit_pair(bar(BAR_AB));
        mbar_drain(bar(BAR_AB), 0);
      }
    }
  }
  } else {
    set_regs_inc<kMathRegs>();
    // ------------------------------------------------ softmax + epilogue
    const int h = (warp - 4) >> 2;   // key half
    const int q4 = warp & 3;         // TMEM lane quadrant
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t t_o = lane_addr + kColO + h * 128;
    const uint32_t oe_lead = lead(BAR_OE);
    int gs = 0, items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = cluster + k * nclusters;
      if (item >= p.num_items) break;
      const int buf = k & 1;
      if (!(ok = cx.warp_wait(bar(BAR_LF + buf), (k >> 1) & 1))) break;
      const ItemInfo* inf = &misc->info[buf];
      const int n = inf->n;
      const int b = inf->b, g = inf->g, i = inf->i;
      const int R = inf->tile * 128 + r;
      const bool valid = R < p.rows_per_unit;
      const int hrow = g * p.G + (valid ? R / BS : 0);
      const int tb = R % BS;
      const int64_t orow_idx = (static_cast<int64_t>(b) * p.Hq + hrow) * p.N + i * BS + tb;
      if (n == 0) {
        if (valid) {
          __nv_bfloat16* orow = p.o + orow_idx * kD + h * 64;
          for (int c = 0; c < 64; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
          if (h == 0 && p.lse) p.lse[orow_idx] = -INFINITY;
        }
      } else {
        const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
        float m_run = -INFINITY, l_run = 0.0f;
        bool had = false;
        for (int s = 0; s < nsteps; ++s, ++gs) {
          const int sb = gs & 1;
          if (!(ok = cx.warp_wait(bar(BAR_SF + sb), (gs >> 1) & 1))) break;
          tc_fence_after();
          const int e = (BS == 64) ? 2 * s + h : s;
          if (e < n) {
            const int j = inf->list[e];
            const float bias = inf->bias[e];
            const int koff0 = (BS == 64) ? 0 : h * 64;
            const uint32_t t_s = lane_addr + sb * 128 + h * 64;
            const uint32_t ve = bar(BAR_VE + ((gs + kStages - 1) % kStages));
            const uint32_t vpar = ((gs - 1) / kStages) & 1;
            if (j == i)
              ok = softmax_half<true>(t_s, t_o, !had, p.scale_log2, bias, koff0, tb, m_run, l_run, ve, vpar, cx);
            else
              ok = softmax_half<false>(t_s, t_o, !had, p.scale_log2, bias, koff0, tb, m_run, l_run, ve, vpar, cx);
            if (!ok) break;
            had = true;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(BAR_PF + h * 2 + sb));
        }
        if (!ok) break;
        // ---- epilogue: merge the two halves' partials of each row
        const int last = gs - 1;
        if (!(ok = cx.warp_wait(bar(BAR_VE + last % kStages), (last / kStages) & 1))) break;
        tc_fence_after();
        const int eb = items & 1;
        misc->ml[eb][h][r] = make_float2(m_run, l_run);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_ML));
        if (!(ok = cx.warp_wait(bar(BAR_ML), items & 1))) break;
        const float2 other = misc->ml[eb][h ^ 1][r];
        const bool has1 = (BS == 128) || n >= 2;   // half 1 held keys in this item
        const float m0 = h ? other.x : m_run, l0 = h ? other.y : l_run;
        const float m1 = h ? m_run : other.x, l1 = h ? l_run : other.y;
        const float m = fmaxf(m0, m1);
        const float w0 = (m0 == -INFINITY) ? 0.0f : fast_exp2(m0 - m);
        const float w1 = (!has1 || m1 == -INFINITY) ? 0.0f : fast_exp2(m1 - m);
        const float L = l0 * w0 + l1 * w1;
        const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
        const float c0 = w0 * inv, c1 = w1 * inv;
        uint32_t ob[32];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t a[32], bv[32];
          tmem_ld32(lane_addr + kColO + h * 64 + ch * 32, a);
          if (has1) {
            tmem_ld32(lane_addr + kColO + 128 + h * 64 + ch * 32, bv);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              ob[ch * 16 + e] =
                  pack_bf16x2(fmaf(__uint_as_float(a[2 * e]), c0, __uint_as_float(bv[2 * e]) * c1),
                              fmaf(__uint_as_float(a[2 * e + 1]), c0, __uint_as_float(bv[2 * e + 1]) * c1));
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              ob[ch * 16 + e] = pack_bf16x2(__uint_as_float(a[2 * e]) * c0, __uint_as_float(a[2 * e + 1]) * c0);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(oe_lead);   // O may be overwritten by the next item from here on
        ++items;
        if (valid) {
          if (p.o_v8) {
#pragma unroll
            for (int e = 0; e < 4; ++e) st_global_v8(p.o + orow_idx * kD + h * 64 + 16 * e, ob + 8 * e);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(p.o + orow_idx * kD + h * 64);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2], ob[4 * e + 3]);
          }
          if (h == 0 && p.lse) p.lse[orow_idx] = (L > 0.0f) ? (m + __log2f(L)) * kLn2 : -INFINITY;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LE + buf));
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // neither CTA leaves while the pair's MMAs, copies or arrives may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

template <int BS>
static cudaError_t launch_bs(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                             const Params& p, int max_clusters, cudaStream_t st) {
  auto kern = attn_prefill_pair_kernel<BS>;
  cudaError_t e = ensure_dynamic_smem<attn_prefill_pair_kernel<BS>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many clusters as fit on the device at once (persistent kernel); the
  // answer is kept per device and context
  static std::atomic<uint64_t> fit_ctx[32];
  static std::atomic<int> fit_val[32];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
  const uint64_t ctx = current_context_id();
  int fit = fit_val[dev].load(std::memory_order_acquire);
  if (ctx == 0 || fit_ctx[dev].load(std::memory_order_acquire) != ctx || fit < 1) {
    cfg.gridDim = dim3(2 * max_clusters);
    e = cudaOccupancyMaxActiveClusters(&fit, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (fit < 1) return cudaErrorInvalidConfiguration;
    fit_val[dev].store(fit, std::memory_order_release);
    fit_ctx[dev].store(ctx, std::memory_order_release);
  }
  if (fit > max_clusters) fit = max_clusters;
  const int clusters = p.num_items < fit ? p.num_items : fit;
  cfg.gridDim = dim3(2 * clusters);
  return cudaLaunchKernelEx(&cfg, kern, *tmQ, *tmK, *tmV, p);
}

}  // namespace prefill_pair

cudaError_t launch_attn_prefill_pair_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                          const PrefillArgs& a, cudaStream_t st) {
  prefill_pair::Params p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.N = a.N;
  p.nb = a.N / a.bs;
  p.G = a.Hq / a.Hkv;
  p.rows_per_unit = p.G * a.bs;
  p.tiles_per_unit = (p.rows_per_unit + 127) / 128;
  p.pairs_per_unit = (p.tiles_per_unit + 1) / 2;
  const int64_t items = static_cast<int64_t>(a.B) * a.Hkv * p.nb * p.pairs_per_unit;
  if (items <= 0) return cudaSuccess;
  p.num_items = static_cast<int>(items);
  p.idx = a.idx;
  p.idx_stride = a.idx_stride;
  p.sel = a.sel_scores;
  p.scale_log2 = a.softmax_scale * prefill_pair::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) & 31u) == 0 ? 1 : 0;
  p.lse = a.lse;
  p.status = a.status;
  const int max_clusters = a.num_sms / 2;
  if (a.bs == 64) return prefill_pair::launch_bs<64>(tmQ, tmK, tmV, p, max_clusters, st);
  return prefill_pair::launch_bs<128>(tmQ, tmK, tmV, p, max_clusters, st);
}

}  // namespace bsa
