// attn_prefill_split.cu -- block-sparse causal attention, prefill, bf16,
// d = 128, on sm_100a tensor cores (tcgen05 MMA into tensor memory, TMA tile
// loads): the one-tile-per-item kernel with split key halves.
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
// When it runs.  attn_prefill.cu pairs two 128-row tiles of a unit per item,
// so each K/V tile is fetched once per 256 rows; a unit with an odd number of
// tiles leaves one tile without a partner there, and that tile runs its
// softmax -> O += P V -> next S chain alone.  Units with an odd tile count
// (G*bs/128 rounded up) come here instead: every item is one tile, and the
// two S buffers keep the tensor core busy during the softmax, at the price of
// fetching each K/V tile once per 128 rows.
//
// Work decomposition.  A unit is (batch b, KV group g, query block i): the
// G heads of the group share one kept-block list, so their bs query rows
// each are stacked into G*bs rows that all read the same K/V tiles.  An item
// is one 128-row tile of a unit; the tiles of a unit are consecutive items,
// so the CTAs that run them at the same time share the unit's K/V tiles
// through L2.  The kernel is persistent: one CTA per SM walks items
// blockIdx.x, +gridDim.x, ... (heavy items first); the K/V rings, the two Q
// slots and the item metadata roll over from one item to the next, so the
// next item's loads and first S = Q K^T overlap the previous item's tail.
//
// A step covers 128 keys: two 64-token blocks (bs = 64) or one 128-token
// block (bs = 128); the last step of an odd list holds one 64-token block.
// Each step is split into two key halves of 64 keys (for bs = 64: one block
// each).  Half h has its own softmax warps, its own running maximum and sum
// per row and its own output accumulator O_h; the two partial results of a
// row are merged once, in the epilogue, by the usual rescale-and-add of two
// softmax partials.  So the halves never exchange per-step maxima.
//
// Roles (384 threads, three warpgroups):
//   warp 0      TMA producer of Q (per item, two slots) and K (per step,
//               two-stage ring, gathered by block index);
//   warp 3      TMA producer of V (per step, two-stage ring);
//   warp 1      TMEM owner + MMA issuer (one thread): S(s) = Q K^T into
//               S buffer s mod 2 (SS form), then O_h += P_h(s-1) V_h for the
//               previous step (TS form, P from tensor memory); the issue
//               order runs across item boundaries, so S of an item's first
//               step is issued before O += P V of the previous item's last;
//   warp 2      item loader: kept-block list and gate biases into a
//               double-buffered metadata slot;
//   warps 4-7   softmax of key half 0 (thread = query row = TMEM lane);
//   warps 8-11  softmax of key half 1; the epilogue is shared: warps of half
//               h write output columns 64h..64h+63 of their rows.
// The control warpgroup gives registers up (setmaxnreg) to the softmax
// warpgroups.
// Tensor memory (512 columns): S buffer 0 | S buffer 1 | O_0 | O_1, 128
// columns each.  Half h writes its P (bf16 pairs, 32 columns) over the
// first half of its own 64 S columns.  Two S buffers let S(s+1) run on the
// tensor core while the softmax of step s runs; tcgen05.mma instructions
// from one thread execute in issue order, so S(s+2), issued after
// O += P(s) V, never overwrites P(s) before that MMA has read it.
//
// Softmax uses the base-2 exponent with the scale and the gate bias folded
// into one packed (f32x2) FMA per key pair, and a lazy rescale: the running
// maximum is only moved (and O_h rescaled in tensor memory, after the
// previous step's O_h += P V has completed) when a row's new maximum exceeds
// it by more than 8 (a factor 256), which keeps every P <= 256 and is exact
// after the final division.
#include "common.cuh"
#include "kernels.h"
#include "tmem_wide.cuh"


namespace bsa {
namespace prefill_split {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kStages = 2;
constexpr int kMaxList = 256;
constexpr uint32_t kHalfBytes = 128u * 128u;          // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kTileBytes = 2u * kHalfBytes;      // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;                        // two Q slots
constexpr uint32_t kSmemK = kSmemQ + 2 * kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kTileBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kTileBytes;
constexpr uint32_t kColO = 256;     // O_0 at 256, O_1 at 384; S buffers at 0 and 128
constexpr int kCtrlRegs = 120;      // warps 0-3 after setmaxnreg.dec
constexpr int kMathRegs = 184;      // warps 4-11 after setmaxnreg.inc (128*120 + 256*184 <= 384*168)
static_assert(128 * kCtrlRegs + 256 * kMathRegs <= kThreads * 168, "register split exceeds the launch pool");

enum {
  BAR_QF = 0,                  // per Q slot: loaded
  BAR_QE = BAR_QF + 2,         // per Q slot: the item's last S has completed
  BAR_KF = BAR_QE + 2,         // per K stage: loaded (the stage is free again once S of its step completes)
  BAR_VF = BAR_KF + kStages,   // per V stage: loaded
  BAR_VE = BAR_VF + kStages,   // per V stage: O += P V of its step completed
  BAR_SF = BAR_VE + kStages,   // per S buffer: S complete
  BAR_PF = BAR_SF + 2,         // per (half, S buffer): P written
  BAR_OE = BAR_PF + 4,         // O_0 and O_1 read back by the epilogue
  BAR_ML = BAR_OE + 1,         // both halves' (m, l) of an item published
  BAR_LF = BAR_ML + 1,         // per metadata slot: filled
  BAR_LE = BAR_LF + 2,         // per metadata slot: consumed by every role
  BAR_AB = BAR_LE + 2,
  NUM_BARS
};
constexpr uint32_t kListConsumers = 3 + 8;   // two producers, MMA, one lane per softmax warp

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
  int rows_per_unit, tiles_per_unit, num_items;
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

// One softmax step of one key half (64 keys of this thread's row).  t_s: the
// half's 64 S columns, t_o: the half's O accumulator.  MASK: the keys are in
// the query block itself (causal mask: key offset koff0 + c against the
// row's offset tb).  A rescale of O first waits (ve_bar, ve_par) for the
// previous step's O += P V.  Returns false only when that wait was aborted.
template <bool MASK>
__device__ __forceinline__ bool softmax_half(uint32_t t_s, uint32_t t_o, bool first, float scale_log2, float bias,
                                             int koff0, int tb, float& m_run, float& l_run, uint32_t ve_bar,
                                             uint32_t ve_par, volatile int* ab, uint32_t* status) {
  uint32_t v[64];
  tmem_ld64(t_s, v);
  if constexpr (MASK) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (koff0 + c > tb) v[c] = 0xFF800000u;   // -inf
  }
  // row maximum of the raw scores (the scale is positive and the bias is
  // constant over the half, so the maximum commutes with both); three-input
  // maxima in 8 independent chains
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
    if (!warp_wait(ve_bar, ve_par, ab, status)) return false;
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
  // p = 2^(s * scale*log2(e) + bias - m), two keys per packed FMA; packed
  // partial row sums
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
  const uint64_t off = f2_pack(bias - m_sub, bias - m_sub);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // independent packed partial row sums (+0.0f pairs)
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
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BAR_QF + s), 1);
      mbar_init(bar(BAR_QE + s), 1);
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
      mbar_init(bar(BAR_SF + s), 1);
      mbar_init(bar(BAR_PF + s), 4);       // one arrive per softmax warp of half 0
      mbar_init(bar(BAR_PF + 2 + s), 4);   // ... of half 1
      mbar_init(bar(BAR_LF + s), 1);
      mbar_init(bar(BAR_LE + s), kListConsumers);
    }
    mbar_init(bar(BAR_OE), 8);
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
      const int unit = item / p.tiles_per_unit, tile = item % p.tiles_per_unit;
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
        inf->b = bg / p.Hkv;
        inf->g = bg % p.Hkv;
        inf->i = i;
        inf->tile = tile;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LF + buf));
    }
  } else if (warp == 0 || warp == 3) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producers
      // warp 0 loads Q and K, warp 3 loads V: the K stage of a step is free
      // once its S has completed, the V stage once its O += P V has.
      const int kv = (warp == 3) ? 1 : 0;
      const int full = kv ? BAR_VF : BAR_KF, empty = kv ? BAR_VE : BAR_SF;
      const CUtensorMap* map = kv ? &tmV : &tmK;
      const uint32_t ring = sbase + (kv ? kSmemV : kSmemK);
      int gs = 0, qc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int tile = inf->tile, b = inf->b, g = inf->g, i = inf->i;
          if (kv == 0) {
            const int qslot = qc & 1;
            if (qc >= 2 && !(ok = mbar_wait(bar(BAR_QE + qslot), ((qc >> 1) - 1) & 1, abortp, p.status))) break;
            uint32_t qbytes = 0;
            for (int pc = 0; pc < 2; ++pc)
              if (tile * 128 + pc * 64 < p.rows_per_unit) qbytes += 2 * 8192;
            mbar_arrive_expect_tx(bar(BAR_QF + qslot), qbytes);
            for (int pc = 0; pc < 2; ++pc) {
              const int R0 = tile * 128 + pc * 64;
              if (R0 >= p.rows_per_unit) continue;
              const int h = g * p.G + R0 / BS;
              const int y = (b * p.Hq + h) * p.N + i * BS + R0 % BS;
              for (int hf = 0; hf < 2; ++hf)
                tma_load_2d(sbase + kSmemQ + qslot * kTileBytes + hf * kHalfBytes + pc * 8192, &tmQ,
                            bar(BAR_QF + qslot), hf * 64, y);
            }
            ++qc;
          }
          const int kvrow0 = (b * p.Hkv + g) * p.N;
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int slot = gs % kStages;
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
            if (gs >= kStages && !(ok = mbar_wait(bar(empty + slot), ((gs / kStages) - 1) & 1, abortp, p.status)))
              break;
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
        for (int c = max(0, qc - 2); c < qc; ++c) mbar_drain(bar(BAR_QF + (c & 1)), (c >> 1) & 1);
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
      auto issue_s = [&](int qslot, int kslot, int sbuf, int keys) {
        const uint64_t qd = q_desc0 + ((qslot * kTileBytes) >> 4);
        const uint64_t kd = k_desc0 + ((kslot * kTileBytes) >> 4);
        const uint32_t id = (keys == 128) ? id_s128 : id_s64;
        const uint32_t d_tmem = tmem + sbuf * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss(d_tmem, qd + off, kd + off, id, kk > 0 ? 1u : 0u);
        }
      };
      // O_h += P_h V_h: the 64 keys of half h, P from its S buffer columns
      auto issue_pv_half = [&](int h, int vslot, int sbuf, bool acc) {
        const uint64_t vd = v_desc0 + ((vslot * kTileBytes) >> 4);
        const uint32_t d_tmem = tmem + kColO + h * 128;
        const uint32_t a_tmem = tmem + sbuf * 128 + h * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(d_tmem, a_tmem + kk * 8, vd + (((h * 4 + kk) * 2048) >> 4), id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      int gs = 0, qc = 0, items_pv = 0;
      int pend_g = -1, pend_keys = 0;   // the step whose O += P V is still to be issued
      bool pend_first = false;
      auto issue_pv = [&]() -> bool {
        const int g = pend_g, vslot = g % kStages, sb = g & 1;
        if (!mbar_wait(bar(BAR_VF + vslot), (g / kStages) & 1, abortp, p.status)) return false;
        if (pend_first) {
          // the previous item's epilogue must have read O_0 and O_1
          if (items_pv > 0 && !mbar_wait(bar(BAR_OE), (items_pv - 1) & 1, abortp, p.status)) return false;
          ++items_pv;
        }
        if (!mbar_wait(bar(BAR_PF + sb), (g >> 1) & 1, abortp, p.status)) return false;
        tc_fence_after();
        issue_pv_half(0, vslot, sb, !pend_first);
        if (pend_keys == 128) {
          if (!mbar_wait(bar(BAR_PF + 2 + sb), (g >> 1) & 1, abortp, p.status)) return false;
          tc_fence_after();
          issue_pv_half(1, vslot, sb, !pend_first);
        }
        tc_commit(bar(BAR_VE + vslot));
        return true;
      };
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        if (item >= p.num_items) break;
        const int buf = k & 1;
        if (!(ok = mbar_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
        const ItemInfo* inf = &misc->info[buf];
        const int n = inf->n;
        if (n > 0) {
          const int nsteps = (BS == 64) ? (n + 1) / 2 : n;
          const int qslot = qc & 1;
          if (!(ok = mbar_wait(bar(BAR_QF + qslot), (qc >> 1) & 1, abortp, p.status))) break;
          ++qc;
          tc_fence_after();
          for (int s = 0; s < nsteps; ++s, ++gs) {
            const int kslot = gs % kStages;
            const int keys = (BS == 64) ? ((2 * s + 1 < n) ? 128 : 64) : 128;
            if (!(ok = mbar_wait(bar(BAR_KF + kslot), (gs / kStages) & 1, abortp, p.status))) break;
            tc_fence_after();
            issue_s(qslot, kslot, gs & 1, keys);
            tc_commit(bar(BAR_SF + (gs & 1)));
            if (s == nsteps - 1) tc_commit(bar(BAR_QE + qslot));   // Q slot free once this S completes
            if (pend_g >= 0 && !(ok = issue_pv())) break;
            pend_g = gs;
            pend_keys = keys;
            pend_first = (s == 0);
          }
          if (!ok) break;
        } else if (pend_g >= 0) {
          // An item without keys: the pending O += P V cannot wait for the
          // next item's first S, whose metadata slot is only refilled after
          // the pending item's epilogue, which needs this MMA.
          if (!(ok = issue_pv())) break;
          pend_g = -1;
        }
        mbar_arrive(bar(BAR_LE + buf));
      }
      if (ok && pend_g >= 0) ok = issue_pv();
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
    const int h = (warp - 4) >> 2;   // key half
    const int q4 = warp & 3;         // TMEM lane quadrant
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t t_o = lane_addr + kColO + h * 128;
    int gs = 0, items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = blockIdx.x + k * gridDim.x;
      if (item >= p.num_items) break;
      const int buf = k & 1;
      if (!(ok = warp_wait(bar(BAR_LF + buf), (k >> 1) & 1, abortp, p.status))) break;
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
          if (!(ok = warp_wait(bar(BAR_SF + sb), (gs >> 1) & 1, abortp, p.status))) break;
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
              ok = softmax_half<true>(t_s, t_o, !had, p.scale_log2, bias, koff0, tb, m_run, l_run, ve, vpar, abortp,
                                      p.status);
            else
              ok = softmax_half<false>(t_s, t_o, !had, p.scale_log2, bias, koff0, tb, m_run, l_run, ve, vpar,
                                       abortp, p.status);
            if (!ok) break;
            had = true;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_PF + h * 2 + sb));
        }
        if (!ok) break;
        // ---- epilogue: merge the two halves' partials of each row
        const int last = gs - 1;
        if (!(ok = warp_wait(bar(BAR_VE + last % kStages), (last / kStages) & 1, abortp, p.status))) break;
        tc_fence_after();
        const int eb = items & 1;
        misc->ml[eb][h][r] = make_float2(m_run, l_run);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_ML));
        if (!(ok = warp_wait(bar(BAR_ML), items & 1, abortp, p.status))) break;
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
        if (lane == 0) mbar_arrive(bar(BAR_OE));   // O may be overwritten by the next item from here on
        ++items;
        if (valid) {
          if (p.o_v8) {   // whole 32-byte sectors per store
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

}  // namespace prefill_split

cudaError_t launch_attn_prefill_split_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                           const PrefillArgs& a, cudaStream_t st) {
  prefill_split::Params p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.N = a.N;
  p.nb = a.N / a.bs;
  p.G = a.Hq / a.Hkv;
  p.rows_per_unit = p.G * a.bs;
  p.tiles_per_unit = (p.rows_per_unit + 127) / 128;
  const int64_t items = static_cast<int64_t>(a.B) * a.Hkv * p.nb * p.tiles_per_unit;
  if (items <= 0) return cudaSuccess;
  p.num_items = static_cast<int>(items);
  p.idx = a.idx;
  p.idx_stride = a.idx_stride;
  p.sel = a.sel_scores;
  p.scale_log2 = a.softmax_scale * prefill_split::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) & 31u) == 0 ? 1 : 0;
  p.lse = a.lse;
  p.status = a.status;
  const unsigned grid = static_cast<unsigned>(items < a.num_sms ? items : a.num_sms);
  if (a.bs == 64) return prefill_split::launch_bs<64>(tmQ, tmK, tmV, p, grid, st);
  return prefill_split::launch_bs<128>(tmQ, tmK, tmV, p, grid, st);
}

}  // namespace bsa
