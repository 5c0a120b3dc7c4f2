// attn_bwd.cu -- backward of the block-sparse (and SAS gated) prefill
// attention, bf16 inputs, d = 128, on sm_100a tensor cores (tcgen05 MMA into
// tensor memory, TMA tile loads).
//
// What it computes (SAS page, 核心洞察 and 核心模块 2: the selector's
// continuous score sits inside the softmax logits in log form, so the
// language-modelling loss reaches it by ordinary back-propagation).  With the
// forward's P_{t,u} = exp(scale q_t.k_u + log g_{j(u)} - LSE_t) over the kept,
// causal keys of row t (LSE_t: the forward's natural-log row LSE) and the
// upstream gradient dO:
//   D_t      = sum_u P_{t,u} (dO_t . v_u)        (= dO_t . O_t in exact arithmetic;
//              formed from P and V rather than from the stored bf16 O, whose
//              rounding would otherwise enter every gradient through D)
//   dS_{t,u} = P_{t,u} (dO_t . v_u - D_t)
//   dQ_t     = scale sum_u dS_{t,u} k_u
//   dK_u     = scale sum_t dS_{t,u} q_t,  dV_u = sum_t P_{t,u} dO_t
//   for a unit (b, g, i) and its kept block l:
//   dsel_l   = dlogg_l - g_l sum_j dlogg_j,  dlogg_j = sum over the unit's
//              rows t and block j's keys u of dS_{t,u}.
// P is recomputed from Q, K and the saved LSE (no n x n storage).  Two
// passes, neither accumulating by atomics, every sum in a fixed order:
//   query-major (dq_tc_kernel): per 128-row tile of a unit (the unit's G
//     heads' rows stacked, as in the forward), two sweeps over its kept
//     blocks: S = Q K^T and dP = dO V^T on the tensor core, the first sweep
//     sums D_t, the second writes dS (bf16) over S in tensor memory and
//     accumulates dQ += dS K there, plus the rows' share of dlogg;
//   key-major (dkv_tc_kernel): per key block j, every (query block i that
//     kept j, 128 of its rows): S^T = K Q^T and dP^T = V dO^T, then P^T and
//     dS^T (bf16) over them, dV += P^T dO and dK += dS^T Q accumulated in
//     tensor memory over all of them (a transposed index, built first, lists
//     the query blocks of each key block).
// P and dS enter the dQ/dK/dV products rounded to bf16, as the forward's P
// enters O += P V; D and dlogg are summed in fp32 from the unrounded values.
//
// Roles of both kernels (192 threads): warps 0-3 one TMEM lane each (a row
// in the query-major pass, a key in the key-major one), warp 4 one thread
// issuing the MMAs, warp 5 one thread issuing the TMA loads.  Waits are
// bounded (mbarrier try-wait with a clock budget); a wait that gives up
// raises the CTA's abort flag and the device status word.
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace bwd {

constexpr int kD = 128;
constexpr int kMaxList = 256;
constexpr int kThreadsTC = 192;
constexpr uint32_t kHalf = 128u * 128u;   // 128 rows x 64 bf16 (one swizzle span)
constexpr uint32_t kTile = 2u * kHalf;    // 128 rows x 128 bf16
constexpr float kLog2e = 1.44269504088896340736f;

// A wait by a whole warp: every lane polls, all agree on the outcome.
__device__ __forceinline__ bool warp_wait_all(uint32_t bar, uint32_t parity, volatile int* ab, uint32_t* st) {
  bool ok = mbar_wait(bar, parity, ab, st);
  return __all_sync(0xffffffffu, ok);
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
// with the slot of j in i's list.  One CTA per (b, g): counts per key block
// by shared-memory atomics, an exclusive scan, then the fill, which walks the
// query blocks in ascending order (a list's entries are distinct, so its
// entries take their cursors without conflict), so every transposed list
// comes out in a fixed order.  Lists are staged in shared memory kTrChunk at
// a time.  Dynamic shared memory: transpose_smem_bytes(nb, idx_stride).
constexpr int kTrThreads = 256;
constexpr int kTrChunk = 32;
inline size_t transpose_smem_bytes(int nb, int idx_stride) {
  return static_cast<size_t>(nb) * sizeof(int) + static_cast<size_t>(kTrChunk) * (idx_stride + 1) * sizeof(int) +
         kTrThreads * sizeof(int);
}

__global__ void __launch_bounds__(kTrThreads) transpose_kernel(const int* __restrict__ lists,
                                                               const int* __restrict__ counts, int idx_stride,
                                                               int nb, int* __restrict__ toff,
                                                               int2* __restrict__ tlist) {
  extern __shared__ int tr_sm[];
  int* cur = tr_sm;                            // [nb] counts, then cursors
  int* lbuf = cur + nb;                        // [kTrChunk][idx_stride] staged lists
  int* lcnt = lbuf + kTrChunk * idx_stride;    // [kTrChunk] their counts
  int* part = lcnt + kTrChunk;                 // [kTrThreads] scan partials
  const int bg = blockIdx.x, tid = threadIdx.x;
  const int64_t ubase = static_cast<int64_t>(bg) * nb;
  int* off = toff + static_cast<int64_t>(bg) * (nb + 1);
  int2* tl = tlist + ubase * idx_stride;
  for (int j = tid; j < nb; j += kTrThreads) cur[j] = 0;
  auto stage = [&](int i0) {
    __syncthreads();
    const int nl = min(kTrChunk, nb - i0);
    for (int x = tid; x < nl * idx_stride; x += kTrThreads)
      lbuf[x] = lists[(ubase + i0) * idx_stride + x];
    for (int x = tid; x < nl; x += kTrThreads) lcnt[x] = counts[ubase + i0 + x];
    __syncthreads();
    return nl;
  };
  // counts
  for (int i0 = 0; i0 < nb; i0 += kTrChunk) {
    const int nl = stage(i0);
    for (int x = tid; x < nl * idx_stride; x += kTrThreads)
      if (x % idx_stride < lcnt[x / idx_stride]) atomicAdd(&cur[lbuf[x]], 1);
  }
  __syncthreads();
  // exclusive scan: each thread a contiguous segment
  const int seg = (nb + kTrThreads - 1) / kTrThreads;
  const int j0 = min(nb, tid * seg), j1 = min(nb, j0 + seg);
  int sum = 0;
  for (int j = j0; j < j1; ++j) sum += cur[j];
  part[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int t = 0; t < kTrThreads; ++t) {
      const int v = part[t];
      part[t] = acc;
      acc += v;
    }
    off[nb] = acc;
  }
  __syncthreads();
  int acc = part[tid];
  for (int j = j0; j < j1; ++j) {
    const int v = cur[j];
    cur[j] = acc;
    off[j] = acc;
    acc += v;
  }
  // fill: query blocks in ascending order, one list at a time
  for (int i0 = 0; i0 < nb; i0 += kTrChunk) {
    const int nl = stage(i0);
    for (int x = 0; x < nl; ++x) {
      const int c = lcnt[x];
      for (int s = tid; s < c; s += kTrThreads) {
        const int j = lbuf[x * idx_stride + s];
        tl[cur[j]++] = make_int2(i0 + x, s);
      }
      __syncthreads();
    }
  }
}

struct Params {
  const float *lse, *logg;
  const int *lists, *counts, *toff;
  const int2* tlist;
  float* D;                 // written by the query-major pass, read by the key-major pass
  float* dlogg_part;        // [units][idx_stride][tiles]
  int B, Hq, Hkv, N, nb, G, idx_stride, tiles;   // tiles: 128-row tiles per unit
  float scale;
  float *dq, *dk, *dv;
  uint32_t* status;
};

// ------------------------------------------------------------------ query-major
// Steps of 64 keys; two S | dP buffers in tensor memory, so the MMAs of step
// s+1 run while the lanes work on step s.
namespace qm {
constexpr int kStagesK = 4;                                    // K/V stages of 64 keys
constexpr uint32_t kKV = 64u * 128u * 2u;                      // 64 keys x 128 bf16
constexpr uint32_t kKVHalf = kKV / 2;
constexpr uint32_t SM_Q = 0, SM_DO = kTile;
constexpr uint32_t SM_K = 2 * kTile, SM_V = SM_K + kStagesK * kKV;
constexpr uint32_t SM_RED = SM_V + kStagesK * kKV;              // float [4][kMaxList]
constexpr uint32_t SM_BAR = SM_RED + 4 * kMaxList * 4;
enum { QF = 0, QE, KF, KE = KF + kStagesK, SF = KE + kStagesK, PF = SF + 2, OF = PF + 2, OE, RS, NBAR };
constexpr uint32_t SM_MISC = SM_BAR + NBAR * 8;   // tmem base, abort flag
constexpr uint32_t kSmem = SM_MISC + 16 + 1024;
}  // namespace qm

template <int BS>
__global__ void __launch_bounds__(kThreadsTC, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
  using namespace qm;
  constexpr int kHalves = BS / 64;   // 64-key steps per block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int b) -> uint32_t { return sb + SM_BAR + 8u * b; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abortp = reinterpret_cast<volatile int*>(smem + SM_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + SM_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_unit = p.G * BS;
  const int64_t units = static_cast<int64_t>(p.B) * p.Hkv * p.nb;
  const int64_t items = units * p.tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar(QF), 1);
    mbar_init(bar(QE), 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(bar(KF + s), 1);
      mbar_init(bar(KE + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(SF + b), 1);
      mbar_init(bar(PF + b), 4);
    }
    mbar_init(bar(OF), 1);
    mbar_init(bar(OE), 4);
    mbar_init(bar(RS), 128);
    *abortp = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // [S | dP] x 2 buffers (64 + 64 columns each) | dQ
  auto item_unit = [&](int64_t item, int& tile, int64_t& bg, int& i) {
    const int64_t unit = item / p.tiles;
    tile = static_cast<int>(item % p.tiles);
    bg = unit / p.nb;
    i = p.nb - 1 - static_cast<int>(unit % p.nb);   // heavy (late) query blocks first
    return bg * p.nb + i;
  };

  if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int gs = 0, qc = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
        int tile, i;
        int64_t bg;
        const int64_t unit = item_unit(item, tile, bg, i);
        const int n = p.counts[unit];
        if (n == 0) continue;
        const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
        if (qc > 0 && !(ok = mbar_wait(bar(QE), (qc - 1) & 1, abortp, p.status))) break;
        uint32_t bytes = 0;
        for (int pc = 0; pc < 2; ++pc)
          if (tile * 128 + pc * 64 < rows_per_unit) bytes += 4 * 8192;
        mbar_arrive_expect_tx(bar(QF), bytes);
        for (int pc = 0; pc < 2; ++pc) {
          const int R0 = tile * 128 + pc * 64;
          if (R0 >= rows_per_unit) continue;
          const int h = g * p.G + R0 / BS;
          const int y = (b * p.Hq + h) * p.N + i * BS + R0 % BS;
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_2d(sb + SM_Q + hf * kHalf + pc * 8192, &tmQ, bar(QF), hf * 64, y);
            tma_load_2d(sb + SM_DO + hf * kHalf + pc * 8192, &tmDO, bar(QF), hf * 64, y);
          }
        }
        ++qc;
        const int* list = p.lists + unit * p.idx_stride;
        const int kvrow0 = static_cast<int>(bg) * p.N;
        const int nst = n * kHalves;
        for (int sw = 0; ok && sw < 2; ++sw)
          for (int s = 0; s < nst; ++s, ++gs) {
            const int st = gs % kStagesK, use = gs / kStagesK;
            if (gs >= kStagesK && !(ok = mbar_wait(bar(KE + st), (use - 1) & 1, abortp, p.status))) break;
            mbar_arrive_expect_tx(bar(KF + st), 4u * 8192u);
            const int y = kvrow0 + list[s / kHalves] * BS + (s % kHalves) * 64;
            for (int hf = 0; hf < 2; ++hf) {
              tma_load_2d(sb + SM_K + st * kKV + hf * kKVHalf, &tmK, bar(KF + st), hf * 64, y);
              tma_load_2d(sb + SM_V + st * kKV + hf * kKVHalf, &tmV, bar(KF + st), hf * 64, y);
            }
          }
      }
      if (*abortp) {
        if (qc > 0) mbar_drain(bar(QF), (qc - 1) & 1);
        for (int s = max(0, gs - kStagesK); s < gs; ++s) mbar_drain(bar(KF + s % kStagesK), (s / kStagesK) & 1);
      }
    }
  } else if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16_f32(128, 64, 0, 0);     // S, dP: 128 rows x 64 keys
      const uint32_t id_mn = idesc_bf16_f32(128, 128, 0, 1);   // dQ: 128 rows x 128 channels
      const uint64_t qd = smem_desc_sw128(sb + SM_Q, 16, 1024);
      const uint64_t dod = smem_desc_sw128(sb + SM_DO, 16, 1024);
      const uint64_t kd0 = smem_desc_sw128(sb + SM_K, 16, 1024);
      const uint64_t vd0 = smem_desc_sw128(sb + SM_V, 16, 1024);
      const uint64_t kmn0 = smem_desc_sw128(sb + SM_K, kKVHalf, 1024);
      const uint32_t tQ = tmem + 256;
      int gs = 0, qc = 0, done = 0;
      int pfu[2] = {0, 0};
      bool ok = true;
      // S = Q K^T and dP = dO V^T of global step `g` into buffer g & 1; in the
      // first sweep the K/V stage is free once they complete
      auto issue_sdp = [&](int g, bool release) -> bool {
        const int st = g % kStagesK, buf = g & 1;
        if (!mbar_wait(bar(KF + st), (g / kStagesK) & 1, abortp, p.status)) return false;
        tc_fence_after();
        const uint64_t kd = kd0 + ((st * kKV) >> 4), vd = vd0 + ((st * kKV) >> 4);
        const uint32_t tS = tmem + buf * 128, tP = tS + 64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
          mma_ss(tS, qd + oa, kd + ob, id_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
          mma_ss(tP, dod + oa, vd + ob, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(SF + buf));
        if (release) tc_commit(bar(KE + st));
        return true;
      };
      for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
        int tile, i;
        int64_t bg;
        const int64_t unit = item_unit(item, tile, bg, i);
        const int n = p.counts[unit];
        if (n == 0) continue;
        const int nst = n * kHalves;
        if (!(ok = mbar_wait(bar(QF), qc & 1, abortp, p.status))) break;
        ++qc;
        tc_fence_after();
        if (!(ok = issue_sdp(gs, true))) break;
        for (int x = 0; x < 2 * nst; ++x, ++gs) {
          const int sw = x / nst, s = x % nst;
          const int st = gs % kStagesK, buf = gs & 1;
          // the next step's products go out before this step's lanes are done
          if (x + 1 < 2 * nst && !(ok = issue_sdp(gs + 1, x + 1 < nst))) break;
          if (!(ok = mbar_wait(bar(PF + buf), pfu[buf] & 1, abortp, p.status))) break;
          ++pfu[buf];
          if (sw == 0) continue;
          // second sweep: dQ += dS K once the lanes have written dS over S
          if (s == 0 && done > 0 && !(ok = mbar_wait(bar(OE), (done - 1) & 1, abortp, p.status))) break;
          tc_fence_after();
          const uint64_t kmn = kmn0 + ((st * kKV) >> 4);
          const uint32_t tS = tmem + buf * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tQ, tS + kk * 8, kmn + ((kk * 2048) >> 4), id_mn, (s > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(KE + st));
        }
        if (!ok) break;
        tc_commit(bar(OF));
        tc_commit(bar(QE));
        ++done;
      }
      if (!ok) {
        // every MMA issued so far must finish before tensor memory is freed
        tc_commit(bar(OF));
        mbar_drain(bar(OF), done & 1);
      }
    }
  } else {
    // ------------------------------------------------ lanes (one row each)
    const int r = warp * 32 + lane;
    const uint32_t la = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t tQ = la + 256;
    const float scale2 = p.scale * kLog2e;
    int gs = 0, done = 0, rs = 0;
    int sfu[2] = {0, 0};
    bool ok = true;
    for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
      int tile, i;
      int64_t bg;
      const int64_t unit = item_unit(item, tile, bg, i);
      const int n = p.counts[unit];
      const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
      const int R = tile * 128 + r;
      const bool valid = R < rows_per_unit;
      const int h = g * p.G + (valid ? R / BS : 0);
      const int tb = R % BS;
      const int64_t row = (static_cast<int64_t>(b) * p.Hq + h) * p.N + static_cast<int64_t>(i) * BS + tb;
      if (n == 0) {
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.dq + row * kD);
          for (int c = 0; c < kD / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          p.D[row] = 0.0f;
        }
        continue;
      }
      const float lse = valid ? p.lse[row] : -INFINITY;
      const bool live = valid && lse > -INFINITY;
      const float lse2 = live ? lse * kLog2e : 0.0f;
      const int* list = p.lists + unit * p.idx_stride;
      const float* lg = p.logg + unit * p.idx_stride;
      const int nst = n * kHalves;
      float Dt = 0.0f, dl = 0.0f;
      // the next step's block and gate weight are read one step ahead
      int jj_next = list[0];
      float lg_next = lg[0];
      for (int x = 0; ok && x < 2 * nst; ++x, ++gs) {
        const int sw = x / nst, s = x % nst;
        const int slot = s / kHalves, half = s % kHalves;
        const int jj = jj_next;
        const float off = lg_next * kLog2e - lse2;
        if (x + 1 < 2 * nst) {
          const int slot1 = ((x + 1) % nst) / kHalves;
          jj_next = list[slot1];
          lg_next = lg[slot1];
        }
        const int buf = gs & 1;
        if (!(ok = warp_wait_all(bar(SF + buf), sfu[buf] & 1, abortp, p.status))) break;
        ++sfu[buf];
        tc_fence_after();
        const uint32_t tS = la + buf * 128, tP = tS + 64;
        // keys of this step this row may see: all 64, or (the diagonal block)
        // those not after the row, or none (a row that attends to nothing)
        const int lim_step = !live ? 0 : (jj == i ? min(64, max(0, tb - half * 64 + 1)) : 64);
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          uint32_t sv[32], dv[32];
          tmem_ld32(tS + part * 32, sv);
          tmem_ld32(tP + part * 32, dv);
          const int lim = min(32, max(0, lim_step - part * 32));
          if (sw == 0) {
            // D_t += sum of P dP over the part, four independent partial sums
            float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if (lim == 32) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                a[e & 3] = fmaf(fast_exp2(fmaf(__uint_as_float(sv[e]), scale2, off)), __uint_as_float(dv[e]), a[e & 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float pv = (e < lim) ? fast_exp2(fmaf(__uint_as_float(sv[e]), scale2, off)) : 0.0f;
                a[e & 3] = fmaf(pv, __uint_as_float(dv[e]), a[e & 3]);
              }
            }
            Dt += (a[0] + a[1]) + (a[2] + a[3]);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float de[2];
#pragma unroll
              for (int y = 0; y < 2; ++y) {
                const float pv = fast_exp2(fmaf(__uint_as_float(sv[e + y]), scale2, off));
                de[y] = (e + y < lim) ? pv * (__uint_as_float(dv[e + y]) - Dt) : 0.0f;
              }
              pk[e >> 1] = pack_bf16x2(de[0], de[1]);
              dl += de[0] + de[1];
            }
            tmem_st16(tS + part * 16, pk);
          }
        }
        if (sw == 1) {
          tmem_wait_st();
          if (half == kHalves - 1) {
            // the rows' share of dlogg for this block, per warp
#pragma unroll
            for (int o = 16; o; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
            if (lane == 0) red[warp * kMaxList + slot] = dl;
            dl = 0.0f;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(PF + buf));
        if (sw == 0 && s == nst - 1 && valid) p.D[row] = Dt;
      }
      if (!ok) break;
      if (!(ok = warp_wait_all(bar(OF), done & 1, abortp, p.status))) break;
      ++done;
      tc_fence_after();
      float* dst = p.dq + row * kD;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        tmem_ld32(tQ + ch * 32, v);
        if (valid) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + ch * 32 + c) =
                make_float4(__uint_as_float(v[c]) * p.scale, __uint_as_float(v[c + 1]) * p.scale,
                            __uint_as_float(v[c + 2]) * p.scale, __uint_as_float(v[c + 3]) * p.scale);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(OE));
      // this tile's dlogg partial per kept slot: the four warps' sums in
      // order.  (A warp writes the next item's sums only after every warp has
      // passed this point: its S waits on all four warps' earlier P arrivals.)
      mbar_arrive(bar(RS));
      if (!(ok = warp_wait_all(bar(RS), rs & 1, abortp, p.status))) break;
      ++rs;
      for (int x = r; x < n; x += 128)
        p.dlogg_part[(unit * p.idx_stride + x) * p.tiles + tile] =
            ((red[x] + red[kMaxList + x]) + red[2 * kMaxList + x]) + red[3 * kMaxList + x];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ key-major
// Chunks of 64 query rows; two S^T | dP^T buffers in tensor memory, so the
// MMAs of chunk c+1 run while the lanes turn chunk c into P^T and dS^T.
namespace km {
constexpr int kStagesC = 4;                                   // Q/dO chunk stages
constexpr uint32_t kChunk = 64u * 128u * 2u;                  // 64 rows x 128 bf16
constexpr uint32_t kChunkHalf = kChunk / 2;                   // 64 rows x 64 bf16
constexpr uint32_t SM_K = 0, SM_V = kTile;
constexpr uint32_t SM_Q = 2 * kTile, SM_DO = SM_Q + kStagesC * kChunk;
constexpr uint32_t SM_ROW = SM_DO + kStagesC * kChunk;        // float [2 slots][2 arrays][64]
constexpr uint32_t SM_BAR = SM_ROW + 2 * 2 * 64 * 4;
enum { KVF = 0, KVE, CF, CE = CF + kStagesC, SF = CE + kStagesC, PF = SF + 2, OF = PF + 2, OE, RS, NBAR };
constexpr uint32_t SM_MISC = SM_BAR + NBAR * 8;
constexpr uint32_t kSmem = SM_MISC + 16 + 1024;
}  // namespace km

template <int BS>
__global__ void __launch_bounds__(kThreadsTC, 1)
    dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
  using namespace km;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int b) -> uint32_t { return sb + SM_BAR + 8u * b; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abortp = reinterpret_cast<volatile int*>(smem + SM_MISC + 4);
  float* rowc = reinterpret_cast<float*>(smem + SM_ROW);   // [2][64] log2 offsets (logg - lse) * log2e
  float* rowd = rowc + 2 * 64;                             // [2][64] D
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 64-row chunks per (query block, key block): one head each (bs 64), or
  // the two halves of each head's 128 rows (bs 128)
  const int cpe = (BS == 128) ? 2 * p.G : p.G;
  const int64_t items = static_cast<int64_t>(p.B) * p.Hkv * p.nb;

  // the upper 64 keys of a 64-token block are never loaded: zero them (and
  // the rest of the K/V tiles) once, before the first copy lands
  if (warp < 4) {
    uint4* z = reinterpret_cast<uint4*>(smem);
    for (uint32_t x = threadIdx.x; x < 2 * kTile / 16; x += 128) z[x] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    mbar_init(bar(KVF), 1);
    mbar_init(bar(KVE), 1);
    for (int s = 0; s < kStagesC; ++s) {
      mbar_init(bar(CF + s), 1);
      mbar_init(bar(CE + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(SF + b), 1);
      mbar_init(bar(PF + b), 4);
    }
    mbar_init(bar(OF), 1);
    mbar_init(bar(OE), 4);
    mbar_init(bar(RS), 128);
    *abortp = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // [S^T | dP^T] x 2 buffers (64 + 64 columns each) | dV | dK

  if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int gc = 0, kvc = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const int64_t bg = item / p.nb;
        const int j = static_cast<int>(item % p.nb);
        const int* off = p.toff + bg * (p.nb + 1);
        const int e0 = off[j], ne = off[j + 1] - e0;
        if (ne == 0) continue;
        const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
        const int2* tl = p.tlist + bg * static_cast<int64_t>(p.nb) * p.idx_stride + e0;
        if (kvc > 0 && !(ok = mbar_wait(bar(KVE), (kvc - 1) & 1, abortp, p.status))) break;
        mbar_arrive_expect_tx(bar(KVF), static_cast<uint32_t>(BS) * 512u);
        for (int r = 0; r < BS / 64; ++r) {
          const int y = static_cast<int>(bg) * p.N + j * BS + r * 64;
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_2d(sb + SM_K + hf * kHalf + r * 8192, &tmK, bar(KVF), hf * 64, y);
            tma_load_2d(sb + SM_V + hf * kHalf + r * 8192, &tmV, bar(KVF), hf * 64, y);
          }
        }
        ++kvc;
        for (int c = 0; ok && c < ne * cpe; ++c, ++gc) {
          const int st = gc % kStagesC, use = gc / kStagesC;
          const int i = tl[c / cpe].x, hc = c % cpe;
          const int hh = (BS == 128) ? hc >> 1 : hc;
          const int r0 = (BS == 128) ? (hc & 1) * 64 : 0;
          if (gc >= kStagesC && !(ok = mbar_wait(bar(CE + st), (use - 1) & 1, abortp, p.status))) break;
          mbar_arrive_expect_tx(bar(CF + st), 4u * 8192u);
          const int y = (b * p.Hq + g * p.G + hh) * p.N + i * BS + r0;
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_2d(sb + SM_Q + st * kChunk + hf * kChunkHalf, &tmQ, bar(CF + st), hf * 64, y);
            tma_load_2d(sb + SM_DO + st * kChunk + hf * kChunkHalf, &tmDO, bar(CF + st), hf * 64, y);
          }
        }
      }
      if (*abortp) {
        if (kvc > 0) mbar_drain(bar(KVF), (kvc - 1) & 1);
        for (int s = max(0, gc - kStagesC); s < gc; ++s) mbar_drain(bar(CF + s % kStagesC), (s / kStagesC) & 1);
      }
    }
  } else if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16_f32(128, 64, 0, 0);     // S^T, dP^T: 128 keys x 64 rows
      const uint32_t id_mn = idesc_bf16_f32(128, 128, 0, 1);   // dV, dK: 128 keys x 128 channels
      const uint64_t kd = smem_desc_sw128(sb + SM_K, 16, 1024);
      const uint64_t vd = smem_desc_sw128(sb + SM_V, 16, 1024);
      const uint64_t qd0 = smem_desc_sw128(sb + SM_Q, 16, 1024);
      const uint64_t dod0 = smem_desc_sw128(sb + SM_DO, 16, 1024);
      const uint64_t qmn0 = smem_desc_sw128(sb + SM_Q, kChunkHalf, 1024);
      const uint64_t domn0 = smem_desc_sw128(sb + SM_DO, kChunkHalf, 1024);
      const uint32_t tV = tmem + 256, tK = tmem + 384;
      int gc = 0, kvc = 0, done = 0;
      int pfu[2] = {0, 0};   // P-ready phases consumed per buffer
      bool ok = true;
      // S^T = K Q^T and dP^T = V dO^T of chunk number `cg` into buffer cg & 1
      auto issue_sdp = [&](int cg) -> bool {
        const int st = cg % kStagesC, buf = cg & 1;
        if (!mbar_wait(bar(CF + st), (cg / kStagesC) & 1, abortp, p.status)) return false;
        tc_fence_after();
        const uint64_t qd = qd0 + ((st * kChunk) >> 4), dod = dod0 + ((st * kChunk) >> 4);
        const uint32_t tS = tmem + buf * 128, tP = tS + 64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * kChunkHalf + (kk & 3) * 32) >> 4;
          mma_ss(tS, kd + oa, qd + ob, id_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * kChunkHalf + (kk & 3) * 32) >> 4;
          mma_ss(tP, vd + oa, dod + ob, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(SF + buf));
        return true;
      };
      for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const int64_t bg = item / p.nb;
        const int j = static_cast<int>(item % p.nb);
        const int* off = p.toff + bg * (p.nb + 1);
        const int nch = (off[j + 1] - off[j]) * cpe;
        if (nch == 0) continue;
        if (!(ok = mbar_wait(bar(KVF), kvc & 1, abortp, p.status))) break;
        ++kvc;
        if (!(ok = issue_sdp(gc))) break;
        for (int c = 0; c < nch; ++c, ++gc) {
          const int st = gc % kStagesC, buf = gc & 1;
          // the next chunk's products go out before this chunk's lanes are done
          if (c + 1 < nch && !(ok = issue_sdp(gc + 1))) break;
          if (!(ok = mbar_wait(bar(PF + buf), pfu[buf] & 1, abortp, p.status))) break;
          ++pfu[buf];
          if (c == 0 && done > 0 && !(ok = mbar_wait(bar(OE), (done - 1) & 1, abortp, p.status))) break;
          tc_fence_after();
          const uint32_t tS = tmem + buf * 128, tP = tS + 64;
          const uint64_t qmn = qmn0 + ((st * kChunk) >> 4), domn = domn0 + ((st * kChunk) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tV, tS + kk * 8, domn + ((kk * 2048) >> 4), id_mn, (c > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tK, tP + kk * 8, qmn + ((kk * 2048) >> 4), id_mn, (c > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(CE + st));
        }
        if (!ok) break;
        tc_commit(bar(OF));
        tc_commit(bar(KVE));
        ++done;
      }
      if (!ok) {
        tc_commit(bar(OF));
        mbar_drain(bar(OF), done & 1);
      }
    }
  } else {
    // ------------------------------------------------ lanes (one key each)
    const int u = warp * 32 + lane;
    const uint32_t la = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t tV = la + 256, tK = la + 384;
    const float scale2 = p.scale * kLog2e;
    const bool kvalid = (BS == 128) || u < 64;
    int gc = 0, done = 0;
    int sfu[2] = {0, 0};
    bool ok = true;
    for (int64_t item = blockIdx.x; ok && item < items; item += gridDim.x) {
      const int64_t bg = item / p.nb;
      const int j = static_cast<int>(item % p.nb);
      const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
      const int* off = p.toff + bg * (p.nb + 1);
      const int e0 = off[j], ne = off[j + 1] - e0;
      const int64_t krow = bg * static_cast<int64_t>(p.N) + static_cast<int64_t>(j) * BS + u;
      if (ne == 0) {
        if (kvalid) {
          float4* dk = reinterpret_cast<float4*>(p.dk + krow * kD);
          float4* dv = reinterpret_cast<float4*>(p.dv + krow * kD);
          for (int c = 0; c < kD / 4; ++c) dk[c] = dv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      const int2* tl = p.tlist + bg * static_cast<int64_t>(p.nb) * p.idx_stride + e0;
      // a chunk's 64 rows: log2 offset (logg - LSE) * log2e, or -inf for a
      // row that attends to nothing (its P is then exactly 0); and D.  Lane
      // u < 64 reads row u of the next chunk while this one is processed.
      auto row_data = [&](int c, float& cv, float& dvv, int2& ent) {
        cv = -INFINITY;
        dvv = 0.0f;
        if (c >= ne * cpe) return;
        ent = tl[c / cpe];
        if (u >= 64) return;
        const int hc = c % cpe;
        const int hh = (BS == 128) ? hc >> 1 : hc;
        const int r0 = (BS == 128) ? (hc & 1) * 64 : 0;
        const int64_t row =
            (static_cast<int64_t>(b) * p.Hq + g * p.G + hh) * p.N + static_cast<int64_t>(ent.x) * BS + r0 + u;
        const float lse = p.lse[row];
        if (lse > -INFINITY) {
          cv = (p.logg[(bg * p.nb + ent.x) * p.idx_stride + ent.y] - lse) * kLog2e;
          dvv = p.D[row];
        }
      };
      float cv_next, dv_next;
      int2 ent_next = make_int2(0, 0);
      row_data(0, cv_next, dv_next, ent_next);
      for (int c = 0; c < ne * cpe; ++c, ++gc) {
        const int i = ent_next.x, hc = c % cpe;
        const int r0 = (BS == 128) ? (hc & 1) * 64 : 0;   // first row of the chunk inside query block i
        if (u < 64) {
          rowc[(gc & 1) * 64 + u] = cv_next;
          rowd[(gc & 1) * 64 + u] = dv_next;
        }
        // (the other slot may still be read for the previous chunk: a thread
        // writes it again only after every thread has arrived for that chunk)
        mbar_arrive(bar(RS));
        row_data(c + 1, cv_next, dv_next, ent_next);
        if (!(ok = warp_wait_all(bar(RS), gc & 1, abortp, p.status))) break;
        const int buf = gc & 1;
        if (!(ok = warp_wait_all(bar(SF + buf), sfu[buf] & 1, abortp, p.status))) break;
        ++sfu[buf];
        tc_fence_after();
        const float4* rc4 = reinterpret_cast<const float4*>(rowc + (gc & 1) * 64);
        const float4* rd4 = reinterpret_cast<const float4*>(rowd + (gc & 1) * 64);
        // columns (rows of the chunk) this key may not see: all when the key
        // does not exist, those before the key's position on the diagonal
        const int tmin = !kvalid ? 64 : (i == j ? min(64, max(0, u - r0)) : 0);
        const uint32_t tS = la + buf * 128, tP = tS + 64;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
          uint32_t sv[32], dv[32];
          tmem_ld32(tS + part * 32, sv);
          tmem_ld32(tP + part * 32, dv);
          const int m = min(32, max(0, tmin - part * 32));
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 c4 = rc4[part * 8 + e4], d4 = rd4[part * 8 + e4];
            const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
            float pe[4], de[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const int e = e4 * 4 + y;
              const float pv = (e >= m) ? fast_exp2(fmaf(__uint_as_float(sv[e]), scale2, cc[y])) : 0.0f;
              pe[y] = pv;
              de[y] = pv * (__uint_as_float(dv[e]) - dd[y]);
            }
            pk[e4 * 2] = pack_bf16x2(pe[0], pe[1]);
            pk[e4 * 2 + 1] = pack_bf16x2(pe[2], pe[3]);
            dk[e4 * 2] = pack_bf16x2(de[0], de[1]);
            dk[e4 * 2 + 1] = pack_bf16x2(de[2], de[3]);
          }
          tmem_st16(tS + part * 16, pk);
          tmem_st16(tP + part * 16, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(PF + buf));
      }
      if (!ok) break;
      if (!(ok = warp_wait_all(bar(OF), done & 1, abortp, p.status))) break;
      ++done;
      tc_fence_after();
      float* dkd = p.dk + krow * kD;
      float* dvd = p.dv + krow * kD;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t a[32], v[32];
        tmem_ld32(tK + ch * 32, a);
        tmem_ld32(tV + ch * 32, v);
        if (kvalid) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            *reinterpret_cast<float4*>(dkd + ch * 32 + c) =
                make_float4(__uint_as_float(a[c]) * p.scale, __uint_as_float(a[c + 1]) * p.scale,
                            __uint_as_float(a[c + 2]) * p.scale, __uint_as_float(a[c + 3]) * p.scale);
            *reinterpret_cast<float4*>(dvd + ch * 32 + c) =
                make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2]),
                            __uint_as_float(v[c + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(OE));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dsel per unit: dlogg_l (the row tiles' partials summed in order) minus
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
    for (int c = 0; c < p.tiles; ++c) x += p.dlogg_part[(unit * p.idx_stride + s) * p.tiles + c];
    tot += x;
  }
  for (int off = 16; off; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
  for (int s = lane; s < count; s += 32) {
    float x = 0.0f;
    for (int c = 0; c < p.tiles; ++c) x += p.dlogg_part[(unit * p.idx_stride + s) * p.tiles + c];
    row[list[s]] = x - __expf(p.logg[unit * p.idx_stride + s]) * tot;
  }
}

}  // namespace bwd

size_t attn_bwd_workspace(int B, int Hq, int Hkv, int N, int bs, int idx_stride) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int nb = N / bs;
  const int64_t units = static_cast<int64_t>(B) * Hkv * nb;
  const int tiles = (Hq / Hkv * bs + 127) / 128;
  size_t off = 0;
  off = a256(off + static_cast<size_t>(B) * Hq * N * sizeof(float));            // D (written by the dQ pass)
  off = a256(off + units * idx_stride * sizeof(float));                          // logg
  off = a256(off + units * idx_stride * sizeof(int));                            // lists
  off = a256(off + units * sizeof(int));                                         // counts
  off = a256(off + static_cast<size_t>(B) * Hkv * (nb + 1) * sizeof(int));       // toff
  off = a256(off + units * idx_stride * sizeof(int2));                           // tlist
  off = a256(off + units * idx_stride * tiles * sizeof(float));                  // dlogg partials
  return off;
}

cudaError_t launch_attn_bwd(const CUtensorMap* tmQ, const CUtensorMap* tmDO, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const float* lse, const int* idx, int idx_stride,
                            const float* sel, float scale, int B, int Hq, int Hkv, int N, int bs, float* dq,
                            float* dk, float* dv, float* dsel, void* workspace, uint32_t* status, int num_sms,
                            cudaStream_t st) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int nb = N / bs;
  const int64_t units = static_cast<int64_t>(B) * Hkv * nb;
  const int64_t rows = static_cast<int64_t>(B) * Hq * N;
  bwd::Params p;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.nb = nb;
  p.G = Hq / Hkv;
  p.idx_stride = idx_stride;
  p.tiles = (p.G * bs + 127) / 128;
  p.scale = scale;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = status;
  char* ws = static_cast<char*>(workspace);
  size_t off = 0;
  p.D = reinterpret_cast<float*>(ws + off);
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
  p.logg = logg;
  p.lists = lists;
  p.counts = counts;
  p.toff = toff;
  p.tlist = tlist;
  bwd::gate_kernel<<<static_cast<unsigned>((units + 7) / 8), 256, 0, st>>>(idx, idx_stride, sel, nb, units, lists,
                                                                           counts, logg, status);
  const int bgs = B * Hkv;
  const size_t tr_smem = bwd::transpose_smem_bytes(nb, idx_stride);
  cudaError_t e = ensure_dynamic_smem<bwd::transpose_kernel>(tr_smem);
  if (e != cudaSuccess) return e;
  bwd::transpose_kernel<<<bgs, bwd::kTrThreads, tr_smem, st>>>(lists, counts, idx_stride, nb, toff, tlist);
  const int64_t items_q = units * p.tiles, items_k = static_cast<int64_t>(bgs) * nb;
  const unsigned grid_q = static_cast<unsigned>(items_q < num_sms ? items_q : num_sms);
  const unsigned grid_k = static_cast<unsigned>(items_k < num_sms ? items_k : num_sms);
  if (bs == 64) {
    e = ensure_dynamic_smem<bwd::dq_tc_kernel<64>>(bwd::qm::kSmem);
    if (e == cudaSuccess) e = ensure_dynamic_smem<bwd::dkv_tc_kernel<64>>(bwd::km::kSmem);
    if (e != cudaSuccess) return e;
    if (grid_q > 0) bwd::dq_tc_kernel<64><<<grid_q, bwd::kThreadsTC, bwd::qm::kSmem, st>>>(*tmQ, *tmDO, *tmK, *tmV, p);
    if (grid_k > 0) bwd::dkv_tc_kernel<64><<<grid_k, bwd::kThreadsTC, bwd::km::kSmem, st>>>(*tmQ, *tmDO, *tmK, *tmV, p);
  } else {
    e = ensure_dynamic_smem<bwd::dq_tc_kernel<128>>(bwd::qm::kSmem);
    if (e == cudaSuccess) e = ensure_dynamic_smem<bwd::dkv_tc_kernel<128>>(bwd::km::kSmem);
    if (e != cudaSuccess) return e;
    if (grid_q > 0) bwd::dq_tc_kernel<128><<<grid_q, bwd::kThreadsTC, bwd::qm::kSmem, st>>>(*tmQ, *tmDO, *tmK, *tmV, p);
    if (grid_k > 0) bwd::dkv_tc_kernel<128><<<grid_k, bwd::kThreadsTC, bwd::km::kSmem, st>>>(*tmQ, *tmDO, *tmK, *tmV, p);
  }
  if (dsel != nullptr)
    bwd::dsel_kernel<<<static_cast<unsigned>((units + 7) / 8), 256, 0, st>>>(p, units, dsel);
  return cudaGetLastError();
}

}  // namespace bsa
