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
// blocks (decode) or the union of their expanded chunks (gist), so one CTA
// gathers each 64-token tile once for the whole group: the G query rows form
// the M dimension of the MMA (rows >= G are padding and never read back).
// The tile list of a group is split across `nsplit` CTAs (split-K); each CTA
// writes an unnormalised partial (running max m, sum l, O row) per head and a
// second kernel merges them.
//
// Roles (128 threads): warp 0 softmax (TMEM lanes 0-31 = query rows),
// warp 1 TMA producer, warp 2 TMEM owner + MMA issuer, warp 3 list loader.
// Tensor memory: S buffers A and B (128 columns each, double-buffered so the
// next S = Q K^T runs while the softmax works) and O (128 columns).
#include "common.cuh"
#include "kernels.h"

namespace bsa {
namespace decode {

constexpr int kD = 128;
constexpr int kThreads = 128;
constexpr int kStages = 2;
constexpr int kMaxTiles = 1024;        // tiles one CTA may own
constexpr uint32_t kHalfBytes = 128u * 128u;
constexpr uint32_t kTileBytes = 2u * kHalfBytes;     // 128 rows x 128 bf16
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kTileBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kTileBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kTileBytes;

enum {
  BAR_Q = 0,
  BAR_KF = 1,
  BAR_KE = BAR_KF + kStages,
  BAR_VF = BAR_KE + kStages,
  BAR_VE = BAR_VF + kStages,
  BAR_SF = BAR_VE + kStages,   // two S buffers
  BAR_PF = BAR_SF + 2,
  BAR_OD = BAR_PF + 1,         // one completion per O += P V
  BAR_OF = BAR_OD + 1,
  BAR_AB = BAR_OF + 1,
  NUM_BARS = BAR_AB + 1
};

struct Misc {
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles;
  int pad;
  int tiles[kMaxTiles];
};
constexpr uint32_t kSmemMisc = kSmemBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kSmemMisc + sizeof(Misc) + 1024;

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
  int nsplit;
  float scale_log2;
  float* partial;
  uint32_t* status;
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* ab, uint32_t* st) {
  bool ok = mbar_wait(bar, parity, ab, st);
  return __all_sync(0xffffffffu, ok);
}

// Key-column mask word of a 64-key tile for one head (bit e = key e allowed).
__device__ __forceinline__ uint64_t tile_mask(int tile, const uint32_t* bits) {
  if (bits == nullptr) return ~0ull;                       // plain decode: every key
  if (tile >= 0) return ((bits[tile >> 5] >> (tile & 31)) & 1u) ? ~0ull : 0ull;   // expanded chunk
  const int gb = -(tile + 1);                              // gist block: gists not expanded
  const uint64_t w = static_cast<uint64_t>(bits[2 * gb]) | (static_cast<uint64_t>(bits[2 * gb + 1]) << 32);
  return ~w;
}

template <int KEYS>
__device__ __forceinline__ void softmax_step(uint32_t t_s, uint32_t t_o, float scale_log2, uint64_t mask0,
                                             uint64_t mask1, int s, uint32_t bar_od, volatile int* ab,
                                             uint32_t* st, float& m_run, float& l_run, bool& ok) {
  float mx = -INFINITY;
#pragma unroll
  for (int ch = 0; ch < KEYS / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(t_s + ch * 32, v);
    const uint64_t mk = (ch < 2) ? mask0 : mask1;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int bit = (ch & 1) * 32 + e;
      float x = __uint_as_float(v[e]) * scale_log2;
      if (!((mk >> bit) & 1ull)) x = -INFINITY;
      mx = fmaxf(mx, x);
    }
  }
  const float m_new = fmaxf(m_run, mx);
  const bool need = m_new > m_run + kRescaleThreshold;
  const float m_use = need ? m_new : m_run;
  const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
  const float alpha = need ? fast_exp2(m_run - m_use) : 1.0f;
  if (s > 0 && __any_sync(0xffffffffu, need)) {
    // the previous O += P V must be complete before O is rescaled
    if (!warp_wait(bar_od, (s - 1) & 1, ab, st)) {
      ok = false;
      return;
    }
    tc_fence_after();
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
  float sum = 0.0f;
#pragma unroll
  for (int ch = 0; ch < KEYS / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(t_s + ch * 32, v);
    const uint64_t mk = (ch < 2) ? mask0 : mask1;
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float p2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int bit = (ch & 1) * 32 + 2 * e + h;
        float x = __uint_as_float(v[2 * e + h]) * scale_log2;
        if (!((mk >> bit) & 1ull)) x = -INFINITY;
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

__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmGK,
                       const __grid_constant__ CUtensorMap tmGV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + kSmemMisc);
  auto bar = [&](int b) -> uint32_t { return sbase + kSmemBar + 8u * b; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  volatile int* abortp = &misc->abort_flag;
  const bool gist = p.expanded != nullptr;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KF + s), 1);
      mbar_init(bar(BAR_KE + s), 1);
      mbar_init(bar(BAR_VF + s), 1);
      mbar_init(bar(BAR_VE + s), 1);
    }
    mbar_init(bar(BAR_SF + 0), 1);
    mbar_init(bar(BAR_SF + 1), 1);
    mbar_init(bar(BAR_PF), 32);
    mbar_init(bar(BAR_OD), 1);
    mbar_init(bar(BAR_OF), 1);
    mbar_init(bar(BAR_AB), 1);
    misc->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (gist) {
      prefetch_tmap(&tmGK);
      prefetch_tmap(&tmGV);
    }
  }
  if (warp == 2) {
    tmem_alloc(sbase + kSmemMisc + offsetof(Misc, tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // this CTA's slice of the group's tile list
    const int* src = p.list + static_cast<int64_t>(bg) * p.list_stride;
    int total;
    if (p.list_has_count) {
      total = src[0];
      src += 1;
    } else {
      total = 0;
      for (int base = 0; base < p.list_stride; base += 32) {
        const int t = base + lane;
        const int v = (t < p.list_stride) ? src[t] : -1;
        const unsigned neg = __ballot_sync(0xffffffffu, v < 0);
        total += neg ? __ffs(neg) - 1 : 32;
        if (neg) break;
      }
    }
    const int per = (total + p.nsplit - 1) / p.nsplit;
    const int t0 = min(total, split * per), t1 = min(total, t0 + per);
    int cnt = t1 - t0;
    if (cnt > kMaxTiles) {
      if (lane == 0) atomicOr(p.status, BSA_DEV_BAD_SHAPE);
      cnt = kMaxTiles;
    }
    const int nb_cache = p.Nk / 64;
    const int ngist = p.nc / 64;
    for (int t = lane; t < cnt; t += 32) {
      int v = src[t0 + t];
      const bool bad = gist ? (v >= nb_cache || v < -ngist) : (v < 0 || v >= nb_cache);
      if (bad) {
        atomicOr(p.status, BSA_DEV_BAD_INDEX);
        v = 0x7fffffff;   // marks a skipped tile
      }
      misc->tiles[t] = v;
    }
    __syncwarp();
    if (lane == 0) {
      // drop skipped tiles, keeping order
      int w = 0;
      for (int t = 0; t < cnt; ++t)
        if (misc->tiles[t] != 0x7fffffff) misc->tiles[w++] = misc->tiles[t];
      misc->n_tiles = w;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = misc->tmem_base;
  const int n = misc->n_tiles;
  const int nsteps = (n + 1) / 2;

  if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------ TMA producer
      mbar_arrive_expect_tx(bar(BAR_Q), static_cast<uint32_t>(p.G) * 256u);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_2d(sbase + kSmemQ + hf * kHalfBytes, &tmQ, bar(BAR_Q), hf * 64, b * p.Hq + g * p.G);
      int k_issued = 0, v_issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const int slot = s % kStages, use = s / kStages;
        const int nt = (2 * s + 1 < n) ? 2 : 1;
        const uint32_t bytes = static_cast<uint32_t>(nt) * 64u * 256u;
        for (int kv = 0; kv < 2; ++kv) {
          const int full = kv ? BAR_VF : BAR_KF, empty = kv ? BAR_VE : BAR_KE;
          const uint32_t dst0 = sbase + (kv ? kSmemV : kSmemK) + slot * kTileBytes;
          if (s >= kStages && !mbar_wait(bar(empty + slot), (use - 1) & 1, abortp, p.status)) break;
          mbar_arrive_expect_tx(bar(full + slot), bytes);
          for (int tt = 0; tt < nt; ++tt) {
            const int tile = misc->tiles[2 * s + tt];
            const CUtensorMap* map;
            int y;
            if (tile >= 0) {
              map = kv ? &tmV : &tmK;
              y = bg * p.Nk + tile * 64;
            } else {
              map = kv ? &tmGV : &tmGK;
              y = bg * p.nc + (-(tile + 1)) * 64;
            }
            for (int hf = 0; hf < 2; ++hf)
              tma_load_2d(dst0 + hf * kHalfBytes + tt * 8192u, map, bar(full + slot), hf * 64, y);
          }
          if (kv) ++v_issued; else ++k_issued;
        }
        if (*abortp) break;
      }
      if (*abortp) {
        mbar_drain(bar(BAR_Q), 0);
        for (int s = max(0, k_issued - kStages); s < k_issued; ++s) mbar_drain(bar(BAR_KF + s % kStages), (s / kStages) & 1);
        for (int s = max(0, v_issued - kStages); s < v_issued; ++s) mbar_drain(bar(BAR_VF + s % kStages), (s / kStages) & 1);
      }
    }
  } else if (warp == 2) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t id_s128 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s64 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, 0, 1);
      auto keys_of = [&](int s) -> int { return (2 * s + 1 < n) ? 128 : 64; };
      auto issue_s = [&](int s) {
        const int slot = s % kStages;
        const uint32_t ka = sbase + kSmemK + slot * kTileBytes;
        const uint32_t qa = sbase + kSmemQ;
        const uint32_t id = keys_of(s) == 128 ? id_s128 : id_s64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(tmem + (s & 1) * 128, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), id,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(BAR_SF + (s & 1)));
        tc_commit(bar(BAR_KE + slot));
      };
      bool ok = mbar_wait(bar(BAR_Q), 0, abortp, p.status) &&
                mbar_wait(bar(BAR_KF + 0), 0, abortp, p.status);
      tc_fence_after();
      if (ok) issue_s(0);
      for (int s = 0; ok && s < nsteps; ++s) {
        if (s + 1 < nsteps) {
          const int s1 = s + 1;
          if (!(ok = mbar_wait(bar(BAR_KF + s1 % kStages), (s1 / kStages) & 1, abortp, p.status))) break;
          tc_fence_after();
          issue_s(s1);
        }
        const int slot = s % kStages;
        if (!(ok = mbar_wait(bar(BAR_PF), s & 1, abortp, p.status))) break;
        if (!(ok = mbar_wait(bar(BAR_VF + slot), (s / kStages) & 1, abortp, p.status))) break;
        tc_fence_after();
        const uint32_t va = sbase + kSmemV + slot * kTileBytes;
        const int keys = keys_of(s);
        for (int kk = 0; kk < keys / 16; ++kk)
          mma_ts(tmem + 256, tmem + (s & 1) * 128 + kk * 8, smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), id_pv,
                 (s > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(BAR_OD));
        tc_commit(bar(BAR_VE + slot));
      }
      if (ok) tc_commit(bar(BAR_OF));
      if (!ok) {
        tc_commit(bar(BAR_AB));
        mbar_drain(bar(BAR_AB), 0);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------ softmax + partial out
    const int r = lane;                      // query row = head g*G + r
    const bool valid = r < p.G;
    const int h = g * p.G + (valid ? r : 0);
    const uint32_t* bits = gist ? p.expanded + (static_cast<int64_t>(b) * p.Hq + h) * (p.nc / 32) : nullptr;
    const uint32_t t_o = tmem + 256;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      if (!(ok = warp_wait(bar(BAR_SF + (s & 1)), (s >> 1) & 1, abortp, p.status))) break;
      tc_fence_after();
      const int tA = misc->tiles[2 * s];
      const uint64_t mA = tile_mask(tA, bits);
      const uint32_t t_s = tmem + (s & 1) * 128;
      if (2 * s + 1 < n) {
        const uint64_t mB = tile_mask(misc->tiles[2 * s + 1], bits);
        softmax_step<128>(t_s, t_o, p.scale_log2, mA, mB, s, bar(BAR_OD), abortp, p.status, m_run, l_run, ok);
      } else {
        softmax_step<64>(t_s, t_o, p.scale_log2, mA, 0ull, s, bar(BAR_OD), abortp, p.status, m_run, l_run, ok);
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(bar(BAR_PF));
    }
    float* part = p.partial + ((static_cast<int64_t>(bg) * p.G + r) * p.nsplit + split) * kRec;
    if (n == 0) {
      if (valid) {
        part[0] = -INFINITY;
        part[1] = 0.0f;
        for (int c = 0; c < kD; ++c) part[4 + c] = 0.0f;
      }
    } else if (ok && warp_wait(bar(BAR_OF), 0, abortp, p.status)) {
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < kD / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(t_o + ch * 32, v);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(part + 4 + ch * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      if (valid) {
        part[0] = m_run;
        part[1] = l_run;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the split partials of one row (one warp per row).
__global__ void combine_kernel(const float* __restrict__ partial, int rows, int nsplit, int d, int out_bf16,
                               void* __restrict__ o, float* __restrict__ lse) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int rec = d + 4;
  const float* pr = partial + static_cast<int64_t>(row) * nsplit * rec;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, pr[s * rec]);
  float L = 0.0f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < nsplit; ++s) {
    const float ms = pr[s * rec];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    L += w * pr[s * rec + 1];
    for (int e = 0; e < 4; ++e) {
      const int c = lane + 32 * e;
      if (c < d) acc[e] += w * pr[s * rec + 4 + c];
    }
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
// union of expanded chunks followed by every gist block (-(gb+1)).
__global__ void gist_union_kernel(const int* __restrict__ idx, int Hq, int Hkv, int topk, int idx_stride, int nc,
                                  uint32_t* __restrict__ expanded, int* __restrict__ union_list, int union_stride,
                                  uint32_t* __restrict__ status) {
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
    const int ngb = nc / 64;
    for (int t = lane; t < ngb; t += 32) out[1 + run + t] = -(t + 1);
    if (lane == 0) out[0] = run + ngb;
  }
}

}  // namespace decode

cudaError_t launch_attn_decode_bf16(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                    const CUtensorMap* tmGK, const CUtensorMap* tmGV, const DecodeArgs& a,
                                    cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode::attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(decode::kSmemBytes));
    if (e != cudaSuccess) return e;
    configured = true;
  }
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
  p.nsplit = a.nsplit;
  p.scale_log2 = a.softmax_scale * decode::kLog2e;
  p.partial = a.partial;
  p.status = a.status;
  dim3 grid(a.nsplit, a.B * a.Hkv);
  decode::attn_decode_kernel<<<grid, decode::kThreads, decode::kSmemBytes, st>>>(
      *tmQ, *tmK, *tmV, tmGK ? *tmGK : *tmK, tmGV ? *tmGV : *tmV, p);
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const float* partial, int rows, int nsplit, int d, bool out_bf16, void* o,
                                  float* lse, cudaStream_t st) {
  const int warps = 8;
  decode::combine_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, st>>>(partial, rows, nsplit, d,
                                                                             out_bf16 ? 1 : 0, o, lse);
  return cudaGetLastError();
}

cudaError_t launch_gist_union(const int* idx, int B, int Hq, int Hkv, int topk, int idx_stride, int nc,
                              uint32_t* expanded, int* union_list, int union_stride, uint32_t* status,
                              cudaStream_t st) {
  const int G = Hq / Hkv;
  const size_t smem = static_cast<size_t>(G + 1) * (nc / 32) * sizeof(uint32_t);
  decode::gist_union_kernel<<<B * Hkv, 256, smem, st>>>(idx, Hq, Hkv, topk, idx_stride, nc, expanded, union_list,
                                                        union_stride, status);
  return cudaGetLastError();
}

}  // namespace bsa
