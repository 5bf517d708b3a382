// attn_fwd_wide_kernel.cuh -- attention forward for head dims 192 and 256 on B200 (sm_100a).
//
// The same computation as attn_fwd_kernel.cuh (the pages' tiled forward with an online
// softmax: "HipKittens: fast and furious AMD kernels", section "Performance results", over
// several head dims), for D too wide for its two-tile layout: two Q tiles would need
// 2 x (128 + D) tensor-memory columns, more than the 512 there are.  Here a CTA works on one
// 128-row Q tile at a time and ping-pongs two score buffers instead:
//
//   tensor memory:  S_0 [0,128)  S_1 [128,256)  O [256,256+D)
//   MMA order:      S(0) S(1) | P(0)V(0) S(2) | P(1)V(1) S(3) | ...
//
// S(g+1) is computed while the softmax works on S(g); S(g+2) goes into S(g)'s buffer after
// P(g) V(g) has read P(g) from it (tcgen05 MMAs of one CTA run in issue order).  The lazy
// rescale of O at a block waits for the previous block's P V to have completed.
//
// CTAs walk work items with a stride of the grid (persistent when the grid is below the item
// count).  An item is one query tile or, causal with enough of them to fill the GPU, the
// heaviest and the lightest remaining tile of a head (tiles nb-1-s and s: nb+1 KV blocks per
// item, so equal items).  Items are numbered head by head, so the CTAs running at one time
// share the K/V of a few heads in L2.  The block counter g runs on across tiles: the first
// scores of the next tile are computed while the softmax finishes the current one, and its Q
// is loaded once the current tile's last S has read Q.
//
// Warp roles (256 threads, one CTA per SM; no register reallocation is needed):
//   warps 0-3  softmax: TMEM lane = query row; epilogue of each tile
//   warp  4    TMA producer: per tile Q, then K_0, K_1, V_0, K_2, V_1, ... in MMA order
//   warp  5    MMA issuer (one elected lane)
//   warps 6-7  idle
// Every wait is bounded, as in the other kernels.
//
// kF8: Q, K, V are E4M3 bytes with per-tensor descales, as in the narrow kernel's E4M3 form:
// 128-byte swizzle rows hold 128 columns (D = 192 uses a second chunk half zero-filled by TMA),
// the MMAs are kind::f8f6f4 with K = 32 per instruction, P is packed four E4M3 values per TMEM
// column, the Q and K descales join the exponent constant and the V descale joins 1/l.
#pragma once

#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

constexpr int kWideThreads = 256;

enum : unsigned {
  kSiteWideProducer = 21,
  kSiteWideMma = 22,
  kSiteWideSoftmax = 23,
};

template <int D, bool kF8 = false>
struct WidePlan {
  static_assert(D == 192 || D == 256, "wide head dim must be 192 or 256");
  static constexpr int kElemBytes = kF8 ? 1 : 2;
  static constexpr int kRowElems = 128 / kElemBytes;     // columns per 128-byte swizzle row
  static constexpr int kChunks = (D + kRowElems - 1) / kRowElems;  // 128 B swizzle chunks per row
  static constexpr int kChunkBytes = kBlockM * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = kF8 ? 4 : (D == 256 ? 2 : 3);  // K/V ring depth (tiles)
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // q_full q_empty kv_full[S] kv_empty[S] s_full[2] p_full[2] pv_done o_full o_free drain
  static constexpr int kNumBars = 2 + 2 * kStages + 4 + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "wide forward shared memory plan exceeds 227 KB");
};

// Column pairs of every 8 whose exponentials run on the FMA-pipe polynomial instead of the
// special-function unit.  E4M3 halves the tensor work per block, so the exponentials weigh
// more: interleaved A/B on the eight wide workloads (N 2048/8192, causal or not) gave 3/8
// +1.2 to +3.9 % over 2/8 and 1/8 -1 to -3 % (bf16 keeps 2/8).
template <bool kF8>
__host__ __device__ constexpr int wide_poly_pairs_per8() {
  return kF8 ? 3 : 2;
}

struct WideParams {
  __nv_bfloat16* o;
  float* lse;
  int Hq, group, N, num_blocks;
  int causal;
  int pair;           // causal: an item is a head's heaviest and lightest remaining tile
  int num_items;      // work items: B*Hq*num_blocks tiles, or (pair) B*Hq*ceil(num_blocks/2) tile pairs
  float c;            // |scale| * log2(e) (E4M3: times the Q and K descales)
  float o_scale;      // E4M3: the V descale (1 for bf16)
  uint32_t idesc_s;   // 128 x 128 x D
  uint32_t idesc_pv;  // 128 x D x 128
};

// Tile `which` (0 or 1) of work item k: its query head and query tile; false if the item has
// no such tile (non-causal items hold one tile; the middle tile of an odd count is alone).
__device__ __forceinline__ bool wide_tile(const WideParams& p, int k, int which, int& head_q, int& qt) {
  const int nb = p.num_blocks;
  if (!p.pair) {
    if (which) return false;
    head_q = k / nb;
    const int kk = k - head_q * nb;
    qt = p.causal ? nb - 1 - kk : kk;   // a head's heaviest tiles first when causal
    return true;
  }
  const int sph = (nb + 1) >> 1;
  head_q = k / sph;
  const int s = k - head_q * sph;
  const int heavy = nb - 1 - s;
  if (which == 0) {
    qt = heavy;
    return true;
  }
  if (s >= heavy) return false;
  qt = s;
  return true;
}

template <int D, bool kF8 = false>
__global__ void __launch_bounds__(kWideThreads, 1)
    attn_fwd_wide_sm100(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const WideParams p) {
  using Plan = WidePlan<D, kF8>;
  constexpr int S = Plan::kStages;
  constexpr int kSSteps = D * Plan::kElemBytes / 32;                 // 32-byte K steps of S = Q K^T
  constexpr int kPVSteps = kBlockN * Plan::kElemBytes / 32;          // 32-byte K steps of P V
  constexpr uint32_t kPVStepBytes = (32 / Plan::kElemBytes) * 128;   // K rows of V per step x 128 B
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sQ = smem + Plan::kQOff;
  uint8_t* sKV = smem + Plan::kKVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;        // the tile's last S has read Q
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_full + 2 * S;  // [2]
  uint64_t* p_full = s_full + 2;       // [2]
  uint64_t* pv_done = s_full + 4;      // one phase per P V
  uint64_t* o_full = s_full + 5;       // one phase per tile: its last P V completed
  uint64_t* o_free = s_full + 6;       // one phase per tile: the softmax has read O
  uint64_t* drain = s_full + 7;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Plan::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = p.num_blocks;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kBlockM);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, kBlockM);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row, int head, uint64_t pol) {
#pragma unroll
        for (int ch = 0; ch < Plan::kChunks; ++ch)
          tma_load_3d(dst + ch * Plan::kChunkBytes, map, bar, ch * Plan::kRowElems, row, head, pol);
      };
      Ring ring;
      uint32_t filled = 0u, fill_par = 0u;
      uint32_t tiles = 0u;
      bool ok = true;
      for (int k = blockIdx.x; k < p.num_items && ok; k += gridDim.x) {
        for (int which = 0; which < 2 && ok; ++which) {
          int head_q, qt;
          if (!wide_tile(p, k, which, head_q, qt)) continue;
          const int head_kv = (head_q / p.Hq) * (p.Hq / p.group) + (head_q % p.Hq) / p.group;
          const int n = p.causal ? qt + 1 : nb;
          // Q of this tile once the previous tile's last S has read the buffer
          if (tiles > 0u && !(ok = wait_phase(q_empty, (tiles - 1u) & 1u, abort_flag, kSiteWideProducer))) break;
          mbar_arrive_expect_tx(q_full, Plan::kTileBytes);
          load_tile(&tmap_q, sQ, q_full, qt * kBlockM, head_q, pol_q);
          ++tiles;
          // Tiles in the order the MMAs read them: K_0, K_1, V_0, K_2, V_1, ..., V_{n-1}.
          const int total = 2 * n;
          for (int i = 0; i < total && ok; ++i) {
            bool is_k;
            int j;
            if (i < 2) {
              is_k = (i == 0) || n > 1;
              j = (i == 0) ? 0 : (n > 1 ? 1 : 0);
            } else {
              const int q2 = (i - 2) >> 1;   // pairs (V_q2, K_{q2+2}) after the first two K
              const bool second = ((i - 2) & 1) != 0;
              if (!second) {
                is_k = false;
                j = q2;
              } else {
                is_k = q2 + 2 < n;
                j = is_k ? q2 + 2 : q2 + 1;
              }
            }
            if (!(ok = wait_phase(&kv_empty[ring.stage], ring.phase ^ 1u, abort_flag, kSiteWideProducer))) break;
            mbar_arrive_expect_tx(&kv_full[ring.stage], Plan::kTileBytes);
            load_tile(is_k ? &tmap_k : &tmap_v, sKV + ring.stage * Plan::kTileBytes, &kv_full[ring.stage],
                      j * kBlockN, head_kv, pol_kv);
            filled |= 1u << ring.stage;
            fill_par = (fill_par & ~(1u << ring.stage)) | (ring.phase << ring.stage);
            ring.advance<S>();
          }
        }
      }
      // Drain: every issued copy lands before the CTA may exit.
      if (tiles > 0u) drain_phase(q_full, (tiles - 1u) & 1u, abort_flag);
      for (int s = 0; s < S; ++s)
        if (filled & (1u << s)) drain_phase(&kv_full[s], (fill_par >> s) & 1u, abort_flag);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
    const uint64_t desc_q = smem_desc_kmajor_sw128(smem_u32(sQ));
    const uint64_t desc_k = smem_desc_kmajor_sw128(smem_u32(sKV));
    const uint64_t desc_v = smem_desc_mnmajor_sw128(smem_u32(sKV), Plan::kChunkBytes);
    auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) tc_commit(bar);
      __syncwarp();
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool mine = wait_phase(bar, parity, abort_flag, kSiteWideMma);
      return __all_sync(0xffffffffu, mine);
    };
    Ring ring;
    // Takes the next ring tile (waits for it); returns its stage.
    auto next_tile = [&](bool& ok) -> uint32_t {
      const uint32_t st = ring.stage;
      ok = wait_all(&kv_full[st], ring.phase);
      ring.advance<S>();
      return st;
    };
    auto issue_s = [&](int b, uint32_t st) {
      const uint64_t db = adv(desc_k, st * Plan::kTileBytes);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kSSteps; ++kk) {
          const uint32_t off = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
          if constexpr (kF8)
            mma_ss_f8(tmem + b * 128, adv(desc_q, off), adv(db, off), p.idesc_s, kk > 0 ? 1u : 0u);
          else
            mma_ss(tmem + b * 128, adv(desc_q, off), adv(db, off), p.idesc_s, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto issue_pv = [&](int b, uint32_t st, bool accumulate) {
      const uint64_t dv = adv(desc_v, st * Plan::kTileBytes);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kPVSteps; ++kk) {
          if constexpr (kF8)
            mma_ts_f8(tmem + 256, tmem + b * 128 + kk * 8, adv(dv, kk * kPVStepBytes), p.idesc_pv,
                      (accumulate || kk > 0) ? 1u : 0u);
          else
            mma_ts(tmem + 256, tmem + b * 128 + kk * 8, adv(dv, kk * kPVStepBytes), p.idesc_pv,
                   (accumulate || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    uint32_t g = 0u;      // KV blocks of all earlier tiles: block j of this tile is g + j
    uint32_t tiles = 0u;
    bool ok = true;
    for (int k = blockIdx.x; k < p.num_items && ok; k += gridDim.x) {
      for (int which = 0; which < 2 && ok; ++which) {
        int head_q, qt;
        if (!wide_tile(p, k, which, head_q, qt)) continue;
        const int n = p.causal ? qt + 1 : nb;
        if (!(ok = wait_all(q_full, tiles & 1u))) break;
        // First two blocks' scores.  Their buffers last held P of the previous tile's last two
        // blocks, whose P V were issued before (issue order).
        uint32_t st = next_tile(ok);
        if (!ok) break;
        tc_fence_after();
        issue_s((int)(g & 1u), st);
        commit(&s_full[g & 1u]);
        commit(&kv_empty[st]);
        if (n == 1) commit(q_empty);
        if (n > 1) {
          st = next_tile(ok);
          if (!ok) break;
          tc_fence_after();
          issue_s((int)((g + 1u) & 1u), st);
          commit(&s_full[(g + 1u) & 1u]);
          commit(&kv_empty[st]);
          if (n == 2) commit(q_empty);
        }
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t gj = g + (uint32_t)j;
          const int b = (int)(gj & 1u);
          if (!(ok = wait_all(&p_full[b], (gj >> 1) & 1u))) break;
          // the first P V of a tile overwrites O: the previous tile's epilogue must have read it
          if (j == 0 && tiles > 0u && !(ok = wait_all(o_free, (tiles - 1u) & 1u))) break;
          const uint32_t vst = next_tile(ok);
          if (!ok) break;
          tc_fence_after();
          issue_pv(b, vst, j > 0);
          commit(pv_done);
          commit(&kv_empty[vst]);
          if (j + 2 < n) {
            const uint32_t kst = next_tile(ok);
            if (!ok) break;
            tc_fence_after();
            issue_s(b, kst);
            commit(&s_full[b]);
            commit(&kv_empty[kst]);
            if (j + 3 == n) commit(q_empty);
          }
        }
        if (!ok) break;
        commit(o_full);
        g += (uint32_t)n;
        ++tiles;
      }
    }
    commit(drain);
    drain_phase(drain, 0u, abort_flag);
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax warpgroup
    const int r = threadIdx.x;                     // query row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t t_o = tmem_base + lane_off + 256;
    const float c = p.c;
    uint32_t g = 0u, tiles = 0u;
    bool ok = true;
    for (int k = blockIdx.x; k < p.num_items && ok; k += gridDim.x) {
      for (int which = 0; which < 2 && ok; ++which) {
        int head_q, qt;
        if (!wide_tile(p, k, which, head_q, qt)) continue;
        const int n = p.causal ? qt + 1 : nb;
        const int row = qt * kBlockM + r;
        const int key_lim = p.causal ? min(row, p.N - 1) : (p.N - 1);
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t gj = g + (uint32_t)j;
          const int b = (int)(gj & 1u);
          const uint32_t t_s = tmem_base + lane_off + b * 128;
          if (!(ok = wait_phase(&s_full[b], (gj >> 1) & 1u, abort_flag, kSiteWideSoftmax))) break;
          tc_fence_after();
          float s[kBlockN];
          {
            uint32_t a0[32], a1[32], a2[32], a3[32];
            tmem_ld32(t_s + 0, a0);
            tmem_ld32(t_s + 32, a1);
            tmem_ld32(t_s + 64, a2);
            tmem_ld32(t_s + 96, a3);
            tmem_ld_wait();
            reg_fence32(a0);
            reg_fence32(a1);
            reg_fence32(a2);
            reg_fence32(a3);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              s[i] = __uint_as_float(a0[i]);
              s[32 + i] = __uint_as_float(a1[i]);
              s[64 + i] = __uint_as_float(a2[i]);
              s[96 + i] = __uint_as_float(a3[i]);
            }
          }
          const int k0 = j * kBlockN;
          if (k0 + kBlockN - 1 > key_lim) {
#pragma unroll
            for (int i = 0; i < kBlockN; ++i)
              if (k0 + i > key_lim) s[i] = -INFINITY;
          }
          float mx[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e] = max3f(s[e], s[4 + e], s[8 + e]);
#pragma unroll
          for (int i = 12; i < kBlockN - 4; i += 8) {
#pragma unroll
            for (int e = 0; e < 4; ++e) mx[e] = max3f(mx[e], s[i + e], s[i + 4 + e]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e] = fmaxf(mx[e], s[kBlockN - 4 + e]);
          const float m_new = fmaxf(m, fmaxf(max3f(mx[0], mx[1], mx[2]), mx[3]) * c);
          // Lazy rescale (as in the narrow kernel): the running max moves only when the row's
          // maximum grew by more than kRescaleLog2, and O (holding blocks < j once the previous
          // block's P V has completed) and l are then scaled by 2^(m - m_new).
          bool any_rescale = false;
          float alpha = 1.f;
          if (j == 0) {
            m = m_new;
          } else {
            const bool need = m_new > m + kRescaleLog2;
            any_rescale = __any_sync(0xffffffffu, need);
            if (need) {
              alpha = ex2_approx(m - m_new);
              l *= alpha;
              m = m_new;
            }
          }
          if (any_rescale) {
            // P(gj-1) V is the one P V that can still be running (S(gj) was issued after
            // P(gj-2) V): its phase is gj-1.
            if (!(ok = wait_phase(pv_done, (gj - 1u) & 1u, abort_flag, kSiteWideSoftmax))) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t ov[32];
              tmem_ld32(t_o + ch * 32, ov);
              tmem_ld_wait();
              reg_fence32(ov);
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st32(t_o + ch * 32, ov);
            }
          }
          // P = 2^(s c - m) -> bf16 pairs over the first 64 columns of S (E4M3: four per column
          // over the first 32); row sum in fp32.
          {
            const float2 c2 = make_float2(c, c);
            const float2 nm2 = make_float2(-m, -m);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t pk[32];
              float prev = 0.f, prev2 = 0.f;  // E4M3: the first pair of a group of four
#pragma unroll
              for (int i = 0; i < 64; i += 2) {
                const int col = half * 64 + i;
                const float2 x = fma2(make_float2(s[col], s[col + 1]), c2, nm2);
                float2 pr;
                if (((col >> 1) & 7) < wide_poly_pairs_per8<kF8>()) {
                  pr = exp2_poly2(x);
                } else {
                  pr.x = ex2_approx(x.x);
                  pr.y = ex2_approx(x.y);
                }
                acc[(i >> 1) & 3] = add2(acc[(i >> 1) & 3], pr);
                if constexpr (kF8) {
                  if ((i & 2) == 0) {
                    prev = pr.x;
                    prev2 = pr.y;
                  } else {
                    pk[i >> 2] = pack_e4m3x4(prev, prev2, pr.x, pr.y);
                  }
                } else {
                  pk[i >> 1] = pack_bf16x2(pr.x, pr.y);
                }
              }
              if constexpr (kF8) {
                uint32_t pk16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk16[i] = pk[i];
                tmem_st16(t_s + half * 16, pk16);
              } else {
                tmem_st32(t_s + half * 32, pk);
              }
            }
            const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
            l += a.x + a.y;
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_full[b]);
        }
        if (!ok) break;
        // Epilogue: O / l -> bf16, LSE = (m + log2 l) ln 2; O's columns are handed back to the
        // MMA warp (the next tile's first P V) once read.
        if (!(ok = wait_phase(o_full, tiles & 1u, abort_flag, kSiteWideSoftmax))) break;
        tc_fence_after();
        const bool row_ok = row < p.N;
        __nv_bfloat16* orow = p.o + ((size_t)head_q * p.N + (row_ok ? row : 0)) * D;
        const float inv_l = (kF8 ? p.o_scale : 1.f) / l;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld32(t_o + ch * 32, ov);
          tmem_ld_wait();
          reg_fence32(ov);
          if (ch == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(o_free);
          }
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
        if (row_ok) p.lse[(size_t)head_q * p.N + row] = (m + log2f(l)) * 0.69314718055994530942f;
        g += (uint32_t)n;
        ++tiles;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace attn
