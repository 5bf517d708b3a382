// attn_fwd_colsplit_kernel.cuh -- bf16 attention forward for head dims 32..128 on B200 (sm_100a),
// one Q tile per work unit, two score buffers, and the score columns split between two softmax
// warpgroups.  The library runs it for causal D = 128 at N <= 2048, where it measured 5-8 %
// faster than the two-tile kernel (attn_fwd_kernel.cuh); at longer N the two-tile kernel wins,
// because there each K/V tile it loads serves 256 query rows instead of 128.
//
// Method: the tiled attention forward with an online softmax ("Making AMD GPUs go brrr",
// section "Real kernel example": score matmul, exp2, row sums, probability-times-V matmul;
// "HipKittens: fast and furious AMD kernels", section "Performance results": causal and
// non-causal over several D and N).  The pages' AMD schedule keeps two wave groups alternating
// between compute and memory; here the B200 tensor core must never wait for the exponentials,
// so the dependency chain of a block is cut short in two ways:
//
//  * two score buffers: S(j+1) = Q K_{j+1}^T is computed while the softmax works on S(j);
//  * each 128-key score block is split by columns between two softmax warpgroups: warpgroup h
//    (h = 0, 1) handles keys 64h .. 64h+63 of every block for all 128 rows of the tile, with its
//    own running max m_h, row sum l_h and output accumulator O_h = sum_j P_h(j) V_j[64h:64h+64].
//    The halves never exchange anything per block; at the end of a unit the two partial results
//    are merged exactly:  M = max(m_0, m_1),  a_h = 2^(m_h - M),
//        O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1),   LSE = (M + log2(a_0 l_0 + a_1 l_1)) ln 2.
//
//   warps 0-3   softmax warpgroup 0 (score columns 0-63; TMEM lane = query row)
//   warps 4-7   softmax warpgroup 1 (score columns 64-127)
//   warp  8     TMA producer: Q per unit (two buffers), K and V through a ring, in MMA order
//   warp  9     MMA issuer
//   warp  10    output store: TMA tensor stores of each unit's staged O
//   warp  11    idle (completes the third warpgroup, which gives up registers)
//
// Tensor memory (512 columns):  S_0 [0,128)  S_1 [128,256)  O_0 [256,256+D)  O_1 [384,384+D).
// P_h(j) (bf16 pairs) overwrites the first 32 columns of warpgroup h's own 64 score columns.
//
// MMA order over the CTA's whole sequence of blocks (units back to back):
//     S(0) S(1) | P(0)V(0) S(2) | P(1)V(1) S(3) | ...
// where P(g)V(g) is two MMAs of K = 64 (O_0 += P_0 V[0:64], O_1 += P_1 V[64:128]) and S(g+2)
// reuses S(g)'s buffer after both have been issued (tcgen05 MMAs of a CTA run in issue order).
// S of a unit's first blocks is computed while the previous unit finishes: Q has two buffers.
// The epilogue of a unit stages O in that unit's Q buffer, free once its last S has completed
// (64-byte swizzle, 32-column chunks); the store warp writes it out with TMA tensor stores and
// hands the buffer back to the producer once the stores have read it.
//
// A work unit is one 128-row query tile of one head.  Persistent grid, static stride: causal
// steps pair a head's heaviest and lightest tiles (tile T-1-s and tile s: T+1 blocks per step);
// consecutive steps stay in one head and the heads of a GQA group are consecutive, so the CTAs
// running at the same time share K and V through L2.  Every mbarrier wait is bounded; named
// barriers are only ever reached by all of their participants (failures are agreed on at the
// end of each unit).
#pragma once

#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

constexpr int kCsThreads = 384;

enum : unsigned {
  kSiteCsProducer = 31,
  kSiteCsMma = 32,
  kSiteCsSoftmax = 33,
  kSiteCsEpilogue = 34,
  kSiteCsStore = 35,
};

template <int D>
struct CsPlan {
  static_assert(D == 32 || D == 64 || D == 96 || D == 128, "head dim must be 32, 64, 96 or 128");
  static constexpr int kChunks = (D + 63) / 64;          // 64-column (128-byte) swizzle chunks of a Q/K/V row
  static constexpr int kChunkBytes = kBlockM * 128;       // 16 KB
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = kChunks == 2 ? 4 : 8;    // K/V ring depth (tiles)
  static constexpr int kOChunks = D / 32;                 // 32-column output chunks (64-byte rows)
  static constexpr int kStageBytes = kBlockM * 64;        // one staged output chunk: 8 KB
  static_assert(kOChunks * kStageBytes <= kTileBytes, "staged O must fit in a Q buffer");
  static constexpr int kQOff = 0;                         // two Q buffers (O staging after their last use)
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kXOff = kKVOff + kStages * kTileBytes;  // (m, l) exchange [unit parity][warpgroup][row]
  static constexpr int kBarOff = kXOff + 2 * 2 * kBlockM * 8;
  // q_full[2] q_empty[2] o_staged[2] kv_full[S] kv_empty[S] s_full[2] p_full[2 buffers][2 halves]
  // pv_done o_full o_free drain
  static constexpr int kNumBars = 6 + 2 * kStages + 2 + 4 + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;             // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "column-split forward shared memory plan exceeds 227 KB");
};

struct CsParams {
  float* lse;
  int Hq, Hkv, N;
  int group;          // Hq / Hkv
  int num_tiles;      // T = ceil(N / 128): query tiles per head = KV blocks per head
  int num_units;      // B * Hq * T
  int num_steps;      // causal: B * Hq * ceil(T / 2); otherwise num_units
  int causal;
  FastDiv div_tiles;  // T
  FastDiv div_steps;  // ceil(T / 2)
  FastDiv div_hq;     // Hq
  FastDiv div_group;  // group
  float c;            // |scale| * log2(e)
  uint32_t idesc_s;   // S = Q K^T: 128 x 128 x D (negates A when scale < 0)
  uint32_t idesc_pv;  // O_h += P_h V_h: 128 x D x 64
};

struct CsUnit {
  int row0;     // first query row of the tile
  int head_q;   // b * Hq + hq
  int head_kv;  // b * Hkv + hq / group
  int n;        // KV blocks the tile visits
};

__device__ __forceinline__ CsUnit cs_make_unit(const CsParams& p, uint32_t head, int tile) {
  CsUnit w;
  const uint32_t b = fast_div(head, p.div_hq);
  const uint32_t hq = head - b * (uint32_t)p.Hq;
  w.row0 = tile * kBlockM;
  w.head_q = (int)head;
  w.head_kv = (int)(b * (uint32_t)p.Hkv + fast_div(hq, p.div_group));
  w.n = p.causal ? tile + 1 : p.num_tiles;
  return w;
}

// Work item `it` of this CTA: 0 = no more items, 1 = a unit in `w`, 2 = an empty slot (the
// middle tile of a head with an odd tile count, causal).
__device__ __forceinline__ int cs_item(const CsParams& p, int it, CsUnit& w) {
  if (p.causal) {
    const long long step = blockIdx.x + (long long)(it >> 1) * gridDim.x;
    if (step >= p.num_steps) return 0;
    const uint32_t head = fast_div((uint32_t)step, p.div_steps);
    const int s = (int)((uint32_t)step - head * p.div_steps.d);
    const int heavy = p.num_tiles - 1 - s;
    if ((it & 1) && s == heavy) return 2;
    w = cs_make_unit(p, head, (it & 1) ? s : heavy);
    return 1;
  }
  const long long u = blockIdx.x + (long long)it * gridDim.x;
  if (u >= p.num_units) return 0;
  const uint32_t head = fast_div((uint32_t)u, p.div_tiles);
  w = cs_make_unit(p, head, (int)((uint32_t)u - head * (uint32_t)p.num_tiles));
  return 1;
}

// Position in the CTA's sequence of (unit, KV block) pairs.
struct CsCursor {
  int it = 0;       // next work item to fetch
  CsUnit w;
  int j = 0;        // KV block within the unit
  int u = -1;       // ordinal of the current unit among this CTA's units
  bool valid = false;
};

__device__ __forceinline__ void cs_next_unit(const CsParams& p, CsCursor& c) {
  while (true) {
    const int got = cs_item(p, c.it++, c.w);
    if (got == 0) {
      c.valid = false;
      return;
    }
    if (got == 1) break;
  }
  c.valid = true;
  c.j = 0;
  ++c.u;
}

__device__ __forceinline__ void cs_advance(const CsParams& p, CsCursor& c) {
  if (++c.j >= c.w.n) cs_next_unit(p, c);
}

template <int D>
__global__ void __launch_bounds__(kCsThreads, 1)
    attn_fwd_colsplit_sm100(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                            const CsParams p) {
  using Plan = CsPlan<D>;
  constexpr int S = Plan::kStages;
  constexpr int kSSteps = D / 16;  // K = 16 steps of S = Q K^T
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem + Plan::kQOff;
  uint8_t* sKV = smem + Plan::kKVOff;
  float2* xml = reinterpret_cast<float2*>(smem + Plan::kXOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint64_t* q_full = bars;                 // [2]
  uint64_t* q_empty = bars + 2;            // [2]: released by the store warp
  uint64_t* o_staged = bars + 4;           // [2]: the unit's O is staged in Q buffer [qb]
  uint64_t* kv_full = bars + 6;            // [S]
  uint64_t* kv_empty = kv_full + S;        // [S]
  uint64_t* s_full = kv_empty + S;         // [2]
  uint64_t* p_full = s_full + 2;           // [2 buffers][2 halves]
  uint64_t* pv_done = p_full + 4;
  uint64_t* o_full = pv_done + 1;
  uint64_t* o_free = pv_done + 2;
  uint64_t* drain = pv_done + 3;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Plan::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&o_staged[i], 2 * kBlockM);
      mbar_init(&s_full[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&p_full[i], kBlockM);
    for (int i = 0; i < S; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 2 * kBlockM);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    tma_prefetch_desc(&tmap_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    regs_decrease<kRegsControl>();
    if (lane == 0) {
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      Ring ring;
      uint32_t filled = 0u, fill_par = 0u;      // per stage: ever filled / parity of its last fill
      // per Q buffer (bit qb): parity of the next empty-barrier wait (starting on the completed
      // "previous" phase), ever filled, parity of the last fill
      uint32_t q_par = 3u, q_filled = 0u, q_fill_par = 0u;
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row, int head, uint64_t pol) {
#pragma unroll
        for (int ch = 0; ch < Plan::kChunks; ++ch)
          tma_load_3d(dst + ch * Plan::kChunkBytes, map, bar, ch * 64, row, head, pol);
      };
      auto load_kv = [&](const CUtensorMap* map, int row, int head) -> bool {
        if (!wait_phase(&kv_empty[ring.stage], ring.phase ^ 1u, abort_flag, kSiteCsProducer)) return false;
        mbar_arrive_expect_tx(&kv_full[ring.stage], Plan::kTileBytes);
        load_tile(map, sKV + ring.stage * Plan::kTileBytes, &kv_full[ring.stage], row, head, pol_kv);
        filled |= 1u << ring.stage;
        fill_par = (fill_par & ~(1u << ring.stage)) | (ring.phase << ring.stage);
        ring.advance<S>();
        return true;
      };
      // K of the cursor's block, preceded by the unit's Q tile when the block is its first.
      auto load_k = [&](const CsCursor& c) -> bool {
        if (c.j == 0) {
          const int qb = c.u & 1;
          if (!wait_phase(&q_empty[qb], (q_par >> qb) & 1u, abort_flag, kSiteCsProducer)) return false;
          q_par ^= 1u << qb;
          mbar_arrive_expect_tx(&q_full[qb], Plan::kTileBytes);
          load_tile(&tmap_q, sQ + qb * Plan::kTileBytes, &q_full[qb], c.w.row0, c.w.head_q, pol_q);
          if (q_filled & (1u << qb)) q_fill_par ^= 1u << qb;
          q_filled |= 1u << qb;
        }
        return load_kv(&tmap_k, c.j * kBlockN, c.w.head_kv);
      };
      CsCursor sc, pc;
      cs_next_unit(p, sc);
      cs_next_unit(p, pc);
      bool ok = true;
      // The order the MMA warp reads the ring in: K(0), K(1), then V(g), K(g+2) for g = 0, 1, ...
      for (int i = 0; i < 2 && ok && sc.valid; ++i) {
        ok = load_k(sc);
        cs_advance(p, sc);
      }
      while (ok && pc.valid) {
        ok = load_kv(&tmap_v, pc.j * kBlockN, pc.w.head_kv);
        if (ok && sc.valid) {
          ok = load_k(sc);
          cs_advance(p, sc);
        }
        cs_advance(p, pc);
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      for (int s = 0; s < S; ++s)
        if (filled & (1u << s)) drain_phase(&kv_full[s], (fill_par >> s) & 1u, abort_flag);
      for (int t = 0; t < 2; ++t)
        if (q_filled & (1u << t)) drain_phase(&q_full[t], (q_fill_par >> t) & 1u, abort_flag);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule (warp-uniform control flow); one elected lane issues.
    regs_decrease<kRegsControl>();
    {
      Ring ring;
      uint32_t q_par = 0u, of_par = 1u;  // q_par bit qb: parity of the next wait on q_full[qb]
      const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
      const uint64_t desc_q = smem_desc_kmajor_sw128(smem_u32(sQ));
      const uint64_t desc_k = smem_desc_kmajor_sw128(smem_u32(sKV));
      const uint64_t desc_v = smem_desc_mnmajor_sw128(smem_u32(sKV), Plan::kChunkBytes);
      const uint32_t idesc_s = p.idesc_s, idesc_pv = p.idesc_pv;
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool mine = wait_phase(bar, parity, abort_flag, kSiteCsMma);
        return __all_sync(0xffffffffu, mine);
      };
      auto next_stage = [&](bool& ok) -> uint32_t {
        const uint32_t st = ring.stage;
        ok = wait_all(&kv_full[st], ring.phase);
        ring.advance<S>();
        return st;
      };
      uint32_t gs = 0;  // blocks whose S has been issued
      // S(g) = Q K_j^T into score buffer g & 1.
      auto issue_s = [&](const CsCursor& c) -> bool {
        const int qb = c.u & 1;
        if (c.j == 0) {
          if (!wait_all(&q_full[qb], (q_par >> qb) & 1u)) return false;
          q_par ^= 1u << qb;
        }
        bool ok;
        const uint32_t st = next_stage(ok);
        if (!ok) return false;
        tc_fence_after();
        const uint64_t da = adv(desc_q, qb * Plan::kTileBytes);
        const uint64_t db = adv(desc_k, st * Plan::kTileBytes);
        const uint32_t d_tmem = tmem + (gs & 1u) * 128;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kSSteps; ++kk) {
            const uint32_t off = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
            mma_ss(d_tmem, adv(da, off), adv(db, off), idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
        commit(&s_full[gs & 1u]);
        commit(&kv_empty[st]);
        ++gs;
        return true;
      };
      // O_h += P_h(g) V(g)[64h : 64h+64]: four K = 16 steps, P_h from TMEM (8 columns per step),
      // V as an MN-major operand (16 key rows of 128 bytes per step).
      auto issue_pv = [&](int h, uint32_t sbuf, uint32_t vst, bool accumulate) {
        const uint64_t dv = adv(desc_v, vst * Plan::kTileBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + 256 + 128 * h, tmem + sbuf * 128 + 64 * h + kk * 8, adv(dv, (4 * h + kk) * 2048),
                   idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
      };

      CsCursor sc, pc;
      cs_next_unit(p, sc);
      cs_next_unit(p, pc);
      bool ok = true;
      for (int i = 0; i < 2 && ok && sc.valid; ++i) {
        ok = issue_s(sc);
        cs_advance(p, sc);
      }
      uint32_t gp = 0;  // blocks whose P V has been issued
      while (ok && pc.valid) {
        const uint32_t b = gp & 1u, ph = (gp >> 1) & 1u;
        if (!(ok = wait_all(&p_full[2 * b], ph))) break;
        if (pc.j == 0) {
          if (!(ok = wait_all(o_free, of_par))) break;
          of_par ^= 1u;
        }
        const uint32_t vst = next_stage(ok);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, b, vst, pc.j > 0);
        if (!(ok = wait_all(&p_full[2 * b + 1], ph))) break;
        tc_fence_after();
        issue_pv(1, b, vst, pc.j > 0);
        commit(pv_done);
        commit(&kv_empty[vst]);
        if (pc.j == pc.w.n - 1) commit(o_full);
        if (sc.valid) {
          if (!(ok = issue_s(sc))) break;
          cs_advance(p, sc);
        }
        ++gp;
        cs_advance(p, pc);
      }
      // Drain: all MMAs issued by this warp complete before TMEM is released.
      commit(drain);
      drain_phase(drain, 0u, abort_flag);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    regs_increase<kRegsSoftmax>();
    const int h = warp >> 2;                        // score columns 64h .. 64h+63
    const int r = threadIdx.x & 127;                // query row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_o0 = tmem_base + lane_off + 256;  // O_0; O_1 at +128
    const uint32_t t_oh = t_o0 + 128 * h;
    const float c = p.c;
    uint32_t g = 0, o_par = 0;
    bool ok = true;
    int u = 0;
    for (int it = 0; ok; ++it) {
      CsUnit w;
      const int got = cs_item(p, it, w);
      if (got == 0) break;
      if (got == 2) continue;
      const int row = w.row0 + r;
      const int key_lim = p.causal ? min(row, p.N - 1) : (p.N - 1);
      float m = -INFINITY, l = 0.f;

      for (int j = 0; j < w.n; ++j, ++g) {
        if (!ok) continue;  // after a failed wait: reach the end-of-unit agreement without further waits
        const uint32_t b = g & 1u;
        if (!(ok = wait_phase(&s_full[b], (g >> 1) & 1u, abort_flag, kSiteCsSoftmax))) continue;
        tc_fence_after();
        const uint32_t t_s = tmem_base + lane_off + b * 128 + 64 * h;
        float s[64];
        {
          uint32_t a0[32], a1[32];
          tmem_ld32(t_s + 0, a0);
          tmem_ld32(t_s + 32, a1);
          tmem_ld_wait();
          reg_fence32(a0);
          reg_fence32(a1);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(a0[i]);
            s[32 + i] = __uint_as_float(a1[i]);
          }
        }
        const int k0 = j * kBlockN + 64 * h;
        if (k0 + 63 > key_lim) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (k0 + i > key_lim) s[i] = -INFINITY;
        }
        float mx[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mx[e] = max3f(s[e], s[4 + e], s[8 + e]);
#pragma unroll
        for (int i = 12; i < 60; i += 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e] = max3f(mx[e], s[i + e], s[i + 4 + e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) mx[e] = fmaxf(mx[e], s[60 + e]);
        const float m_new = fmaxf(m, fmaxf(max3f(mx[0], mx[1], mx[2]), mx[3]) * c);
        // Lazy correction: the running max moves only when the row's maximum grew by more than
        // kRescaleLog2; O_h (blocks < j, once P(g-1) V has completed) and l are then scaled.
        bool any_rescale = false;
        float alpha = 1.f;
        if (j == 0) {
          m = m_new;
        } else {
          const bool need = m_new > m + kRescaleLog2;
          any_rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = ex2_approx(m - m_new);  // 0 while m is still -inf (no key of this half seen yet)
            l *= alpha;
            m = m_new;
          }
        }
        if (any_rescale) {
          // S(g) completing implies P(g-2) V has; P(g-1) V may still be running.
          if (!(ok = wait_phase(pv_done, (g - 1u) & 1u, abort_flag, kSiteCsSoftmax))) continue;
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(t_oh + ch * 32, ov);
            tmem_ld_wait();
            reg_fence32(ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(t_oh + ch * 32, ov);
          }
        }
        // P_h = 2^(s c - m) -> bf16 pairs over the first 32 of this half's columns; row sum in fp32.
        // While no key of this half has been allowed (m = -inf) every p is 0: use 0 for m then.
        const float m_use = (m == -INFINITY) ? 0.f : m;
        {
          const float2 c2 = make_float2(c, c);
          const float2 nm2 = make_float2(-m_use, -m_use);
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            const float2 x = fma2(make_float2(s[i], s[i + 1]), c2, nm2);
            float2 pr;
            if (((i >> 1) & 7) < poly_pairs_per8<D>()) {
              pr = exp2_poly2(x);
            } else {
              pr.x = ex2_approx(x.x);
              pr.y = ex2_approx(x.y);
            }
            acc[(i >> 1) & 3] = add2(acc[(i >> 1) & 3], pr);
            pk[i >> 1] = pack_bf16x2(pr.x, pr.y);
          }
          tmem_st32(t_s, pk);
          const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
          l += a.x + a.y;
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * b + h]);
      }

      // ---- end of the unit: agree on success, exchange (m_h, l_h), merge and store O, LSE.
      if (ok) ok = wait_phase(o_full, o_par, abort_flag, kSiteCsEpilogue);
      o_par ^= 1u;
      xml[((u & 1) * 2 + h) * kBlockM + r] = make_float2(m, l);
      ok = bar_and(7, 2 * kBlockM, ok);
      if (!ok) break;
      const float2 ml0 = xml[((u & 1) * 2 + 0) * kBlockM + r];
      const float2 ml1 = xml[((u & 1) * 2 + 1) * kBlockM + r];
      const float mt = fmaxf(ml0.x, ml1.x);
      const float a0 = (ml0.x == -INFINITY) ? 0.f : ex2_approx(ml0.x - mt);
      const float a1 = (ml1.x == -INFINITY) ? 0.f : ex2_approx(ml1.x - mt);
      const float lt = fmaf(ml1.y, a1, ml0.y * a0);
      const float inv_l = 1.f / lt;
      const float w0 = a0 * inv_l, w1 = a1 * inv_l;
      tc_fence_after();
      if (h >= Plan::kOChunks) {
        // no output chunk for this warpgroup (D = 32): its O columns are not read
        tc_fence_before();
        mbar_arrive(o_free);
      }
      // O is staged in this unit's Q buffer: its last S has completed (o_full follows every MMA
      // of the unit), and the producer reloads it only after the store warp has released it.
      const uint32_t stage_row = smem_u32(sQ + (u & 1) * Plan::kTileBytes) + r * 64;
#pragma unroll
      for (int ch = h; ch < Plan::kOChunks; ch += 2) {
        uint32_t x0[32], x1[32];
        tmem_ld32(t_o0 + ch * 32, x0);
        tmem_ld32(t_o0 + 128 + ch * 32, x1);
        tmem_ld_wait();
        reg_fence32(x0);
        reg_fence32(x1);
        if (ch + 2 >= Plan::kOChunks) {
          // this warpgroup's last reads of O: the next unit's P V may overwrite it
          tc_fence_before();
          mbar_arrive(o_free);
        }
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(fmaf(__uint_as_float(x1[2 * i]), w1, __uint_as_float(x0[2 * i]) * w0),
                                  fmaf(__uint_as_float(x1[2 * i + 1]), w1, __uint_as_float(x0[2 * i + 1]) * w0));
        // chunk ch: 128 rows of 64 bytes, four 16-byte pieces per row, 64-byte swizzle (piece q of
        // row r at position q ^ ((r >> 1) & 3))
        const uint32_t row_addr = stage_row + ch * Plan::kStageBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(row_addr + ((q ^ ((r >> 1) & 3)) << 4), packed[4 * q], packed[4 * q + 1], packed[4 * q + 2],
                       packed[4 * q + 3]);
      }
      // make the staged rows visible to the TMA (async proxy), then hand them to the store warp
      fence_proxy_async_smem();
      mbar_arrive(&o_staged[u & 1]);
      if (h == 0 && row < p.N) p.lse[(size_t)w.head_q * p.N + row] = (mt + log2f(lt)) * 0.69314718055994530942f;
      ++u;
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ output store warp
    // Per unit: wait until both softmax warpgroups have staged O in the unit's Q buffer, store
    // it with TMA tensor stores (rows past N are not written), wait until the stores have read
    // the buffer and give it back to the producer.
    regs_decrease<kRegsControl>();
    if (lane == 0) {
      uint32_t st_par = 0u;  // bit qb: parity of the next wait on o_staged[qb]
      int u = 0;
      for (int it = 0;; ++it) {
        CsUnit w;
        const int got = cs_item(p, it, w);
        if (got == 0) break;
        if (got == 2) continue;
        const int qb = u & 1;
        if (!wait_phase(&o_staged[qb], (st_par >> qb) & 1u, abort_flag, kSiteCsStore)) break;
        st_par ^= 1u << qb;
        const uint8_t* stage = sQ + qb * Plan::kTileBytes;
#pragma unroll
        for (int ch = 0; ch < Plan::kOChunks; ++ch)
          tma_store_3d(&tmap_o, stage + ch * Plan::kStageBytes, ch * 32, w.row0, w.head_q);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(&q_empty[qb]);
        ++u;
      }
      // every TMA store has completed before the CTA exits
      bulk_wait_group0();
    }
    __syncwarp();
  } else {
    regs_decrease<kRegsControl>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace attn
