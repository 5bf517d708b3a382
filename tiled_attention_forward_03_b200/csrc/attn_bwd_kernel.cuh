// attn_bwd_kernel.cuh -- tiled attention backward for B200 (sm_100a).
//
// Gradients of the forward pass in attn_fwd_kernel.cuh.  The pages name an attention
// backward kernel beside the forward one ("HipKittens: fast and furious AMD kernels",
// section "Performance results"; the vendor-library baselines it is compared with are in
// "State of the AMD ecosystem") but print no formula; the plain definition, with P the
// forward's probabilities rebuilt from the saved LSE, is
//
//   P_ij  = exp(scale q_i.k_j - LSE_i)            (0 where the causal mask hides j)
//   dP    = dO V^T,   delta_i = sum_d dO_id O_id,   dS = P o (dP - delta)
//   dV    = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K
//
// and for grouped heads the dK, dV of a KV head sum over the query heads sharing it.
//
// Three launches:
//   attn_bwd_prep   delta and LSE * log2(e) per query row, into a workspace padded to
//                   whole 128-row tiles (pad rows hold 0)
//   attn_bwd_sm100<D, kKV = true>   one CTA per 128-key block of a KV head: keeps K_j, V_j
//                   in shared memory, streams the Q/dO tiles of every query head of the
//                   group, accumulates dV_j and dK_j in tensor memory
//   attn_bwd_sm100<D, kKV = false>  one CTA per 128-query block: keeps Q_i, dO_i, streams
//                   the K/V tiles, accumulates dQ_i in tensor memory
// Each CTA owns its output rows outright, so there are no atomics and the result does
// not depend on the order CTAs run in.  The price is that the score and dP tiles are
// computed by both kernels (7 tile matmuls per (query block, key block) instead of 5).
//
// One kernel serves both passes.  In its own terms a CTA has "row" tiles R0, R1
// (resident: K, V or Q, dO) and streams "column" tiles C0, C1 (Q, dO or K, V):
//
//   S  = R0 C0^T     (scores, or their transpose in the KV pass)
//   dP = R1 C1^T
//   P  = 2^(S c - lse2),  dS = P o (dP - delta)         (lse2, delta per query)
//   acc_p  += P  C1   (KV pass: dV)          acc_ds += dS C0   (dK or dQ)
//
// Warp roles (320 threads):
//   warps 0-7  softmax: TMEM lane = tile row (warp % 4 picks the 32-lane slice), warps 0-3
//              take columns 0-63 and warps 4-7 columns 64-127 of each tile
//   warp  8    TMA producer
//   warp  9    MMA issuer (one elected lane)
//
// Tensor memory (512 columns):
//   [  0,128) S fp32; P (bf16 pairs, KV pass) overwrites columns [0,32) and [64,96)
//   [128,256) dP fp32; dS (bf16 pairs) overwrites columns [128,160) and [192,224)
//   [256,256+D) acc_p (dV);  [384,384+D) acc_ds (dK or dQ)
// Each softmax warpgroup writes its packed P / dS over the first half of the columns it
// has just read, so the two warpgroups never touch each other's columns.
//
// MMA order per column tile t (tcgen05 MMAs of one CTA run in issue order):
//   acc_p(t)  S(t+1)  acc_ds(t)  dP(t+1)
// S(t+1) overwrites P(t) only after acc_p(t) has read it, and dP(t+1) overwrites dS(t)
// only after acc_ds(t); the softmax of t+1 (exponentials) overlaps acc_ds(t) and dP(t+1).
//
// Every wait is bounded, as in the forward kernel.
#pragma once

#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

constexpr int kBwdThreads = 320;
constexpr float kLog2e = 1.4426950408889634f;

enum : unsigned {
  kSiteBwdProducer = 12,
  kSiteBwdMmaRow = 13,
  kSiteBwdMmaCol = 14,
  kSiteBwdMmaP = 15,
  kSiteBwdMmaDS = 16,
  kSiteBwdSoftS = 17,
  kSiteBwdSoftDP = 18,
  kSiteBwdSoftAcc = 19,
};

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16),
// completion counted on `bar` in bytes.
ATTN_DEV void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

template <int D>
struct BwdPlan {
  static_assert(D == 32 || D == 64 || D == 96 || D == 128, "head dim must be 32, 64, 96 or 128");
  static constexpr int kChunks = (D + 63) / 64;
  static constexpr int kChunkBytes = kBlockM * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (kChunks == 2) ? 2 : 4;   // column-tile ring depth
  static constexpr int kROff = 0;                          // R0, R1
  static constexpr int kCOff = 2 * kTileBytes;             // per stage: C0, C1
  static constexpr int kVecOff = kCOff + kStages * 2 * kTileBytes;  // per stage: lse2[128], delta[128]
  static constexpr int kVecBytes = 2 * kBlockN * 4;
  static constexpr int kBarOff = kVecOff + kStages * kVecBytes;
  // r_full c_full[S] c_empty[S] s_full dp_full p_ready ds_ready acc_full drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

struct BwdParams {
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;    // [B*Hq][Npad] LSE * log2(e)
  const float* delta;   // [B*Hq][Npad] rowsum(dO o O)
  int Hq, Hkv, N, Npad, group, num_blocks;
  int causal;
  float c;              // scale * log2(e)
  float scale;
  uint32_t idesc_s;     // 128 x 128 x D, both operands K-major
  uint32_t idesc_acc;   // 128 x D x 128, A from TMEM, B MN-major
};

// delta_i = sum_d dO_id O_id (fp32 sums of the bf16 products) and lse2_i = LSE_i log2(e),
// one 16-thread group per row of the padded [B*Hq][Npad] layout; pad rows get 0.
__global__ void attn_bwd_prep(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                              const float* __restrict__ lse, float* __restrict__ lse2,
                              float* __restrict__ delta, long long rows, int N, int Npad, int D) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4);
  const int l16 = threadIdx.x & 15;
  if (row >= rows) return;  // whole 16-lane groups leave together
  const long long bh = row / Npad;
  const int qi = (int)(row - bh * Npad);
  float acc = 0.f;
  if (qi < N) {
    const size_t base = ((size_t)bh * N + qi) * D;
    for (int d = l16 * 8; d < D; d += 128) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + base + d);
      const uint4 b = *reinterpret_cast<const uint4*>(dout + base + d);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]);
        const float2 fb = __bfloat1622float2(pb[e]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
  }
  const unsigned mask = 0xffffu << (threadIdx.x & 16);
  acc += __shfl_xor_sync(mask, acc, 8, 16);
  acc += __shfl_xor_sync(mask, acc, 4, 16);
  acc += __shfl_xor_sync(mask, acc, 2, 16);
  acc += __shfl_xor_sync(mask, acc, 1, 16);
  if (l16 == 0) {
    delta[row] = acc;
    lse2[row] = qi < N ? lse[(size_t)bh * N + qi] * kLog2e : 0.f;
  }
}

// The CTA's work: its row tile and how many column tiles it streams.
struct BwdUnit {
  int row_head;   // head of the R tiles (KV head in the KV pass, query head otherwise)
  int rb;         // row block
  int n;          // column tiles
  int cpb;        // column tiles per query head (KV pass)
  int c0;         // first column block
};

template <bool kKV>
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams& p) {
  BwdUnit w;
  const int nb = p.num_blocks;
  const long long u = blockIdx.x;
  w.row_head = (int)(u / nb);
  const int k = (int)(u - (long long)w.row_head * nb);
  if (kKV) {
    // key block rb sees query blocks rb..nb-1 (causal): heaviest (rb = 0) first
    w.rb = k;
    w.c0 = p.causal ? w.rb : 0;
    w.cpb = nb - w.c0;
    w.n = w.cpb * p.group;
  } else {
    // query block rb sees key blocks 0..rb (causal): heaviest (rb = nb-1) first
    w.rb = nb - 1 - k;
    w.c0 = 0;
    w.cpb = p.causal ? w.rb + 1 : nb;
    w.n = w.cpb;
  }
  return w;
}

// Column tile `it` of a unit: its block index and head.
template <bool kKV>
__device__ __forceinline__ void bwd_col(const BwdParams& p, const BwdUnit& w, int it, int& cb, int& chead) {
  if (kKV) {
    const int hh = it / w.cpb;
    cb = w.c0 + (it - hh * w.cpb);
    chead = w.row_head * p.group + hh;  // query heads of this KV head's group
  } else {
    cb = it;
    chead = w.row_head / p.group;       // the query head's KV head
  }
}

template <int D, bool kKV>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_sm100(const __grid_constant__ CUtensorMap tmap_r0, const __grid_constant__ CUtensorMap tmap_r1,
                   const __grid_constant__ CUtensorMap tmap_c0, const __grid_constant__ CUtensorMap tmap_c1,
                   const BwdParams p) {
  using Plan = BwdPlan<D>;
  constexpr int S = Plan::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sR = smem + Plan::kROff;
  uint8_t* sC = smem + Plan::kCOff;
  float* sVec = reinterpret_cast<float*>(smem + Plan::kVecOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint64_t* r_full = bars;
  uint64_t* c_full = bars + 1;
  uint64_t* c_empty = bars + 1 + S;
  uint64_t* s_full = bars + 1 + 2 * S;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_ready = s_full + 2;
  uint64_t* ds_ready = s_full + 3;
  uint64_t* acc_full = s_full + 4;
  uint64_t* drain = s_full + 5;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Plan::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const BwdUnit w = bwd_unit<kKV>(p);

  if (threadIdx.x == 0) {
    mbar_init(r_full, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(&c_full[i], 1);
      mbar_init(&c_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmap_r0);
    tma_prefetch_desc(&tmap_r1);
    tma_prefetch_desc(&tmap_c0);
    tma_prefetch_desc(&tmap_c1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_once = l2_policy_evict_first();
      const uint64_t pol_shared = l2_policy_evict_last();
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row, int head, uint64_t pol) {
#pragma unroll
        for (int ch = 0; ch < Plan::kChunks; ++ch)
          tma_load_3d(dst + ch * Plan::kChunkBytes, map, bar, ch * 64, row, head, pol);
      };
      mbar_arrive_expect_tx(r_full, 2 * Plan::kTileBytes);
      load_tile(&tmap_r0, sR, r_full, w.rb * kBlockM, w.row_head, pol_once);
      load_tile(&tmap_r1, sR + Plan::kTileBytes, r_full, w.rb * kBlockM, w.row_head, pol_once);
      Ring ring;
      uint32_t filled = 0u, fill_par = 0u;
      for (int it = 0; it < w.n; ++it) {
        if (!wait_phase(&c_empty[ring.stage], ring.phase ^ 1u, abort_flag, kSiteBwdProducer)) break;
        int cb, chead;
        bwd_col<kKV>(p, w, it, cb, chead);
        uint64_t* bar = &c_full[ring.stage];
        mbar_arrive_expect_tx(bar, 2 * Plan::kTileBytes + (kKV ? Plan::kVecBytes : 0));
        uint8_t* dst = sC + ring.stage * 2 * Plan::kTileBytes;
        load_tile(&tmap_c0, dst, bar, cb * kBlockN, chead, pol_shared);
        load_tile(&tmap_c1, dst + Plan::kTileBytes, bar, cb * kBlockN, chead, pol_shared);
        if (kKV) {
          const size_t off = (size_t)chead * p.Npad + (size_t)cb * kBlockN;
          float* vec = sVec + ring.stage * 2 * kBlockN;
          bulk_load_1d(vec, p.lse2 + off, kBlockN * 4, bar);
          bulk_load_1d(vec + kBlockN, p.delta + off, kBlockN * 4, bar);
        }
        filled |= 1u << ring.stage;
        fill_par = (fill_par & ~(1u << ring.stage)) | (ring.phase << ring.stage);
        ring.advance<S>();
      }
      // Drain: every issued copy lands before the CTA may exit.
      drain_phase(r_full, 0u, abort_flag);
      for (int s = 0; s < S; ++s)
        if (filled & (1u << s)) drain_phase(&c_full[s], (fill_par >> s) & 1u, abort_flag);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
    const uint64_t desc_r0 = smem_desc_kmajor_sw128(smem_u32(sR));
    const uint64_t desc_r1 = smem_desc_kmajor_sw128(smem_u32(sR + Plan::kTileBytes));
    const uint64_t desc_c_k = smem_desc_kmajor_sw128(smem_u32(sC));
    const uint64_t desc_c_mn = smem_desc_mnmajor_sw128(smem_u32(sC), Plan::kChunkBytes);
    auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
    // D = A B^T over the head dim (both K-major): S (R0, C0) or dP (R1, C1).
    auto issue_rc = [&](uint32_t d_col, uint64_t da, uint64_t db) {
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
          mma_ss(tmem + d_col, adv(da, off), adv(db, off), p.idesc_s, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    // acc (+)= X C over the 128 tile columns (X bf16 pairs in TMEM at columns a_col + [0,32)
    // and a_col + 64 + [0,32); C MN-major in shared memory).
    auto issue_acc = [&](uint32_t d_col, uint32_t a_col, uint64_t db, bool accumulate) {
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + 64 * (kk >> 2) + 8 * (kk & 3), adv(db, kk * 2048), p.idesc_acc,
                 (accumulate || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) tc_commit(bar);
      __syncwarp();
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
      const bool mine = wait_phase(bar, parity, abort_flag, site);
      return __all_sync(0xffffffffu, mine);
    };
    auto stage_bytes = [](uint32_t st) -> uint32_t { return st * 2 * Plan::kTileBytes; };

    bool ok = wait_all(r_full, 0u, kSiteBwdMmaRow);
    Ring ring;
    if (ok && w.n > 0) ok = wait_all(&c_full[0], 0u, kSiteBwdMmaCol);
    if (ok && w.n > 0) {
      tc_fence_after();
      issue_rc(0, desc_r0, adv(desc_c_k, stage_bytes(0)));
      commit(s_full);
      issue_rc(128, desc_r1, adv(desc_c_k, stage_bytes(0) + Plan::kTileBytes));
      commit(dp_full);
    }
    for (int it = 0; it < w.n && ok; ++it) {
      const uint32_t st = ring.stage;
      const uint32_t par = (uint32_t)it & 1u;
      if (!(ok = wait_all(p_ready, par, kSiteBwdMmaP))) break;
      tc_fence_after();
      if (kKV) issue_acc(256, 0, adv(desc_c_mn, stage_bytes(st) + Plan::kTileBytes), it > 0);
      ring.advance<S>();
      const bool has_next = it + 1 < w.n;
      if (has_next) {
        if (!(ok = wait_all(&c_full[ring.stage], ring.phase, kSiteBwdMmaCol))) break;
        tc_fence_after();
        issue_rc(0, desc_r0, adv(desc_c_k, stage_bytes(ring.stage)));
        commit(s_full);
      }
      if (!(ok = wait_all(ds_ready, par, kSiteBwdMmaDS))) break;
      tc_fence_after();
      issue_acc(384, 128, adv(desc_c_mn, stage_bytes(st)), it > 0);
      commit(&c_empty[st]);
      if (has_next) {
        issue_rc(128, desc_r1, adv(desc_c_k, stage_bytes(ring.stage) + Plan::kTileBytes));
        commit(dp_full);
      }
    }
    if (ok) commit(acc_full);
    // Drain: all MMAs issued by this warp complete before TMEM is released.
    commit(drain);
    drain_phase(drain, 0u, abort_flag);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int r = threadIdx.x & 127;            // tile row == TMEM lane
    const int h = warp >> 2;                    // column half
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + 64 * h;
    const uint32_t t_dp = tmem_base + lane_off + 128 + 64 * h;
    const float c = p.c;
    const int row = w.rb * kBlockM + r;         // global index of this thread's tile row
    // Q pass: the row's lse2 and delta are fixed for the whole unit.
    float row_lse2 = 0.f, row_delta = 0.f;
    if (!kKV) {
      const size_t off = (size_t)w.row_head * p.Npad + row;
      row_lse2 = p.lse2[off];
      row_delta = p.delta[off];
    }
    uint32_t s_par = 0u;
    bool ok = true;
    Ring ring;
    for (int it = 0; it < w.n && ok; ++it) {
      int cb, chead;
      bwd_col<kKV>(p, w, it, cb, chead);
      const float* vec = sVec + ring.stage * 2 * kBlockN + 64 * h;
      if (!(ok = wait_phase(s_full, s_par, abort_flag, kSiteBwdSoftS))) break;
      if (kKV && !(ok = wait_phase(&c_full[ring.stage], ring.phase, abort_flag, kSiteBwdSoftS))) break;
      tc_fence_after();
      float pv[64];
      {
        uint32_t a0[32], a1[32];
        tmem_ld32(t_s, a0);
        tmem_ld32(t_s + 32, a1);
        tmem_ld_wait();
        reg_fence32(a0);
        reg_fence32(a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pv[i] = __uint_as_float(a0[i]);
          pv[32 + i] = __uint_as_float(a1[i]);
        }
      }
      if (!kKV) {
        // The scores are in registers: the next tile's S may overwrite them now.
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      // P = 2^(S c - lse2) (lse2 of the column's query in the KV pass, of the row's otherwise)
      if (kKV) {
#pragma unroll
        for (int i = 0; i < 64; i += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(vec + i);
          pv[i] = ex2_approx(fmaf(pv[i], c, -l4.x));
          pv[i + 1] = ex2_approx(fmaf(pv[i + 1], c, -l4.y));
          pv[i + 2] = ex2_approx(fmaf(pv[i + 2], c, -l4.z));
          pv[i + 3] = ex2_approx(fmaf(pv[i + 3], c, -l4.w));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) pv[i] = ex2_approx(fmaf(pv[i], c, -row_lse2));
      }
      // Masks.  KV pass: row = key, column = query; the causal mask hides query < key
      // (diagonal block only), and key rows past N are zeroed.  Q pass: row = query,
      // column = key; the mask hides key > query and keys past N.
      {
        const int col0 = cb * kBlockN + 64 * h;   // global index of column 0 of this half
        if (kKV) {
          const bool row_dead = row >= p.N;
          const bool diag = p.causal && cb == w.rb;
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (row_dead || (diag && col0 + i < row)) pv[i] = 0.f;
        } else {
          const int lim = p.causal ? min(row, p.N - 1) : p.N - 1;  // last allowed key
          if (col0 + 63 > lim) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (col0 + i > lim) pv[i] = 0.f;
          }
        }
      }
      if (kKV) {
        // P (bf16 pairs) over the first 32 of this half's score columns, for acc_p += P C1.
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pv[32 * ch + 2 * i], pv[32 * ch + 2 * i + 1]);
          tmem_st16(t_s + 16 * ch, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      s_par ^= 1u;
      // dS = P o (dP - delta) -> bf16 pairs over the first 32 of this half's dP columns.
      if (!(ok = wait_phase(dp_full, (uint32_t)it & 1u, abort_flag, kSiteBwdSoftDP))) break;
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dv[32];
        tmem_ld32(t_dp + 32 * ch, dv);
        tmem_ld_wait();
        reg_fence32(dv);
        uint32_t pk[16];
        if (kKV) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(vec + kBlockN + 32 * ch + i);
            const float e0 = pv[32 * ch + i] * (__uint_as_float(dv[i]) - d4.x);
            const float e1 = pv[32 * ch + i + 1] * (__uint_as_float(dv[i + 1]) - d4.y);
            const float e2 = pv[32 * ch + i + 2] * (__uint_as_float(dv[i + 2]) - d4.z);
            const float e3 = pv[32 * ch + i + 3] * (__uint_as_float(dv[i + 3]) - d4.w);
            pk[i / 2] = pack_bf16x2(e0, e1);
            pk[i / 2 + 1] = pack_bf16x2(e2, e3);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            pk[i / 2] = pack_bf16x2(pv[32 * ch + i] * (__uint_as_float(dv[i]) - row_delta),
                                    pv[32 * ch + i + 1] * (__uint_as_float(dv[i + 1]) - row_delta));
        }
        tmem_st16(t_dp + 16 * ch, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_ready);
      ring.advance<S>();
    }

    // Epilogue: this thread's row of acc_p / acc_ds, 32-column chunks alternating between
    // the two warpgroups, scaled (dK, dQ) and rounded to bf16.
    if (ok && w.n > 0 && wait_phase(acc_full, 0u, abort_flag, kSiteBwdSoftAcc)) {
      tc_fence_after();
      const bool row_ok = row < p.N;
      auto store_acc = [&](uint32_t col, float mul, __nv_bfloat16* out) {
        for (int ch = h; ch < D / 32; ch += 2) {
          uint32_t av[32];
          tmem_ld32(tmem_base + lane_off + col + 32 * ch, av);
          tmem_ld_wait();
          reg_fence32(av);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(av[2 * i]) * mul, __uint_as_float(av[2 * i + 1]) * mul);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)w.row_head * p.N + row) * D + 32 * ch);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      };
      if (kKV) {
        store_acc(256, 1.f, p.dv);
        store_acc(384, p.scale, p.dk);
      } else {
        store_acc(384, p.scale, p.dq);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace attn
