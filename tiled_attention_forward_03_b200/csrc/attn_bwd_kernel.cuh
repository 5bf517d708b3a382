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
//   attn_bwd_sm100<D, kKV = true>   units of one 128-key block of a KV head: keeps K_j, V_j
//                   in shared memory, streams the Q/dO tiles of every query head of the
//                   group, accumulates dV_j and dK_j in tensor memory
//   attn_bwd_sm100<D, kKV = false>  units of one 128-query block: keeps Q_i, dO_i, streams
//                   the K/V tiles, accumulates dQ_i in tensor memory
// Each unit owns its output rows outright, so there are no atomics and the result does
// not depend on the order units run in.
//
// Persistent CTAs (at most one per SM) walk the work items with a stride of the grid; an item
// is a unit or, causal with enough of them, a head's heaviest and lightest remaining blocks
// (equal items).  Between units the row tiles are reloaded once the last S and dP of the
// previous unit have read them (r_empty), the next unit's first S and dP run while the softmax
// warps store the previous unit's gradients, and the first accumulating MMAs wait until those
// are read (acc_free).  Per-tile barrier phases count the tiles of all units.  The price is that the score and dP tiles are
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
// Warp roles (384 threads, or 320 at D = 96):
//   warps 0-7  softmax: TMEM lane = tile row (warp % 4 picks the 32-lane slice), warps 0-3
//              take columns 0-63 and warps 4-7 columns 64-127 of each tile
//   warp  8    TMA producer
//   warp  9    MMA issuer (one elected lane)
//   warps 10-11 idle (complete the third warpgroup for the register split)
//
// Tensor memory (512 columns):
//   [  0,128) S fp32 (released to the next tile's S as soon as the softmax has loaded it)
//   [128,256) dP fp32; once loaded, each softmax warpgroup writes into its 64 columns
//             P (bf16 pairs, KV pass) over the first 32 and dS (bf16 pairs) over the second 32
//   [256,256+D) acc_p (dV);  [384,384+D) acc_ds (dK or dQ)
//   (D <= 64: a second dP buffer at [256,384), acc_p at [384,448), acc_ds at [448,512); dP
//   alternates between the buffers by tile parity)
// The two warpgroups never touch each other's columns.
//
// MMA order per column tile t (tcgen05 MMAs of one CTA run in issue order):
//   S(t+1)  acc_ds(t)  acc_p(t)  dP(t+1)
// S(t+1) is issued once the softmax holds S(t) in registers, so the exponentials of tile
// t+1 overlap all of tile t's gradient matmuls; dP(t+1) overwrites dS(t) and P(t) only
// after the MMAs reading them.  C0 and C1 tiles have rings of their own, each stage
// refilled as soon as its last reader has completed (C0 after acc_ds, C1 after acc_p, or
// after dP in the Q pass), so the next tiles are in flight while the current ones are used
// (D = 128: 2 + 2 stages in the KV pass, 3 + 2 in the Q pass; 4 + 4 at D <= 64).
//
// Every wait is bounded, as in the forward kernel.
#pragma once

#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"

namespace attn {

// Threads per CTA.  D = 32, 64, 128: three warpgroups (softmax warps 0-7, producer 8, MMA 9, idle
// 10-11) with the forward kernel's register split, the softmax warpgroups at kRegsSoftmax and the
// third at kRegsControl (launch: 384 x kRegsAtLaunch; removes the spills of a 320-thread CTA's
// 168-register ceiling; interleaved A/B +1 to +3 %).  D = 96 keeps 320 threads without the split
// (the split measured -7 % there).
template <int D>
struct BwdCfg {
  static constexpr bool kSplit = D != 96;
  static constexpr int kThreads = kSplit ? 384 : 320;
};
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= 384 * kRegsAtLaunch,
              "backward register split exceeds the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;
// Column pairs (of every 8) whose exponentials use the FMA-pipe polynomial (exp2_poly2)
// instead of the special-function unit.  Measured on B200 (interleaved A/B): at D = 64 the
// exponentials bound the block and 3 of 8 is best (+7 to +13 % against none; 4 of 8 is
// slower again), at D = 32 2 of 8 (+7 %); at D = 96 and 128 none (the polynomial's FMA work
// only delays P there).
template <int D, bool kKV>
__host__ __device__ constexpr int bwd_poly_pairs_per8() { return D <= 32 ? 2 : (D <= 64 ? 3 : 0); }

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

template <int D, bool kKV>
struct BwdPlan {
  static_assert(D == 32 || D == 64 || D == 96 || D == 128, "head dim must be 32, 64, 96 or 128");
  static constexpr int kChunks = (D + 63) / 64;
  static constexpr int kChunkBytes = kBlockM * 128;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // Ring depths of the C0 tiles (Q, or K in the Q pass; they are read first, by S, and last, by
  // acc_ds) and the C1 tiles (dO or V).  At D = 128 the Q pass, which needs no per-query
  // vectors, fits a third C0 stage (64 + 96 + 64 KB); the KV pass does not.
  static constexpr int kStages0 = (kChunks == 2) ? (kKV ? 2 : 3) : 4;
  static constexpr int kStages1 = (kChunks == 2) ? 2 : 4;
  static constexpr int kROff = 0;                                  // R0, R1
  static constexpr int kC0Off = 2 * kTileBytes;                    // C0 ring
  static constexpr int kC1Off = kC0Off + kStages0 * kTileBytes;    // C1 ring
  static constexpr int kVecBytes = kKV ? 2 * kBlockN * 4 : 0;      // per C0 stage: -lse2[128], -delta[128]
  static constexpr int kVecOff = kC1Off + kStages1 * kTileBytes;
  static constexpr int kBarOff = kVecOff + kStages0 * kVecBytes;
  // r_full c0_full[S0] c0_empty[S0] c1_full[S1] c1_empty[S1] s_full s_free dp_full[2] p_ready
  // ds_ready acc_full drain r_empty acc_free p_ready' ds_ready' (the last two: second dP buffer)
  static constexpr int kNumBars = 1 + 2 * kStages0 + 2 * kStages1 + 12;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

struct BwdParams {
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* nlse2;   // [B*Hq][Npad] -LSE * log2(e)
  const float* ndelta;  // [B*Hq][Npad] -rowsum(dO o O)
  int Hq, Hkv, N, Npad, group, num_blocks;
  int causal;
  float c;              // scale * log2(e)
  float scale;
  uint32_t idesc_s;     // 128 x 128 x D, both operands K-major
  uint32_t idesc_acc;   // 128 x D x 128, A from TMEM, B MN-major
  int pair;             // causal: an item is a row head's heaviest and lightest remaining row blocks
  int num_items;        // items of the pass being launched
};

// -delta_i = -sum_d dO_id O_id (fp32 sums of the bf16 products) and -lse2_i = -LSE_i log2(e)
// over the padded [B*Hq][Npad] layout (pad rows get 0); stored negated so that the kernels add
// them with paired fp32 instructions.  A 16-lane group takes kPrepRows consecutive rows (D <= 128:
// one 16-byte piece of O and of dO per lane and row) and issues all their loads before using
// any, to keep enough bytes in flight for HBM.
constexpr int kPrepRows = 4;
__global__ void attn_bwd_prep(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                              const float* __restrict__ lse, float* __restrict__ nlse2,
                              float* __restrict__ ndelta, long long rows, int N, int Npad, int D) {
  const long long row0 = ((long long)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4)) * kPrepRows;
  const int l16 = threadIdx.x & 15;
  if (row0 >= rows) return;  // whole 16-lane groups leave together (rows is a multiple of 128)
  uint4 a[kPrepRows], b[kPrepRows];
  bool live[kPrepRows];
#pragma unroll
  for (int k = 0; k < kPrepRows; ++k) {
    const long long row = row0 + k;
    const long long bh = row / Npad;
    const int qi = (int)(row - bh * Npad);
    live[k] = qi < N && l16 * 8 < D;
    a[k] = b[k] = make_uint4(0u, 0u, 0u, 0u);
    if (live[k]) {
      const size_t off = ((size_t)bh * N + qi) * D + l16 * 8;
      a[k] = *reinterpret_cast<const uint4*>(o + off);
      b[k] = *reinterpret_cast<const uint4*>(dout + off);
    }
  }
  const unsigned mask = 0xffffu << (threadIdx.x & 16);
#pragma unroll
  for (int k = 0; k < kPrepRows; ++k) {
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[k]);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b[k]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(pa[e]);
      const float2 fb = __bfloat1622float2(pb[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
    acc += __shfl_xor_sync(mask, acc, 8, 16);
    acc += __shfl_xor_sync(mask, acc, 4, 16);
    acc += __shfl_xor_sync(mask, acc, 2, 16);
    acc += __shfl_xor_sync(mask, acc, 1, 16);
    if (l16 == k) {
      const long long row = row0 + k;
      const long long bh = row / Npad;
      const int qi = (int)(row - bh * Npad);
      ndelta[row] = -acc;
      nlse2[row] = qi < N ? -lse[(size_t)bh * N + qi] * kLog2e : 0.f;
    }
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

// Unit `which` (0 or 1) of work item `item`; false if the item has no such unit.  Items are
// numbered row head by row head; a causal item pairs the heaviest and the lightest remaining
// row blocks of a head (equal items) when p.pair is set, else an item is one row block,
// heaviest first.
template <bool kKV>
__device__ __forceinline__ bool bwd_unit(const BwdParams& p, int item, int which, BwdUnit& w) {
  const int nb = p.num_blocks;
  int k;
  if (p.pair) {
    const int sph = (nb + 1) >> 1;
    w.row_head = item / sph;
    const int s = item - w.row_head * sph;
    if (which == 1 && s >= nb - 1 - s) return false;
    k = which ? nb - 1 - s : s;   // k = 0 is the heaviest block in both passes
  } else {
    if (which) return false;
    w.row_head = item / nb;
    k = item - w.row_head * nb;
  }
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
  return true;
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
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    attn_bwd_sm100(const __grid_constant__ CUtensorMap tmap_r0, const __grid_constant__ CUtensorMap tmap_r1,
                   const __grid_constant__ CUtensorMap tmap_c0, const __grid_constant__ CUtensorMap tmap_c1,
                   const BwdParams p) {
  using Plan = BwdPlan<D, kKV>;
  constexpr int S0 = Plan::kStages0;
  constexpr int S1 = Plan::kStages1;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sR = smem + Plan::kROff;
  uint8_t* sC0 = smem + Plan::kC0Off;
  uint8_t* sC1 = smem + Plan::kC1Off;
  float* sVec = reinterpret_cast<float*>(smem + Plan::kVecOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint64_t* r_full = bars;
  uint64_t* c0_full = bars + 1;
  uint64_t* c0_empty = c0_full + S0;
  uint64_t* c1_full = c0_full + 2 * S0;
  uint64_t* c1_empty = c1_full + S1;
  uint64_t* s_full = c1_full + 2 * S1;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_full + 2;   // [2]: one per dP buffer ([0] only at D = 128)
  uint64_t* p_ready = s_full + 4;
  uint64_t* ds_ready = s_full + 5;
  uint64_t* acc_full = s_full + 6;
  uint64_t* drain = s_full + 7;
  uint64_t* r_empty = s_full + 8;    // the unit's last S and dP have read R0, R1
  uint64_t* acc_free = s_full + 9;   // the epilogue has read the accumulators (256 arrivals)
  // At D <= 64 tensor memory has room for a second dP buffer (S 128 + dP 2 x 128 + two
  // accumulators of D <= 64 columns): dP(t+1) then goes into the other buffer as soon as S(t+1)
  // is issued, instead of waiting for the MMAs that read P(t) and dS(t).
  constexpr bool kDualDP = D <= 64;
  constexpr uint32_t kAccP = kDualDP ? 384u : 256u;            // acc_p (dV) column
  constexpr uint32_t kAccDS = kDualDP ? 384u + 64u : 384u;     // acc_ds (dK or dQ) column
  auto dp_col = [](int t) -> uint32_t { return 128u + (kDualDP ? 128u * (uint32_t)(t & 1) : 0u); };
  auto dp_bar = [](int t) -> int { return kDualDP ? (t & 1) : 0; };
  auto dp_par = [](int t) -> uint32_t { return kDualDP ? (((uint32_t)t >> 1) & 1u) : ((uint32_t)t & 1u); };
  // dS and P of tile t are ready: one barrier per dP buffer, like dp_full.  With two buffers the
  // softmax can finish tile t+1 (its S and dP are issued early) before the MMA warp has waited for
  // tile t; a single barrier would then complete twice and its parity wait for t would stall.
  auto ds_ready_bar = [&](int t) -> uint64_t* { return (kDualDP && (t & 1)) ? s_full + 11 : s_full + 5; };
  auto p_ready_bar = [&](int t) -> uint64_t* { return (kDualDP && (t & 1)) ? s_full + 10 : s_full + 4; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Plan::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(r_full, 1);
    for (int i = 0; i < S0; ++i) {
      mbar_init(&c0_full[i], 1);
      mbar_init(&c0_empty[i], 1);
    }
    for (int i = 0; i < S1; ++i) {
      mbar_init(&c1_full[i], 1);
      mbar_init(&c1_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(&dp_full[0], 1);
    mbar_init(&dp_full[1], 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(s_full + 10, 256);
    mbar_init(s_full + 11, 256);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(r_empty, 1);
    mbar_init(acc_free, 256);
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
    if constexpr (BwdCfg<D>::kSplit) regs_decrease<kRegsControl>();
    // Two rings of S stages: C0 tiles (with the KV pass's per-query vectors) and C1 tiles,
    // each refilled as soon as the MMAs that read it have completed.
    if (lane == 0) {
      const uint64_t pol_once = l2_policy_evict_first();
      const uint64_t pol_shared = l2_policy_evict_last();
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row, int head, uint64_t pol) {
#pragma unroll
        for (int ch = 0; ch < Plan::kChunks; ++ch)
          tma_load_3d(dst + ch * Plan::kChunkBytes, map, bar, ch * 64, row, head, pol);
      };
      Ring r0, r1;
      uint32_t filled0 = 0u, par0 = 0u, filled1 = 0u, par1 = 0u;  // per stage: ever filled / parity of last fill
      uint32_t units = 0u;
      bool ok = true;
      for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x)
      for (int which = 0; which < 2 && ok; ++which) {
      BwdUnit w;
      if (!bwd_unit<kKV>(p, item, which, w)) continue;
      // the row tiles once the previous unit's last S and dP have read them
      if (units > 0u && !(ok = wait_phase(r_empty, (units - 1u) & 1u, abort_flag, kSiteBwdProducer))) break;
      mbar_arrive_expect_tx(r_full, 2 * Plan::kTileBytes);
      load_tile(&tmap_r0, sR, r_full, w.rb * kBlockM, w.row_head, pol_once);
      load_tile(&tmap_r1, sR + Plan::kTileBytes, r_full, w.rb * kBlockM, w.row_head, pol_once);
      ++units;
      for (int it = 0; it < w.n; ++it) {
        int cb, chead;
        bwd_col<kKV>(p, w, it, cb, chead);
        if (!(ok = wait_phase(&c0_empty[r0.stage], r0.phase ^ 1u, abort_flag, kSiteBwdProducer))) break;
        uint64_t* bar0 = &c0_full[r0.stage];
        mbar_arrive_expect_tx(bar0, Plan::kTileBytes + Plan::kVecBytes);
        load_tile(&tmap_c0, sC0 + r0.stage * Plan::kTileBytes, bar0, cb * kBlockN, chead, pol_shared);
        if (kKV) {
          const size_t off = (size_t)chead * p.Npad + (size_t)cb * kBlockN;
          float* vec = sVec + r0.stage * 2 * kBlockN;
          bulk_load_1d(vec, p.nlse2 + off, kBlockN * 4, bar0);
          bulk_load_1d(vec + kBlockN, p.ndelta + off, kBlockN * 4, bar0);
        }
        filled0 |= 1u << r0.stage;
        par0 = (par0 & ~(1u << r0.stage)) | (r0.phase << r0.stage);
        r0.advance<S0>();
        if (!(ok = wait_phase(&c1_empty[r1.stage], r1.phase ^ 1u, abort_flag, kSiteBwdProducer))) break;
        uint64_t* bar1 = &c1_full[r1.stage];
        mbar_arrive_expect_tx(bar1, Plan::kTileBytes);
        load_tile(&tmap_c1, sC1 + r1.stage * Plan::kTileBytes, bar1, cb * kBlockN, chead, pol_shared);
        filled1 |= 1u << r1.stage;
        par1 = (par1 & ~(1u << r1.stage)) | (r1.phase << r1.stage);
        r1.advance<S1>();
      }
      }
      // Drain: every issued copy lands before the CTA may exit.
      if (units > 0u) drain_phase(r_full, (units - 1u) & 1u, abort_flag);
      for (int s = 0; s < S0; ++s)
        if (filled0 & (1u << s)) drain_phase(&c0_full[s], (par0 >> s) & 1u, abort_flag);
      for (int s = 0; s < S1; ++s)
        if (filled1 & (1u << s)) drain_phase(&c1_full[s], (par1 >> s) & 1u, abort_flag);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (BwdCfg<D>::kSplit) regs_decrease<kRegsControl>();
    // Per column tile t (tcgen05 MMAs of one CTA run in issue order):
    //   S(t+1) once the softmax has S(t) in registers;
    //   acc_ds(t) once dS(t) is in TMEM, then C0(t) is released;
    //   acc_p(t) (KV pass) once P(t) is in TMEM, then C1(t) is released;
    //   dP(t+1), which overwrites the dP columns holding dS(t) and P(t).
    // The Q pass releases C1(t) as soon as dP(t) has completed (its only reader).
    const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
    const uint64_t desc_r0 = smem_desc_kmajor_sw128(smem_u32(sR));
    const uint64_t desc_r1 = smem_desc_kmajor_sw128(smem_u32(sR + Plan::kTileBytes));
    const uint64_t desc_c0_k = smem_desc_kmajor_sw128(smem_u32(sC0));
    const uint64_t desc_c1_k = smem_desc_kmajor_sw128(smem_u32(sC1));
    const uint64_t desc_c0_mn = smem_desc_mnmajor_sw128(smem_u32(sC0), Plan::kChunkBytes);
    const uint64_t desc_c1_mn = smem_desc_mnmajor_sw128(smem_u32(sC1), Plan::kChunkBytes);
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
    // acc (+)= X C over the 128 tile columns: X bf16 pairs in TMEM at columns a_col + [0,32)
    // (tile columns 0-63) and a_col + 64 + [0,32) (tile columns 64-127); C MN-major in smem.
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
    auto st_bytes = [](uint32_t st) -> uint32_t { return st * Plan::kTileBytes; };

    Ring r0, r1;  // ring positions of the current tile's C0 and C1
    uint32_t T = 0u;      // column tiles of earlier units: tile it of this unit is T + it
    uint32_t units = 0u;
    bool ok = true;
    for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x)
    for (int which = 0; which < 2 && ok; ++which) {
    BwdUnit w;
    if (!bwd_unit<kKV>(p, item, which, w)) continue;
    if (!(ok = wait_all(r_full, units & 1u, kSiteBwdMmaRow))) break;
    // First tile's S and dP.  S's columns were read by the softmax (s_free of the previous unit's
    // last tile was waited for); dP's buffer was last read by MMAs issued before these.
    if (!(ok = wait_all(&c0_full[r0.stage], r0.phase, kSiteBwdMmaCol))) break;
    tc_fence_after();
    issue_rc(0, desc_r0, adv(desc_c0_k, st_bytes(r0.stage)));
    commit(s_full);
    if (!(ok = wait_all(&c1_full[r1.stage], r1.phase, kSiteBwdMmaCol))) break;
    tc_fence_after();
    issue_rc(dp_col((int)T), desc_r1, adv(desc_c1_k, st_bytes(r1.stage)));
    commit(&dp_full[dp_bar((int)T)]);
    if (!kKV) commit(&c1_empty[r1.stage]);
    if (w.n == 1) commit(r_empty);
    for (int it = 0; it < w.n && ok; ++it) {
      const int t = (int)T + it;          // tile index over all units (barrier phases)
      const uint32_t par = (uint32_t)t & 1u;
      Ring n0 = r0, n1 = r1;  // the next tile's
      n0.advance<S0>();
      n1.advance<S1>();
      const bool has_next = it + 1 < w.n;
      if (!(ok = wait_all(s_free, par, kSiteBwdMmaP))) break;
      if (has_next) {
        if (!(ok = wait_all(&c0_full[n0.stage], n0.phase, kSiteBwdMmaCol))) break;
        tc_fence_after();
        issue_rc(0, desc_r0, adv(desc_c0_k, st_bytes(n0.stage)));
        commit(s_full);
        if (kDualDP) {
          // dP(t+1) into the other buffer, whose P(t-1) / dS(t-1) the previous MMAs have read
          if (!(ok = wait_all(&c1_full[n1.stage], n1.phase, kSiteBwdMmaCol))) break;
          tc_fence_after();
          issue_rc(dp_col(t + 1), desc_r1, adv(desc_c1_k, st_bytes(n1.stage)));
          commit(&dp_full[dp_bar(t + 1)]);
          if (!kKV) commit(&c1_empty[n1.stage]);
          if (it + 2 == w.n) commit(r_empty);
        }
      }
      // the first accumulating MMAs of a unit overwrite the accumulators: the previous unit's
      // epilogue must have read them
      if (it == 0 && units > 0u && !(ok = wait_all(acc_free, (units - 1u) & 1u, kSiteBwdMmaDS))) break;
      if (!(ok = wait_all(ds_ready_bar(t), dp_par(t), kSiteBwdMmaDS))) break;
      tc_fence_after();
      issue_acc(kAccDS, dp_col(t) + 32, adv(desc_c0_mn, st_bytes(r0.stage)), it > 0);
      commit(&c0_empty[r0.stage]);
      if (kKV) {
        if (!(ok = wait_all(p_ready_bar(t), dp_par(t), kSiteBwdMmaP))) break;
        tc_fence_after();
        issue_acc(kAccP, dp_col(t), adv(desc_c1_mn, st_bytes(r1.stage)), it > 0);
        commit(&c1_empty[r1.stage]);
      }
      if (!kDualDP && has_next) {
        if (!(ok = wait_all(&c1_full[n1.stage], n1.phase, kSiteBwdMmaCol))) break;
        tc_fence_after();
        issue_rc(128, desc_r1, adv(desc_c1_k, st_bytes(n1.stage)));
        commit(&dp_full[0]);
        if (!kKV) commit(&c1_empty[n1.stage]);
        if (it + 2 == w.n) commit(r_empty);
      }
      r0 = n0;
      r1 = n1;
    }
    if (!ok) break;
    commit(acc_full);
    T += (uint32_t)w.n;
    ++units;
    }
    // Drain: all MMAs issued by this warp complete before TMEM is released.
    commit(drain);
    drain_phase(drain, 0u, abort_flag);
    __syncwarp();
  } else if (warp >= 10) {
    // idle: completes the third warpgroup, whose registers go to the softmax warps
    if constexpr (BwdCfg<D>::kSplit) regs_decrease<kRegsControl>();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    if constexpr (BwdCfg<D>::kSplit) regs_increase<kRegsSoftmax>();
    const int r = threadIdx.x & 127;            // tile row == TMEM lane
    const int h = warp >> 2;                    // column half
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + 64 * h;
    const uint32_t t_dp0 = tmem_base + lane_off + 64 * h;   // + dp_col(t): this thread's dP columns
    const float c = p.c;
    bool ok = true;
    Ring ring;  // position of the current tile's C0 (and per-query vectors)
    // bits 0-1: column tiles of earlier units mod 4 (the per-tile barrier phases need no more);
    // bit 2: earlier units mod 2 (the accumulator barrier's phase)
    uint32_t st = 0u;
    for (int q = 0; ok; ++q) {
    const int item = (int)blockIdx.x + (q >> 1) * (int)gridDim.x;
    if (item >= p.num_items) break;
    BwdUnit w;
    if (!bwd_unit<kKV>(p, item, q & 1, w)) continue;
    const int row = w.rb * kBlockM + r;         // global index of this thread's tile row
    // Q pass: the row's -lse2 and -delta are fixed for the whole unit.
    float row_nlse2 = 0.f, row_ndelta = 0.f;
    if (!kKV) {
      const size_t off = (size_t)w.row_head * p.Npad + row;
      row_nlse2 = p.nlse2[off];
      row_ndelta = p.ndelta[off];
    }
    int cb = w.c0;                              // column block of the current tile
    for (int it0 = 0; it0 < w.n && ok; ++it0) {
      const int it = (int)(st & 3u) + it0;      // tile index over all units, mod 4 (barrier phases)
      const uint32_t par = (uint32_t)it & 1u;
      const float* vec = sVec + ring.stage * 2 * kBlockN + 64 * h;
      if (!(ok = wait_phase(s_full, par, abort_flag, kSiteBwdSoftS))) break;
      if (kKV && !(ok = wait_phase(&c0_full[ring.stage], ring.phase, abort_flag, kSiteBwdSoftS))) break;
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
      // The scores are in registers: the next tile's S may overwrite them now.
      tc_fence_before();
      mbar_arrive(s_free);
      // P = 2^(S c - lse2), lse2 of the column's query in the KV pass, of the row's otherwise;
      // the workspace holds -lse2.  Column pairs (of every 8) below the polynomial share take
      // the FMA-pipe exponential instead of the special-function unit.
      {
        const float2 c2 = make_float2(c, c);
        auto exp_pair = [&](int i, float2 nl) {
          const float2 x = fma2(make_float2(pv[i], pv[i + 1]), c2, nl);
          float2 e;
          if (((i >> 1) & 7) < bwd_poly_pairs_per8<D, kKV>()) {
            e = exp2_poly2(x);
          } else {
            e.x = ex2_approx(x.x);
            e.y = ex2_approx(x.y);
          }
          pv[i] = e.x;
          pv[i + 1] = e.y;
        };
        if (kKV) {
#pragma unroll
          for (int i = 0; i < 64; i += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(vec + i);
            exp_pair(i, make_float2(l4.x, l4.y));
            exp_pair(i + 2, make_float2(l4.z, l4.w));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 64; i += 2) exp_pair(i, make_float2(row_nlse2, row_nlse2));
        }
      }
      // Masks.  KV pass: row = key, column = query; the causal mask hides query < key
      // (diagonal block only), and key rows past N are zeroed.  Q pass: row = query,
      // column = key; the mask hides key > query and keys past N.
      {
        const int col0 = cb * kBlockN + 64 * h;   // global index of column 0 of this half
        if (kKV) {
          const bool row_dead = row >= p.N;
          const bool diag = p.causal && cb == w.rb;
          if (row_dead || diag) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (row_dead || col0 + i < row) pv[i] = 0.f;
          }
        } else {
          const int lim = p.causal ? min(row, p.N - 1) : p.N - 1;  // last allowed key
          if (col0 + 63 > lim) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (col0 + i > lim) pv[i] = 0.f;
          }
        }
      }
      // dS = P o (dP - delta) (the workspace holds -delta), as bf16 pairs over the second 32
      // of this half's dP columns; then (KV pass) P as bf16 pairs over the first 32.
      if (!(ok = wait_phase(&dp_full[dp_bar(it)], dp_par(it), abort_flag, kSiteBwdSoftDP))) break;
      tc_fence_after();
      const uint32_t t_dp = t_dp0 + dp_col(it);
      {
        uint32_t d0[32], d1[32];
        tmem_ld32(t_dp, d0);
        tmem_ld32(t_dp + 32, d1);
        tmem_ld_wait();
        reg_fence32(d0);
        reg_fence32(d1);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const uint32_t* dv = ch ? d1 : d0;
            float4 n4;
            if (kKV) {
              n4 = *reinterpret_cast<const float4*>(vec + kBlockN + 32 * ch + i);
            } else {
              n4 = make_float4(row_ndelta, row_ndelta, row_ndelta, row_ndelta);
            }
            const float2 e0 = mul2(make_float2(pv[32 * ch + i], pv[32 * ch + i + 1]),
                                   add2(make_float2(__uint_as_float(dv[i]), __uint_as_float(dv[i + 1])),
                                        make_float2(n4.x, n4.y)));
            const float2 e1 = mul2(make_float2(pv[32 * ch + i + 2], pv[32 * ch + i + 3]),
                                   add2(make_float2(__uint_as_float(dv[i + 2]), __uint_as_float(dv[i + 3])),
                                        make_float2(n4.z, n4.w)));
            pk[i / 2] = pack_bf16x2(e0.x, e0.y);
            pk[i / 2 + 1] = pack_bf16x2(e1.x, e1.y);
          }
          tmem_st16(t_dp + 32 + 16 * ch, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_ready_bar(it));
      if (kKV) {
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pv[32 * ch + 2 * i], pv[32 * ch + 2 * i + 1]);
          tmem_st16(t_dp + 16 * ch, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_ready_bar(it));
      }
      ring.advance<S0>();
      if (++cb == p.num_blocks) cb = w.c0;     // the next query head of the group (KV pass)
    }

    if (!ok) break;
    // Epilogue: this thread's row of acc_p / acc_ds, 32-column chunks alternating between
    // the two warpgroups, scaled (dK, dQ) and rounded to bf16.
    if (!(ok = wait_phase(acc_full, (st >> 2) & 1u, abort_flag, kSiteBwdSoftAcc))) break;
    {
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
        store_acc(kAccP, 1.f, p.dv);
        store_acc(kAccDS, p.scale, p.dk);
      } else {
        store_acc(kAccDS, p.scale, p.dq);
      }
      // the accumulators are read: the next unit's first accumulating MMAs may overwrite them
      tc_fence_before();
      mbar_arrive(acc_free);
    }
    st = ((st + (uint32_t)w.n) & 3u) | ((st ^ 4u) & 4u);
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
