// attn_fwd_kernel.cuh -- tiled attention forward for B200 (sm_100a).
//
// Method: the tiled attention forward with an online (running max / running sum)
// softmax whose hot loop is a score matmul, a base-2 exponential and row sums,
// followed by the probability-times-V matmul ("Making AMD GPUs go brrr", section
// "Real kernel example"; "HipKittens: fast and furious AMD kernels", section
// "Performance results": causal and non-causal, several D and N).  The pages'
// AMD schedule (two wave groups alternating memory and compute clusters) becomes,
// on sm_100a, warp specialisation with two Q tiles ping-ponging on the tensor core:
//
//   warps 0-3  softmax warpgroup for Q tile 0 (one TMEM lane = one query row per thread)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp  8    TMA producer: Q tiles once per unit, K_j / V_j through a smem ring
//   warp  9    MMA issuer (one elected lane): S_t = Q_t K_j^T and O_t += P_t V_j on tcgen05
//   warp  10   output store (D = 128): TMA tensor stores of each tile's O, staged in shared memory
//   warp  11   idle (completes the third warpgroup, which gives up registers)
//
// Non-causal bf16 D <= 64 (kSepP): P gets tensor-memory columns of its own beside O, and each
// tile has its own MMA warp (warp 9: tile 0, warp 11: tile 1), which issues the tile's next S as
// soon as its softmax has read the current one, so S no longer waits for the P V before it.
//
// A work unit is 256 query rows (two 128-row tiles) of one query head; a persistent
// grid walks the units with a static stride.  Units of one head are adjacent (and
// the heads of one GQA group are adjacent) so K/V blocks are re-read from L2; in the
// causal case a head's units run heaviest first.
//
// Tensor memory (512 columns of 128 lanes x 32 bit):
//   [  0,128) S_0 fp32 scores of tile 0; its first 64 columns are overwritten by P_0 (bf16x2)
//   [128,256) S_1 / P_1
//   [256,256+D) O_0 fp32 accumulator;  [384,384+D) O_1
//   kSepP (D <= 64): P_0 at [320,384) and P_1 at [448,512) instead of over the scores
//
// Online softmax in base 2 with c = |scale| * log2(e):  m = running max of s*c,
// p = 2^(s*c - m), l = sum p.  The max is applied lazily: O and l are rescaled only
// when a row's max grows by more than RESCALE_LOG2 (so p <= 2^RESCALE_LOG2); the final
// O / l and LSE = (m + log2 l) * ln 2 use the same m, so the result is unchanged.
//
// Every mbarrier wait is bounded: on timeout the CTA records a site code in
// g_attn_fault_site, all roles leave their loops, in-flight copies and MMAs are
// drained (bounded again), TMEM is freed and the kernel returns.
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace attn {

constexpr int kThreads = 384;  // three warpgroups
// Register split (launch: 384 x 168): softmax warpgroups 2 x 128 x 224, the
// producer/MMA warpgroup 128 x 56; 2*128*224 + 128*56 == 384*168.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsSoftmax = 224;
constexpr int kRegsControl = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr int kBlockM = 128;  // query rows per tile
constexpr int kBlockN = 128;  // keys per KV block
constexpr float kRescaleLog2 = 8.0f;
// Column pairs (of every 8) whose exponentials use the FMA-pipe polynomial instead of the
// special-function unit, measured best on B200 (interleaved A/B; more polynomial work costs
// issue slots that the MMA-issuing warp shares with the softmax warps): bf16 2 at D = 128 and
// 64, 3 at D = 96 and 32 (+3 to +6 % against 1 there); 2 in the separate-P form (both softmax
// warpgroups busy back to back; 3 was slower); E4M3 2 at D = 128 and 3 at D = 64, whose halved
// tensor work leaves the exponentials the limit (+4 to +12 % against 1).
template <int D, bool kF8 = false, bool kSepP = false>
__host__ __device__ constexpr int poly_pairs_per8() {
  return kF8 ? (D == 128 ? 2 : 3) : (kSepP ? 2 : ((D == 128 || D == 64) ? 2 : 3));
}
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s for any single wait

// Fault-site codes written to g_attn_fault_site when a bounded wait gives up.
enum : unsigned {
  kSiteProducerQ = 1,
  kSiteProducerKV = 2,
  kSiteMmaQ = 3,
  kSiteMmaKV = 4,
  kSiteMmaP = 5,
  kSiteMmaOFree = 6,
  kSiteSoftmaxS = 7,
  kSiteSoftmaxO = 8,
  kSiteDrain = 9,
  kSiteSelfTest = 10,
  kSiteSplitMerge = 11,
  kSiteStore = 25,      // the store warp waiting for a staged O tile
  kSiteStageFree = 26,  // a softmax warpgroup waiting for the staging buffer
  kSitePFree = 27,      // kSepP: a softmax warpgroup waiting for the last P V to have read P
  kSiteMmaSFree = 28,   // kSepP: an MMA warp waiting for the softmax to have read S
};

__device__ unsigned int g_attn_fault_site = 0;

// kF8: Q, K, V are E4M3 bytes (one 128-byte swizzle chunk holds 128 columns) instead of bf16.
template <int D, bool kF8 = false, bool kSepP = false>
struct SmemPlan {
  static_assert(D == 32 || D == 64 || D == 96 || D == 128, "head dim must be 32, 64, 96 or 128");
  static constexpr int kElemBytes = kF8 ? 1 : 2;
  static constexpr int kRowElems = 128 / kElemBytes;        // columns per 128-byte swizzle row
  static constexpr int kChunks = (D + kRowElems - 1) / kRowElems;  // 128-byte swizzle chunks per row
  static constexpr int kChunkBytes = kBlockM * 128;         // one chunk of a tile: 16 KB
  // one 128-row tile; a partly used last chunk (D = 32, 96) is zero-filled by TMA
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (kChunks == 2) ? 4 : 8;    // K/V ring depth
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  // D = 128, and bf16 D = 64 in the separate-P form: one tile's O (bf16) staged for the TMA
  // store: 64-column chunks of 128-byte rows, 128-byte swizzle, the two tiles using it in turn
  // (measured against 16-byte stores from the softmax warps: 1-3 % faster for bf16 and 5-8 % for
  // E4M3 inputs at D = 128, 1-4 % in the separate-P form; 6-10 % slower for the bf16 D = 64 form
  // with P in S, where the softmax warps bound the kernel, and up to 7 % slower for E4M3 at D = 64;
  // the other instances store O directly)
  static constexpr bool kStagedStore = D == 128 || (D == 64 && kSepP && !kF8);
  static constexpr int kOChunks = (D + 63) / 64;
  static constexpr int kOStageOff = kKVOff + kStages * kTileBytes;
  static constexpr int kBarOff = kOStageOff + (kStagedStore ? kOChunks * kChunkBytes : 0);
  // barriers: q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] o_free[2] drain
  // o_staged stage_free s_free[2] p_free[2] (the last four used by the separate-P form only)
  static constexpr int kNumBars = 4 + 2 * kStages + 8 + 1 + 2 + 4;
  // tmem base (u32), abort flag (u32), per-tile "last range" flags (2 x u32)
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;              // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "forward shared memory plan exceeds 227 KB");
};

// Division by a divisor fixed for the launch, as a multiply-high by a precomputed reciprocal
// (T. Granlund and P. L. Montgomery, "Division by invariant integers using multiplication",
// PLDI 1994): with m = ceil(2^64 / d), floor(n / d) is the high 64 bits of n * m for every
// n < 2^32 and 2 <= d < 2^32, since n * m / 2^64 = n / d + n * (m - 2^64 / d) / 2^64 and the
// second term is below 2^-32 <= 1 / d.  m = 0 stands for d = 1.  The scheduler evaluates
// its work items with these: on the MMA warp a new unit waits for that arithmetic, where a
// 64-bit division costs hundreds of cycles.
struct FastDiv {
  unsigned long long m;
  uint32_t d;
};

inline FastDiv make_fast_div(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.m = d > 1u ? ~0ull / d + 1ull : 0ull;
  return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
  return f.m ? (uint32_t)__umul64hi((unsigned long long)n, f.m) : n;
}

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int Hq, Hkv, N;
  int group;         // Hq / Hkv
  int num_pairs;     // ceil(N / 256): units per head
  int num_blocks;    // ceil(N / 128): KV blocks per head
  long long num_units;
  long long num_steps;  // scheduling steps walked by the persistent grid
  int units_per_step;   // 1 (non-causal) or 2 (causal: heaviest + lightest pair of a head)
  int causal;
  // Split tail (non-causal): every CTA first runs `whole_per_cta` whole units; the
  // `tail_units` units of the last, partial wave are each split into `parts` (= 2) KV
  // ranges, one per CTA.  parts == 1: no split, whole units round robin until num_units.
  int whole_per_cta;
  int tail_units;
  int parts;
  float* ws_o;        // first range's O rows [tail_units][2 tiles][D/4][128 rows] float4
  float* ws_ml;       // first range's (m, l) [tail_units][2 tiles][128 rows] float2
  unsigned* ws_cnt;   // [tail_units][2 tiles][2]: finished ranges ((epoch << 8) | count), ready flag (epoch)
  unsigned epoch;     // launch tag (24 bits, non-zero): counts of other launches read as 0
  // divisors of the schedule (all counts below 2^31: checked on the host)
  FastDiv div_pairs;  // num_pairs
  FastDiv div_steps;  // (num_pairs + 1) / 2: causal scheduling steps per head
  FastDiv div_hq;     // Hq
  FastDiv div_group;  // group
  // Causal with an even GQA group: a unit is one 128-row query tile of two query heads that
  // share a KV head (tile 0 head h, tile 1 head h + 1, the same rows), so both tiles see the same
  // KV blocks.  num_pairs is then the query-tile count and the "head" of a step is a head pair.
  int head_pairs;
  FastDiv div_hq2;    // Hq / 2
  float c;           // |scale| * log2(e) (times the Q and K descales for E4M3 inputs)
  float o_scale;     // multiplies the normalised output (the V descale for E4M3 inputs, else 1)
  uint32_t idesc_s;  // S = Q K^T instruction descriptor (negates A when scale < 0)
  uint32_t idesc_pv; // O += P V instruction descriptor
};

struct Unit {
  int q0;          // first query row of tile 0
  int head_q;      // b * Hq + hq (tile 0)
  int row1;        // first query row of tile 1
  int head_q1;     // query head of tile 1
  int head_kv;     // b * Hkv + hq / group
  int jb;          // first KV block of this work item (0 unless the unit is split)
  int n0, n1;      // end (exclusive) of the KV blocks visited by tile 0 / tile 1
  bool valid1;     // tile 1 holds at least one row < N
  int nmax;
  int parts;       // KV ranges the unit is split into (1: whole unit)
  int part;        // which range this item is
  int tail;        // index of the split unit among the tail units
};

__device__ __forceinline__ Unit make_unit(const FwdParams& p, uint32_t head, int pair) {
  Unit w;
  const uint32_t b = fast_div(head, p.div_hq);
  const uint32_t hq = head - b * (uint32_t)p.Hq;
  w.q0 = pair * 2 * kBlockM;
  w.head_q = (int)head;
  w.head_kv = (int)(b * (uint32_t)p.Hkv + fast_div(hq, p.div_group));
  w.valid1 = (w.q0 + kBlockM) < p.N;
  w.row1 = w.q0 + kBlockM;
  w.head_q1 = (int)head;
  if (p.causal) {
    w.n0 = min(p.num_blocks, 2 * pair + 1);
    w.n1 = min(p.num_blocks, 2 * pair + 2);
  } else {
    w.n0 = p.num_blocks;
    w.n1 = p.num_blocks;
  }
  w.nmax = w.valid1 ? w.n1 : w.n0;
  w.jb = 0;
  w.parts = 1;
  w.part = 0;
  w.tail = 0;
  return w;
}

// Unit `part` of scheduling step `step`.  Non-causal: one unit per step, the pairs of
// a head in order.  Causal: the work of pair j grows linearly with j, so step s of a
// head holds its pair P-1-s (heaviest first) and pair s; every step then costs the
// same and a static stride over steps balances the grid.  Consecutive steps stay in
// one head (and the heads of one GQA group are consecutive), so K/V tiles are shared
// through L2 by the CTAs running at the same time.  Returns false if the step has no
// such unit (the middle pair of a head with an odd pair count).
// Head-pair unit (causal, even GQA group): query tile `tile` of heads 2hp and 2hp + 1 of batch b.
__device__ __forceinline__ Unit make_unit_hp(const FwdParams& p, uint32_t slot, int tile) {
  Unit w;
  const uint32_t b = fast_div(slot, p.div_hq2);
  const uint32_t hq0 = 2u * (slot - b * p.div_hq2.d);
  w.q0 = tile * kBlockM;
  w.row1 = w.q0;
  w.head_q = (int)(b * (uint32_t)p.Hq + hq0);
  w.head_q1 = w.head_q + 1;
  w.head_kv = (int)(b * (uint32_t)p.Hkv + fast_div(hq0, p.div_group));
  w.valid1 = true;
  w.n0 = w.n1 = w.nmax = min(p.num_blocks, tile + 1);
  w.jb = 0;
  w.parts = 1;
  w.part = 0;
  w.tail = 0;
  return w;
}

__device__ __forceinline__ bool unit_at(const FwdParams& p, uint32_t step, int part, Unit& w) {
  if (!p.causal) {
    const uint32_t head = fast_div(step, p.div_pairs);
    w = make_unit(p, head, (int)(step - head * (uint32_t)p.num_pairs));
    return true;
  }
  const uint32_t head = fast_div(step, p.div_steps);
  const int s = (int)(step - head * p.div_steps.d);
  const int pair = part == 0 ? p.num_pairs - 1 - s : s;
  if (part == 1 && pair == p.num_pairs - 1 - s) return false;
  w = p.head_pairs ? make_unit_hp(p, head, pair) : make_unit(p, head, pair);
  return true;
}

// Counts one finished KV range of a split unit and returns how many had finished before
// it in this launch.  The word holds (epoch << 8) | count; a word left by another launch
// (different epoch) counts as zero, so the workspace never needs clearing.  The merging
// range zeroes the words once it has read them, so a launch that completes leaves none
// behind: the epoch then guards against fresh memory and launches that gave up, and the
// 24-bit epoch wrapping round, or another copy of the library sharing the workspace, cannot
// make a stale word look current.  Each failed compare-and-swap means another range's
// update succeeded, so the loop ends after at most `parts` attempts.
__device__ __forceinline__ unsigned count_finished(unsigned* cnt, unsigned epoch) {
  unsigned old = atomicAdd(cnt, 0u);
  while (true) {
    const unsigned before = ((old >> 8) == epoch) ? (old & 255u) : 0u;
    const unsigned prev = atomicCAS(cnt, old, (epoch << 8) | (before + 1u));
    if (prev == old) return before;
    old = prev;
  }
}

// Work item `it` of this CTA.  Returns 0 when the CTA has no more items, 1 for an item
// in `w`, 2 for an empty slot (causal: the middle pair of a head with an odd pair count).
// Causal: two units per step (see unit_at), steps round robin.  Non-causal: whole units
// round robin; with a split tail, each CTA then runs at most one KV range of one of the
// last wave's units (ranges of a unit go to adjacent CTAs).
__device__ __forceinline__ int item_at(const FwdParams& p, int it, Unit& w) {
  if (p.causal) {
    const long long step = blockIdx.x + (long long)(it >> 1) * gridDim.x;
    if (step >= p.num_steps) return 0;
    return unit_at(p, (uint32_t)step, it & 1, w) ? 1 : 2;
  }
  if (p.parts <= 1 || it < p.whole_per_cta) {
    const long long u = blockIdx.x + (long long)it * gridDim.x;
    if (u >= p.num_units) return 0;
    const uint32_t head = fast_div((uint32_t)u, p.div_pairs);
    w = make_unit(p, head, (int)((uint32_t)u - head * (uint32_t)p.num_pairs));
    return 1;
  }
  if (it > p.whole_per_cta) return 0;
  const uint32_t q = blockIdx.x;
  const uint32_t parts = (uint32_t)p.parts;
  if (q >= (uint32_t)p.tail_units * parts) return 0;
  const uint32_t u = (uint32_t)p.whole_per_cta * gridDim.x + q / parts;
  const uint32_t head = fast_div(u, p.div_pairs);
  w = make_unit(p, head, (int)(u - head * (uint32_t)p.num_pairs));
  w.parts = p.parts;
  w.part = (int)(q % parts);
  w.tail = (int)(q / parts);
  w.jb = (int)((uint32_t)w.part * (uint32_t)p.num_blocks / parts);
  w.n0 = w.n1 = w.nmax = (int)((uint32_t)(w.part + 1) * (uint32_t)p.num_blocks / parts);
  return 1;
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA abort flag,
// recording `site` once per launch) if the phase did not complete within `timeout_ns`,
// or if another role of the CTA has already aborted.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                           unsigned site, uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > timeout_ns) {
      *abort_flag = 1u;
      atomicCAS(&g_attn_fault_site, 0u, site);
      return false;
    }
  }
}

// Bounded wait used when draining in-flight copies/MMAs before exit: it does not stop
// early on the abort flag, only on its own time limit.
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      *abort_flag = 1u;
      atomicCAS(&g_attn_fault_site, 0u, (unsigned)kSiteDrain);
      return;
    }
  }
}

// Ring position: stage index and the parity of its current fill.
struct Ring {
  uint32_t stage = 0, phase = 0;
  template <int S>
  __device__ __forceinline__ void advance() {
    if (++stage == S) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

template <int D, bool kF8 = false, bool kSepP = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                   const FwdParams p) {
  using Plan = SmemPlan<D, kF8, kSepP>;
  static_assert(!kSepP || (D <= 64 && !kF8), "P beside O needs D <= 64 (bf16)");
  // 32-byte K steps of the tensor-core instructions: 16 bf16 or 32 E4M3 elements each
  constexpr int kSSteps = D * Plan::kElemBytes / 32;
  constexpr int kPVSteps = kBlockN * Plan::kElemBytes / 32;
  constexpr uint32_t kPVStepBytes = (32 / Plan::kElemBytes) * 128;  // K rows of V per step x 128 B
  constexpr int S = Plan::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled TMA tiles and UMMA descriptors need 1024-byte aligned tiles.
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  uint8_t* sQ = smem + Plan::kQOff;
  uint8_t* sKV = smem + Plan::kKVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = bars + 4 + S;
  uint64_t* s_full = bars + 4 + 2 * S;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = s_full + 4;
  uint64_t* o_free = s_full + 6;
  uint64_t* drain = s_full + 8;
  uint64_t* o_staged = s_full + 9;   // a tile's O is in the staging buffer (128 arrivals)
  uint64_t* stage_free = s_full + 10;  // the store warp's TMA stores have read it
  uint64_t* s_free = s_full + 11;      // kSepP: the softmax has read S_t (128 arrivals)
  uint64_t* p_free = s_full + 13;      // kSepP: P_t V completed
  uint8_t* sOst = smem + Plan::kOStageOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Plan::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Plan::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kBlockM);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], kBlockM);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], kSepP ? 2 : 1);   // kSepP: released by both MMA warps
    }
    mbar_init(drain, kSepP ? 2 : 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_free[i], kBlockM);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_staged, kBlockM);
    mbar_init(stage_free, 1);
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
      uint32_t q_par[2] = {1u, 1u};     // empty-barrier waits start on the completed "previous" phase
      uint32_t filled = 0u, fill_par = 0u;  // per stage: ever filled / parity of its last fill
      bool q_filled[2] = {false, false};
      uint32_t q_fill_par[2] = {0u, 0u};

      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int row, int head,
                           uint64_t pol) {
#pragma unroll
        for (int ch = 0; ch < Plan::kChunks; ++ch)
          tma_load_3d(dst + ch * Plan::kChunkBytes, map, bar, ch * Plan::kRowElems, row, head, pol);
      };
      auto load_kv = [&](const CUtensorMap* map, int row, int head) -> bool {
        if (!wait_phase(&kv_empty[ring.stage], ring.phase ^ 1u, abort_flag, kSiteProducerKV)) return false;
        mbar_arrive_expect_tx(&kv_full[ring.stage], Plan::kTileBytes);
        load_tile(map, sKV + ring.stage * Plan::kTileBytes, &kv_full[ring.stage], row, head, pol_kv);
        filled |= 1u << ring.stage;
        fill_par = (fill_par & ~(1u << ring.stage)) | (ring.phase << ring.stage);
        ring.advance<S>();
        return true;
      };
      auto load_q = [&](int t, int row, int head) -> bool {
        if (!wait_phase(&q_empty[t], q_par[t], abort_flag, kSiteProducerQ)) return false;
        q_par[t] ^= 1u;
        mbar_arrive_expect_tx(&q_full[t], Plan::kTileBytes);
        load_tile(&tmap_q, sQ + t * Plan::kTileBytes, &q_full[t], row, head, pol_q);
        q_fill_par[t] = q_filled[t] ? (q_fill_par[t] ^ 1u) : 0u;
        q_filled[t] = true;
        return true;
      };

      bool ok = true;
      for (int it = 0; ok; ++it) {
        Unit w;
        const int got = item_at(p, it, w);
        if (got == 0) break;
        if (got == 2) continue;
        ok = load_q(0, w.q0, w.head_q) && load_kv(&tmap_k, w.jb * kBlockN, w.head_kv) &&
             (!w.valid1 || load_q(1, w.row1, w.head_q1)) && load_kv(&tmap_v, w.jb * kBlockN, w.head_kv);
        for (int j = w.jb + 1; j < w.nmax && ok; ++j)
          ok = load_kv(&tmap_k, j * kBlockN, w.head_kv) && load_kv(&tmap_v, j * kBlockN, w.head_kv);
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      for (int s = 0; s < S; ++s)
        if (filled & (1u << s)) drain_phase(&kv_full[s], (fill_par >> s) & 1u, abort_flag);
      for (int t = 0; t < 2; ++t)
        if (q_filled[t]) drain_phase(&q_full[t], q_fill_par[t], abort_flag);
    }
    __syncwarp();
  } else if (kSepP && (warp == 9 || warp == 11)) {
    // ------------------------------------------------------------ MMA issuers, one per tile (D <= 64)
    // P has tensor-memory columns of its own, so a tile's next S is issued as soon as its
    // softmax has read the current one; each warp walks the K/V ring in the producer's order
    // and releases every stage it passes (a stage is refilled once both tiles released it).
    regs_decrease<kRegsControl>();
    {
      const int t = (warp == 9) ? 0 : 1;
      Ring ring;
      // bit 0: Q full parity, 1: P full, 2: S free, 3: O free; bit 4: an S was issued before
      uint32_t par = 0x8u;
      const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
      const uint64_t desc_q = smem_desc_kmajor_sw128(smem_u32(sQ)) + (uint64_t)((t * Plan::kTileBytes) >> 4);
      const uint64_t desc_k = smem_desc_kmajor_sw128(smem_u32(sKV));
      const uint64_t desc_v = smem_desc_mnmajor_sw128(smem_u32(sKV), Plan::kChunkBytes);
      const uint32_t idesc_s = p.idesc_s, idesc_pv = p.idesc_pv;
      const uint32_t t_sacc = tmem + t * 128;          // S of this tile
      const uint32_t t_oacc = tmem + 256 + t * 128;    // O of this tile
      const uint32_t t_pa = t_oacc + 64;               // P of this tile

      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      auto wait_all = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        const bool mine = wait_phase(bar, parity, abort_flag, site);
        return __all_sync(0xffffffffu, mine);
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      // Next ring stage: waits until it holds its tile; returns the stage.
      auto take = [&](uint32_t& st) -> bool {
        st = ring.stage;
        const bool got = wait_all(&kv_full[st], ring.phase, kSiteMmaKV);
        ring.advance<S>();
        return got;
      };
      // S = Q_t K^T into this tile's score columns, once the softmax has read the previous S.
      auto issue_s = [&](uint32_t stage) -> bool {
        if (par & 0x10u) {
          if (!wait_all(&s_free[t], (par >> 2) & 1u, kSiteMmaSFree)) return false;
          par ^= 0x4u;
        }
        par |= 0x10u;
        tc_fence_after();
        const uint64_t db = adv(desc_k, stage * Plan::kTileBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kSSteps; ++kk) {
            const uint32_t off = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
            if constexpr (kF8)
              mma_ss_f8(t_sacc, adv(desc_q, off), adv(db, off), idesc_s, kk > 0 ? 1u : 0u);
            else
              mma_ss(t_sacc, adv(desc_q, off), adv(db, off), idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
        commit(&s_full[t]);
        return true;
      };

      bool ok = true;
      for (int it = 0; ok; ++it) {
        Unit w;
        const int got = item_at(p, it, w);
        if (got == 0) break;
        if (got == 2) continue;
        const int jb = w.jb;
        const int n = t ? (w.valid1 ? w.n1 : 0) : w.n0;
        int j_end = jb;
        if (n > jb) {
          uint32_t ks;
          if (!(ok = wait_all(&q_full[t], par & 1u, kSiteMmaQ))) break;
          par ^= 0x1u;
          if (!(ok = take(ks))) break;
          if (!(ok = issue_s(ks))) break;
          if (n == jb + 1) commit(&q_empty[t]);
          commit(&kv_empty[ks]);
          for (int j = jb; j < n; ++j) {
            const uint32_t vs = ring.stage, vph = ring.phase;
            ring.advance<S>();
            if (j + 1 < n) {
              if (!(ok = take(ks))) break;
              if (!(ok = issue_s(ks))) break;
              if (j + 2 == n) commit(&q_empty[t]);
              commit(&kv_empty[ks]);
            }
            if (!(ok = wait_all(&p_full[t], (par >> 1) & 1u, kSiteMmaP))) break;
            par ^= 0x2u;
            if (j == jb) {
              if (!(ok = wait_all(&o_free[t], (par >> 3) & 1u, kSiteMmaOFree))) break;
              par ^= 0x8u;
            }
            if (!(ok = wait_all(&kv_full[vs], vph, kSiteMmaKV))) break;
            tc_fence_after();
            const uint64_t dv = adv(desc_v, vs * Plan::kTileBytes);
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < kPVSteps; ++kk) {
                if constexpr (kF8)
                  mma_ts_f8(t_oacc, t_pa + kk * 8, adv(dv, kk * kPVStepBytes), idesc_pv, (j > jb || kk > 0) ? 1u : 0u);
                else
                  mma_ts(t_oacc, t_pa + kk * 8, adv(dv, kk * kPVStepBytes), idesc_pv, (j > jb || kk > 0) ? 1u : 0u);
              }
            }
            __syncwarp();
            commit(&p_free[t]);
            if (j == n - 1) commit(&o_full[t]);
            commit(&kv_empty[vs]);
          }
          if (!ok) break;
          j_end = n;
        }
        // K/V stages of blocks this tile does not visit (a causal unit's last block for tile 0,
        // every block when tile 1 has no rows): released once they hold their tile.
        for (int j = j_end; j < w.nmax && ok; ++j) {
#pragma unroll
          for (int kv = 0; kv < 2 && ok; ++kv) {
            uint32_t st;
            if (!(ok = take(st))) break;
            if (lane == 0) mbar_arrive(&kv_empty[st]);
            __syncwarp();
          }
        }
      }
      // Drain: all MMAs issued by this warp complete before TMEM is released.
      commit(drain);
      drain_phase(drain, 0u, abort_flag);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule, so control flow and descriptor arithmetic stay
    // warp-uniform (kept in uniform registers); one elected lane issues each tcgen05
    // instruction.
    regs_decrease<kRegsControl>();
    {
      Ring ring;
      uint32_t q_par[2] = {0u, 0u}, pf_par[2] = {0u, 0u}, of_par[2] = {1u, 1u};
      const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base, 0);
      const uint64_t desc_q = smem_desc_kmajor_sw128(smem_u32(sQ));
      const uint64_t desc_k = smem_desc_kmajor_sw128(smem_u32(sKV));
      const uint64_t desc_v = smem_desc_mnmajor_sw128(smem_u32(sKV), Plan::kChunkBytes);
      const uint32_t idesc_s = p.idesc_s, idesc_pv = p.idesc_pv;

      // Adds a byte offset to a descriptor's start-address field (bits 0-13, in 16-byte units).
      auto adv = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
      // S_t = Q_t K^T over D in 32-byte steps (K-major A and B, 128-byte swizzle).
      auto issue_s = [&](int t, uint32_t stage) {
        const uint64_t da = adv(desc_q, t * Plan::kTileBytes);
        const uint64_t db = adv(desc_k, stage * Plan::kTileBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kSSteps; ++kk) {
            const uint32_t off = (kk >> 2) * Plan::kChunkBytes + (kk & 3) * 32;
            if constexpr (kF8)
              mma_ss_f8(tmem + t * 128, adv(da, off), adv(db, off), idesc_s, kk > 0 ? 1u : 0u);
            else
              mma_ss(tmem + t * 128, adv(da, off), adv(db, off), idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // O_t += P_t V over the 128 keys in 32-byte steps (P from TMEM: 8 columns per step;
      // V MN-major in smem).
      auto issue_pv = [&](int t, uint32_t stage, bool accumulate) {
        const uint64_t dv = adv(desc_v, stage * Plan::kTileBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kPVSteps; ++kk) {
            if constexpr (kF8)
              mma_ts_f8(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, adv(dv, kk * kPVStepBytes), idesc_pv,
                        (accumulate || kk > 0) ? 1u : 0u);
            else
              mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, adv(dv, kk * kPVStepBytes), idesc_pv,
                     (accumulate || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      // Every lane waits; the warp proceeds only if all lanes saw the phase complete.
      auto wait_all = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        const bool mine = wait_phase(bar, parity, abort_flag, site);
        return __all_sync(0xffffffffu, mine);
      };

      bool ok = true;
      for (int it = 0; ok; ++it) {
        Unit w;
        const int got = item_at(p, it, w);
        if (got == 0) break;
        if (got == 2) continue;
        const int jb = w.jb;
        const int n0 = w.n0, n1 = w.valid1 ? w.n1 : 0;

        // First block's scores for both tiles.
        if (!(ok = wait_all(&q_full[0], q_par[0], kSiteMmaQ))) break;
        q_par[0] ^= 1u;
        const uint32_t k0_stage = ring.stage;
        if (!(ok = wait_all(&kv_full[k0_stage], ring.phase, kSiteMmaKV))) break;
        ring.advance<S>();
        tc_fence_after();
        issue_s(0, k0_stage);
        commit(&s_full[0]);
        if (n0 == jb + 1) commit(&q_empty[0]);
        if (n1 > 0) {
          if (!(ok = wait_all(&q_full[1], q_par[1], kSiteMmaQ))) break;
          q_par[1] ^= 1u;
          tc_fence_after();
          issue_s(1, k0_stage);
          commit(&s_full[1]);
          if (n1 == jb + 1) commit(&q_empty[1]);
        }
        commit(&kv_empty[k0_stage]);

        for (int j = jb; j < w.nmax && ok; ++j) {
          const uint32_t v_stage = ring.stage;
          if (!(ok = wait_all(&kv_full[v_stage], ring.phase, kSiteMmaKV))) break;
          ring.advance<S>();
          const bool has_next = (j + 1) < w.nmax;
          const uint32_t kn_stage = ring.stage, kn_phase = ring.phase;
          // K_{j+1} is waited for before P: it was loaded an iteration ago, and this way the
          // P V and next-S MMAs of a tile are issued back to back once P is ready.
          if (has_next && !(ok = wait_all(&kv_full[kn_stage], kn_phase, kSiteMmaKV))) break;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int n = t ? n1 : n0;
            if (!ok || j >= n) continue;
            if (!(ok = wait_all(&p_full[t], pf_par[t], kSiteMmaP))) continue;
            pf_par[t] ^= 1u;
            if (j == jb) {
              if (!(ok = wait_all(&o_free[t], of_par[t], kSiteMmaOFree))) continue;
              of_par[t] ^= 1u;
            }
            tc_fence_after();
            issue_pv(t, v_stage, j > jb);
            if (j == n - 1) commit(&o_full[t]);
            if (j + 1 < n) {
              issue_s(t, kn_stage);
              commit(&s_full[t]);
              if (j + 2 == n) commit(&q_empty[t]);
            }
          }
          if (!ok) break;
          commit(&kv_empty[v_stage]);
          if (has_next) {
            commit(&kv_empty[kn_stage]);
            ring.advance<S>();
          }
        }
      }
      // Drain: all MMAs issued by this warp complete before TMEM is released.
      commit(drain);
      drain_phase(drain, 0u, abort_flag);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    regs_increase<kRegsSoftmax>();
    const int t = warp >> 2;                       // Q tile of this warpgroup
    const int r = threadIdx.x & 127;               // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + t * 128;
    // where P goes: over the scores, or (kSepP) its own columns after O_t
    const uint32_t t_p = kSepP ? tmem_base + lane_off + 256 + t * 128 + 64 : t_s;
    uint32_t p_uses = 0u;   // kSepP: P tiles written by this warpgroup
    const uint32_t t_o = tmem_base + lane_off + 256 + t * 128;
    const float c = p.c;
    uint32_t s_par = 0u, o_par = 0u;
    uint32_t stage_uses = 0u;  // tiles staged before this unit (both tiles, in the store warp's order)
    bool ok = true;

    for (int it = 0; ok; ++it) {
      Unit w;
      const int got_item = item_at(p, it, w);
      if (got_item == 0) break;
      if (got_item == 2) continue;
      // staging order: per unit without a split, tile 0 then (if it has rows) tile 1
      const uint32_t my_use = stage_uses + (uint32_t)t;
      if (w.parts == 1) stage_uses += w.valid1 ? 2u : 1u;
      if (t == 1 && !w.valid1) continue;
      const int n = t ? w.n1 : w.n0;
      const int row = (t ? w.row1 : w.q0) + r;
      const int head_o = t ? w.head_q1 : w.head_q;   // query head of this tile's rows
      const int key_lim = p.causal ? min(row, p.N - 1) : (p.N - 1);
      float m = -INFINITY, l = 0.f;

      for (int j = w.jb; j < n; ++j) {
        if (!(ok = wait_phase(&s_full[t], s_par, abort_flag, kSiteSoftmaxS))) break;
        s_par ^= 1u;
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
          if constexpr (kSepP) {
            // the scores are in registers: this tile's MMA warp may compute the next S over them
            tc_fence_before();
            mbar_arrive(&s_free[t]);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(a0[i]);
            s[32 + i] = __uint_as_float(a1[i]);
            s[64 + i] = __uint_as_float(a2[i]);
            s[96 + i] = __uint_as_float(a3[i]);
          }
        }
        const int k0 = j * kBlockN;
        const bool masked = (k0 + kBlockN - 1) > key_lim;
        if (masked) {
#pragma unroll
          for (int i = 0; i < kBlockN; ++i)
            if (k0 + i > key_lim) s[i] = -INFINITY;
        }
        // Row maximum: four independent chains of three-input max, then combined.
        auto row_max = [&]() -> float {
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
          return fmaxf(max3f(mx[0], mx[1], mx[2]), mx[3]);
        };
        // P = 2^(s*c - m_use) in two halves of 64 keys; each half is packed (bf16 pairs, or
        // four E4M3 bytes per column for E4M3 inputs: p <= 2^8 < 448 fits) and written over
        // the (already loaded) score columns it came from.  Returns the row
        // sum of the fp32 values.  Masked keys hold s = -inf, so their p is 0 from the
        // special-function unit and 2^-125 (negligible) from the polynomial (c > 0 always).
        // poly_pairs_per8<D>() of every 8 column pairs use the FMA-pipe polynomial instead
        // of the special-function unit.  Warp-collective (TMEM stores).
        auto exp_row = [&](float m_use) -> float {
          const float2 c2 = make_float2(c, c);
          const float2 nm2 = make_float2(-m_use, -m_use);
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
            float prev = 0.f;  // E4M3: the first value of a group of four
            float prev2 = 0.f;
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              const int col = half * 64 + i;
              const float2 x = fma2(make_float2(s[col], s[col + 1]), c2, nm2);
              float2 pr;
              if (((col >> 1) & 7) < poly_pairs_per8<D, kF8, kSepP>()) {
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
              tmem_st16(t_p + half * 16, pk16);
            } else {
              tmem_st32(t_p + half * 32, pk);
            }
          }
          const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
          return a.x + a.y;
        };

        // Lazy correction: the running max m is replaced only when the row's maximum
        // exceeds it by more than kRescaleLog2, and then O and l are rescaled by 2^(m-m_new).
        const float m_new = fmaxf(m, row_max() * c);
        float alpha = 1.f;
        bool any_rescale = false;
        if (j == w.jb) {
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
        if constexpr (kSepP) {
          // P_t's columns (and O_t, for a rescale) are free once the previous P_t V completed
          if (p_uses > 0u && !(ok = wait_phase(&p_free[t], (p_uses - 1u) & 1u, abort_flag, kSitePFree))) break;
          ++p_uses;
          tc_fence_after();
        }
        l += exp_row(m);
        if (any_rescale) {
          // O_t holds blocks < j (their MMAs completed before S_t(j) was signalled) and
          // P_t(j) V has not been issued yet, so the accumulator can be rescaled here.
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
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;

      // Epilogue: O = O_acc / l -> bf16, LSE = (m + log2 l) ln 2.
      {
        const bool got_o = wait_phase(&o_full[t], o_par, abort_flag, kSiteSoftmaxO);
        // a split unit's epilogue has tile-wide barriers: agree on the outcome first
        ok = (w.parts > 1) ? bar_and(1 + t, kBlockM, got_o) : got_o;
        if (!ok) break;
      }
      o_par ^= 1u;
      tc_fence_after();
      const bool row_ok = row < p.N;
      __nv_bfloat16* orow = p.o + ((size_t)head_o * p.N + (row_ok ? row : 0)) * D;
      if (w.parts == 1 && Plan::kStagedStore) {
        // O / l -> bf16 pairs in registers; O's tensor memory is then free for the next unit.
        const float inv_l = (kF8 ? p.o_scale : 1.f) / l;
        uint32_t packed[D / 2];
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld32(t_o + ch * 32, ov);
          tmem_ld_wait();
          reg_fence32(ov);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[16 * ch + i] =
                pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
        }
        tc_fence_before();
        mbar_arrive(&o_free[t]);
        // Stage the row (64-column chunks, 128-byte swizzle: piece q of row r at q ^ (r % 8)) once
        // the previous tile's stores have read the buffer, then hand it to the store warp.
        if (my_use > 0 && !(ok = wait_phase(stage_free, (my_use - 1u) & 1u, abort_flag, kSiteStageFree))) break;
        const uint32_t srow = smem_u32(sOst) + r * 128;
#pragma unroll
        for (int q = 0; q < D / 8; ++q)
          st_shared_v4(srow + (q >> 3) * Plan::kChunkBytes + (((q & 7) ^ (r & 7)) << 4), packed[4 * q],
                       packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        fence_proxy_async_smem();
        mbar_arrive(o_staged);
        if (row_ok) p.lse[(size_t)head_o * p.N + row] = (m + log2f(l)) * 0.69314718055994530942f;
      } else if (w.parts == 1) {
        const float inv_l = (kF8 ? p.o_scale : 1.f) / l;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld32(t_o + ch * 32, ov);
          tmem_ld_wait();
          reg_fence32(ov);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&o_free[t]);
        if (row_ok) p.lse[(size_t)head_o * p.N + row] = (m + log2f(l)) * 0.69314718055994530942f;
      } else {
        // One of the two KV ranges of a split unit.  The ranges first agree on their
        // finishing order; the first publishes its unnormalised O rows and (m, l) and
        // raises a ready flag, the second waits for the flag (bounded) and merges:
        //   M = max(m0, m1),  O = (O0 2^(m0-M) + O1 2^(m1-M)) / (l0 2^(m0-M) + l1 2^(m1-M))
        // with the ranges always taken in range order, so the result does not depend on
        // which range finished first.
        volatile unsigned* order = reinterpret_cast<volatile unsigned*>(smem + Plan::kMiscOff + 8 + 4 * t);
        unsigned* cnt = &p.ws_cnt[(w.tail * 2 + t) * 2];    // finished ranges (epoch-tagged)
        unsigned* ready = cnt + 1;                          // epoch once range "first" published
        if (r == 0) *order = count_finished(cnt, p.epoch);
        named_bar_sync(1 + t, kBlockM);
        const bool first = (*order == 0u);
        const size_t slot = (size_t)w.tail * 2 + t;
        float4* o_ws = reinterpret_cast<float4*>(p.ws_o) + slot * (kBlockM * D / 4);  // [D/4][128] float4
        float2* ml_ws = reinterpret_cast<float2*>(p.ws_ml) + slot * kBlockM;         // [128]
        if (first) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(t_o + ch * 32, ov);
            tmem_ld_wait();
            reg_fence32(ov);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              o_ws[(ch * 8 + i) * kBlockM + r] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                                             __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
          }
          tc_fence_before();
          mbar_arrive(&o_free[t]);
          ml_ws[r] = make_float2(m, l);
          __threadfence();
          named_bar_sync(1 + t, kBlockM);
          if (r == 0) st_release_gpu(ready, p.epoch);
        } else {
          // wait for the other range's rows (it has counted itself finished, so it is
          // only storing them); one thread polls, the tile's threads then all read.
          bool have = true;
          if (r == 0) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_gpu(ready) != p.epoch) {
              if (global_timer_ns() - t0 > kWaitTimeoutNs) {
                *abort_flag = 1u;
                atomicCAS(&g_attn_fault_site, 0u, (unsigned)kSiteSplitMerge);
                have = false;
                break;
              }
            }
            *order = have ? 1u : 2u;
            // Both ranges have counted themselves and the first has published, so nothing
            // else reads these two words in this launch: they are left at 0 (never an
            // epoch), and no later launch can take them for its own, whatever its epoch.
            if (have) {
              *reinterpret_cast<volatile unsigned*>(cnt) = 0u;
              *reinterpret_cast<volatile unsigned*>(ready) = 0u;
            }
          }
          named_bar_sync(1 + t, kBlockM);
          if (*order == 2u) {
            ok = false;
          } else {
            __threadfence();
            const float2 mo = __ldcg(ml_ws + r);                       // the other range
            const bool own_is_0 = (w.part == 0);
            const float m0 = own_is_0 ? m : mo.x, l0 = own_is_0 ? l : mo.y;
            const float m1 = own_is_0 ? mo.x : m, l1 = own_is_0 ? mo.y : l;
            const float mt = fmaxf(m0, m1);
            const float w0 = ex2_approx(m0 - mt), w1 = ex2_approx(m1 - mt);
            const float lt = fmaf(l1, w1, l0 * w0);
            const float inv_l = (kF8 ? p.o_scale : 1.f) / lt;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              float4 other[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) other[i] = __ldcg(o_ws + (ch * 8 + i) * kBlockM + r);
              uint32_t ov[32];
              tmem_ld32(t_o + ch * 32, ov);
              tmem_ld_wait();
              reg_fence32(ov);
              uint32_t packed[16];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float oth[4] = {other[i].x, other[i].y, other[i].z, other[i].w};
                float res[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float mine = __uint_as_float(ov[4 * i + e]);
                  const float x0 = own_is_0 ? mine : oth[e], x1 = own_is_0 ? oth[e] : mine;
                  res[e] = fmaf(x1, w1, x0 * w0) * inv_l;
                }
                packed[2 * i] = pack_bf16x2(res[0], res[1]);
                packed[2 * i + 1] = pack_bf16x2(res[2], res[3]);
              }
              if (row_ok) {
                uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
              }
            }
            if (row_ok) p.lse[(size_t)head_o * p.N + row] = (mt + log2f(lt)) * 0.69314718055994530942f;
          }
          tc_fence_before();
          mbar_arrive(&o_free[t]);
        }
      }
    }
  } else if (warp == 10 && Plan::kStagedStore) {
    // ------------------------------------------------------------ output store warp
    // Tiles in the order the softmax warpgroups stage them (per unit without a split: tile 0,
    // then tile 1 if it has rows): wait until staged, store with TMA (rows past N are not
    // written), wait until the stores have read the buffer and release it.
    regs_decrease<kRegsControl>();
    if (lane == 0) {
      uint32_t st_par = 0u;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        Unit w;
        const int got = item_at(p, it, w);
        if (got == 0) break;
        if (got == 2 || w.parts > 1) continue;
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 1 && !w.valid1) continue;
          if (!(ok = wait_phase(o_staged, st_par, abort_flag, kSiteStore))) break;
          st_par ^= 1u;
#pragma unroll
          for (int ch = 0; ch < Plan::kOChunks; ++ch)
            tma_store_3d(&tmap_o, sOst + ch * Plan::kChunkBytes, ch * 64, t ? w.row1 : w.q0, t ? w.head_q1 : w.head_q);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(stage_free);
        }
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

// ---------------------------------------------------------------- self-test kernels

// Evaluates the polynomial exp2 used by the softmax on n inputs (n even is not required).
__global__ void selftest_exp2_poly(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 out = exp2_poly2(in);
  y[i] = out.x;
  if (i + 1 < n) y[i + 1] = out.y;
}

// Waits on an mbarrier that nothing ever arrives on, with a short limit: exercises the
// bounded-wait path (abort flag, fault-site record, orderly return) without a fault.
__global__ void selftest_wait_timeout(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_phase(&bar, 0u, &abort_flag, kSiteSelfTest, timeout_ns);
  __syncthreads();
}

}  // namespace attn
