// attn_api.cu -- host side of the C ABI declared in include/attn.h.
//
// Validates arguments before any CUDA call, encodes the TMA tensor maps, sizes the
// grids to the problem and the SM count and launches the sm_100a kernels on the
// caller's stream.  Nothing is allocated per call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_bwd_kernel.cuh"
#include "attn_rope_kernel.cuh"
#include "attn_fwd_wide_kernel.cuh"
#include "attn_fwd_colsplit_kernel.cuh"

#define ATTN_VERSION_STRING "b200-attn 0.1 (sm_100a, tcgen05/TMA/TMEM)"

namespace {

constexpr int kMaxDevices = 64;

thread_local char g_last_cuda_error[256] = "";

void record_cuda_error(const char* what, cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s (%d)", what, cudaGetErrorString(e),
                (int)e);
}

void record_driver_error(const char* what, int code) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: CUresult %d", what, code);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* sym = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &sym, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(sym);
  });
  return fn;
}

struct DeviceInfo {
  std::once_flag once;
  int num_sms = 0;
  bool attrs_ok = false;
  bool bad_regs = false;
  cudaError_t err = cudaSuccess;
};
DeviceInfo g_dev[kMaxDevices];

// Per device: SM count and the kernels' dynamic shared memory opt-in.
bool device_setup(int dev, int* num_sms) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&d, dev] {
    cudaError_t e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    // Every head-dim instance: dynamic shared memory opt-in, and a check that it has the
    // register count its warpgroup register split (setmaxnreg) assumes at launch -- a build
    // that differs would make the increase wait forever, so it refuses to launch.
    bool regs_ok = true;
    auto setup = [&](const void* fn, int smem) {
      if (e != cudaSuccess) return;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      cudaFuncAttributes fa;
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, fn);
      if (e == cudaSuccess && fa.numRegs != attn::kRegsAtLaunch) regs_ok = false;
    };
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<32>), attn::SmemPlan<32>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<64>), attn::SmemPlan<64>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<96>), attn::SmemPlan<96>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<128>), attn::SmemPlan<128>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_colsplit_sm100<32>), attn::CsPlan<32>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_colsplit_sm100<64>), attn::CsPlan<64>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_colsplit_sm100<96>), attn::CsPlan<96>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_colsplit_sm100<128>), attn::CsPlan<128>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<32, false, true>), attn::SmemPlan<32, false, true>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<64, false, true>), attn::SmemPlan<64, false, true>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<32, true>), attn::SmemPlan<32, true>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<64, true>), attn::SmemPlan<64, true>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<96, true>), attn::SmemPlan<96, true>::kAlloc);
    setup(reinterpret_cast<const void*>(attn::attn_fwd_sm100<128, true>), attn::SmemPlan<128, true>::kAlloc);
    // the wide-head kernel has no register split: dynamic shared memory opt-in only
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_fwd_wide_sm100<192>),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, attn::WidePlan<192>::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_fwd_wide_sm100<256>),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, attn::WidePlan<256>::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_fwd_wide_sm100<192, true>),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, attn::WidePlan<192, true>::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_fwd_wide_sm100<256, true>),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, attn::WidePlan<256, true>::kAlloc);
    d.err = e;
    d.attrs_ok = (e == cudaSuccess);
    if (d.attrs_ok && !regs_ok) {
      d.attrs_ok = false;
      d.err = cudaErrorInvalidDeviceFunction;
      d.bad_regs = true;
    }
  });
  if (!d.attrs_ok && d.bad_regs) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "kernel register count differs from the register split it was written for");
    return false;
  }
  if (!d.attrs_ok) {
    record_cuda_error("device setup", d.err);
    return false;
  }
  *num_sms = d.num_sms;
  return true;
}

// [heads, N, D] tensor of bf16 (elem_bytes 2) or E4M3 bytes (1) viewed by TMA as 3-D (D
// fastest), boxes of one 128-byte row chunk x 128 rows x 1 head with 128-byte swizzle; rows past
// N (and columns past D) read as zero.
int encode_map(CUtensorMap* map, const void* base, long long heads, int N, int D, int elem_bytes = 2) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled entry point unavailable");
    return ATTN_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * elem_bytes, (cuuint64_t)N * (cuuint64_t)D * elem_bytes};
  cuuint32_t box[3] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)attn::kBlockM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_driver_error("cuTensorMapEncodeTiled", (int)r);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// The output O [heads, N, D] (bf16) as a TMA store target: boxes of 32 columns (64 bytes) x 128 rows x
// 1 head with 64-byte swizzle, matching the column-split kernel's staging buffers; rows past N are not
// written.
int encode_map_o(CUtensorMap* map, void* base, long long heads, int N, int D) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled entry point unavailable");
    return ATTN_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * (cuuint64_t)D * 2};
  cuuint32_t box[3] = {32, (cuuint32_t)attn::kBlockM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_driver_error("cuTensorMapEncodeTiled (output)", (int)r);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Forward (bf16): 32 ... 128 on the two-tile kernel, 192 and 256 on the wide-head kernel.
bool supported_head_dim(int D) { return D == 32 || D == 64 || D == 96 || D == 128 || D == 192 || D == 256; }
bool narrow_head_dim(int D) { return D == 32 || D == 64 || D == 96 || D == 128; }

// How a non-causal problem is spread over the persistent grid.  Whole units run round
// robin; if the last wave would be at most half full, each of its units is split into two
// KV ranges (of at least two KV blocks) that run on separate CTAs and are merged through
// a workspace holding the first-finished range's rows.  Since 2 x tail_units <= SMs, the
// workspace is bounded by SMs/2 x 2 tiles x 128 rows x (D + 2) floats.
struct Schedule {
  long long grid = 0;
  int whole_per_cta = 0, tail_units = 0, parts = 1;
  size_t cnt_bytes = 0, ml_bytes = 0, o_bytes = 0;
  size_t ws_bytes() const { return cnt_bytes + ml_bytes + o_bytes; }
};

Schedule plan_schedule(long long units, long long steps, int num_blocks, int num_sms, int causal, int D,
                       bool allow_split) {
  Schedule sc;
  sc.grid = steps < num_sms ? steps : num_sms;
  if (causal || !allow_split || units <= 0) return sc;
  const long long tail = units % num_sms, whole = units / num_sms;
  if (tail == 0) return sc;
  // two KV ranges per unit of the last wave, each of at least two KV blocks
  if (2 * tail > num_sms || num_blocks < 4) return sc;
  const long long k = 2;
  sc.whole_per_cta = (int)whole;
  sc.tail_units = (int)tail;
  sc.parts = (int)k;
  sc.grid = whole > 0 ? num_sms : tail * k;
  const size_t slots = (size_t)tail * 2;  // the first range's rows, per unit and tile
  sc.cnt_bytes = ((size_t)tail * 2 * 2 * sizeof(unsigned) + 255) / 256 * 256;
  sc.ml_bytes = slots * attn::kBlockM * 2 * sizeof(float);
  sc.o_bytes = slots * attn::kBlockM * (size_t)D * sizeof(float);
  return sc;
}

unsigned next_epoch() {
  static std::atomic<unsigned> counter{0};
  unsigned e;
  do {
    e = (counter.fetch_add(1u) + 1u) & 0xFFFFFFu;
  } while (e == 0u);
  return e;
}

// e4m3: q, k, v hold E4M3 bytes whose values are multiplied by qk_descale (in the scores) and
// o_scale (in the output); otherwise bf16 and both factors 1.
int launch_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int N, int D, int causal, float scale, void* workspace, size_t workspace_bytes,
                   void* stream, bool e4m3 = false, float qk_descale = 1.f, float o_scale = 1.f);

// bf16 forward without a split last wave: which kernel runs.  Measured on B200 by interleaved
// A/B runs of the two kernels on the same inputs: the column-split kernel (one Q tile per unit,
// two score buffers) is 5-8 % faster for causal D = 128 at N <= 2048, where the two-tile
// kernel's unit boundaries and lone diagonal blocks weigh most; everywhere else the two-tile
// kernel is as fast or faster (N >= 4096: 6-13 %; D = 64: 2-9 %), because each K/V tile it loads
// feeds 256 query rows instead of 128.
bool use_column_split(int N, int D, int causal) { return causal && D == 128 && N <= 2048; }

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

const char* attn_last_cuda_error(void) { return g_last_cuda_error; }

const char* attn_version(void) { return ATTN_VERSION_STRING; }

long long attn_num_units(int B, int Hq, int N) {
  if (B < 0 || Hq < 1 || N < 0) return -1;
  const long long pairs = ((long long)N + 2 * attn::kBlockM - 1) / (2 * attn::kBlockM);
  return (long long)B * Hq * pairs;
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
             int D, int causal, float scale, void* stream) {
  return launch_forward(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, nullptr, 0, stream);
}

int attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                int D, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr && workspace_bytes != 0) return ATTN_ERR_INVALID_ARG;
  if (workspace != nullptr && !aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
  return launch_forward(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, workspace, workspace_bytes, stream);
}

long long attn_fwd_workspace_bytes(int B, int Hq, int N, int D, int causal) {
  if (B < 0 || Hq < 1 || N < 0 || !supported_head_dim(D)) return -1;
  if (B == 0 || N == 0 || causal || !narrow_head_dim(D)) return 0;  // the wide-head kernel never splits
  int dev = 0, num_sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  const long long units = attn_num_units(B, Hq, N);
  const int nb = (int)(((long long)N + attn::kBlockN - 1) / attn::kBlockN);
  return (long long)plan_schedule(units, units, nb, num_sms, 0, D, true).ws_bytes();
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int D, int causal, float scale, float q_descale, float k_descale, float v_descale, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (workspace == nullptr && workspace_bytes != 0) return ATTN_ERR_INVALID_ARG;
  if (workspace != nullptr && !aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
  if (!std::isfinite(q_descale) || !std::isfinite(k_descale) || !std::isfinite(v_descale) || q_descale == 0.f ||
      k_descale == 0.f)
    return ATTN_ERR_INVALID_ARG;
  return launch_forward(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, workspace, workspace_bytes, stream,
                        true, q_descale * k_descale, v_descale);
}

}  // extern "C"

namespace {

int launch_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int N, int D, int causal, float scale, void* workspace, size_t workspace_bytes,
                   void* stream, bool e4m3, float qk_descale, float o_scale) {

  // ---- host-side validation (no CUDA call before this block passes)
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0 || !std::isfinite(scale))
    return ATTN_ERR_INVALID_ARG;
  if (!supported_head_dim(D)) return ATTN_ERR_UNSUPPORTED;
  if (e4m3 && (!std::isfinite(qk_descale) || !std::isfinite(o_scale) || qk_descale == 0.f)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Hq > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  // the scheduler indexes work units (256 query rows of one head) in 32 bits
  if (attn_num_units(B, Hq, N) > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  // D = 192, 256: the wide-head kernel's CTAs step through its tiles in 32 bits
  if (!narrow_head_dim(D) && (long long)B * Hq * (((long long)N + attn::kBlockN - 1) / attn::kBlockN) > (1LL << 30))
    return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;  // empty problem: nothing to compute or write
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return ATTN_ERR_MISALIGNED;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error("cudaGetDevice", e);
    return ATTN_ERR_CUDA;
  }
  int num_sms = 0;
  if (!device_setup(dev, &num_sms)) return ATTN_ERR_CUDA;

  CUtensorMap mq, mk, mv;
  int st;
  const int eb = e4m3 ? 1 : 2;
  if ((st = encode_map(&mq, q, (long long)B * Hq, N, D, eb)) != ATTN_OK) return st;
  if ((st = encode_map(&mk, k, (long long)B * Hkv, N, D, eb)) != ATTN_OK) return st;
  if ((st = encode_map(&mv, v, (long long)B * Hkv, N, D, eb)) != ATTN_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!narrow_head_dim(D)) {
    // D = 192, 256: one CTA per 128-row Q tile on the wide-head kernel
    attn::WideParams wp;
    wp.o = reinterpret_cast<__nv_bfloat16*>(o);
    wp.lse = lse;
    wp.Hq = Hq;
    wp.group = Hq / Hkv;
    wp.N = N;
    wp.num_blocks = (int)(((long long)N + attn::kBlockN - 1) / attn::kBlockN);
    wp.causal = causal ? 1 : 0;
    // (E4M3: the scores carry the product of the Q and K descales; its sign joins scale's.)
    const float ws_eff = scale * qk_descale;
    wp.c = std::fmax(std::fabs(ws_eff) * 1.44269504088896340736f, 1e-30f);
    wp.o_scale = o_scale;
    wp.idesc_s = e4m3 ? attn::idesc_e4m3_f32(attn::kBlockM, attn::kBlockN, false, false, ws_eff < 0.f)
                      : attn::idesc_bf16_f32(attn::kBlockM, attn::kBlockN, false, false, ws_eff < 0.f);
    wp.idesc_pv = e4m3 ? attn::idesc_e4m3_f32(attn::kBlockM, D, false, true, false)
                       : attn::idesc_bf16_f32(attn::kBlockM, D, false, true, false);
    const long long tiles = (long long)B * Hq * wp.num_blocks;   // <= 2^30, checked above
    // Work items: causal, a head's heaviest and lightest tiles together (equal items) when
    // there are enough of them to fill the GPU, else single tiles.  CTAs are persistent for
    // causal shapes and for N <= 2048 (one CTA per SM walking the items: the next tile's Q
    // load and first scores overlap the current tile's last blocks and epilogue); longer
    // non-causal shapes take one CTA per tile, which measured up to 2 % faster there.
    const long long pairs = (long long)B * Hq * ((wp.num_blocks + 1) / 2);
    wp.pair = (causal && pairs >= num_sms) ? 1 : 0;
    wp.num_items = (int)(wp.pair ? pairs : tiles);
    const bool persistent = causal || wp.num_blocks <= 16;
    const long long grid = (persistent && wp.num_items > num_sms) ? num_sms : wp.num_items;
    if (e4m3 && D == 192)
      attn::attn_fwd_wide_sm100<192, true><<<(unsigned)grid, attn::kWideThreads, attn::WidePlan<192, true>::kAlloc,
                                             s>>>(mq, mk, mv, wp);
    else if (e4m3)
      attn::attn_fwd_wide_sm100<256, true><<<(unsigned)grid, attn::kWideThreads, attn::WidePlan<256, true>::kAlloc,
                                             s>>>(mq, mk, mv, wp);
    else if (D == 192)
      attn::attn_fwd_wide_sm100<192><<<(unsigned)grid, attn::kWideThreads, attn::WidePlan<192>::kAlloc, s>>>(
          mq, mk, mv, wp);
    else
      attn::attn_fwd_wide_sm100<256><<<(unsigned)grid, attn::kWideThreads, attn::WidePlan<256>::kAlloc, s>>>(
          mq, mk, mv, wp);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      record_cuda_error("kernel launch", e);
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }

  attn::FwdParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.num_pairs = (int)(((long long)N + 2 * attn::kBlockM - 1) / (2 * attn::kBlockM));
  p.num_blocks = (int)(((long long)N + attn::kBlockN - 1) / attn::kBlockN);
  p.num_units = attn_num_units(B, Hq, N);
  p.causal = causal ? 1 : 0;
  p.units_per_step = p.causal ? 2 : 1;
  p.num_steps = p.causal ? (long long)B * Hq * ((p.num_pairs + 1) / 2) : p.num_units;
  // Causal GQA with an even group: units pair two query heads of one KV head at the same query
  // tile (both tiles then see the same KV blocks; no lone diagonal block for tile 1).
  p.head_pairs = (p.causal && (Hq / Hkv) % 2 == 0) ? 1 : 0;
  p.div_hq2 = attn::make_fast_div((uint32_t)(Hq / 2 > 0 ? Hq / 2 : 1));
  if (p.head_pairs) {
    p.num_pairs = p.num_blocks;                                         // units per head pair
    p.num_units = (long long)B * (Hq / 2) * p.num_blocks;
    p.num_steps = (long long)B * (Hq / 2) * ((p.num_blocks + 1) / 2);
  }
  p.div_pairs = attn::make_fast_div((uint32_t)p.num_pairs);
  p.div_steps = attn::make_fast_div((uint32_t)((p.num_pairs + 1) / 2));
  p.div_hq = attn::make_fast_div((uint32_t)Hq);
  p.div_group = attn::make_fast_div((uint32_t)p.group);
  // c > 0 always: masked scores are -inf and -inf * c must stay -inf.  For scale == 0 every
  // allowed score gives 2^(tiny) == 1 in fp32, the same softmax as c == 0.
  // (E4M3: the scores carry the product of the Q and K descales; its sign joins scale's.)
  const float s_eff = scale * qk_descale;
  p.c = std::fmax(std::fabs(s_eff) * 1.44269504088896340736f, 1e-30f);
  p.o_scale = o_scale;
  p.idesc_s = e4m3 ? attn::idesc_e4m3_f32(attn::kBlockM, attn::kBlockN, false, false, s_eff < 0.f)
                   : attn::idesc_bf16_f32(attn::kBlockM, attn::kBlockN, false, false, s_eff < 0.f);
  p.idesc_pv = e4m3 ? attn::idesc_e4m3_f32(attn::kBlockM, D, false, true, false)
                    : attn::idesc_bf16_f32(attn::kBlockM, D, false, true, false);

  // Split the last wave only when a workspace big enough for it was given.
  const Schedule plan0 = plan_schedule(p.num_units, p.num_steps, p.num_blocks, num_sms, p.causal, D, true);
  const bool split = workspace != nullptr && plan0.parts > 1;
  if (split && workspace_bytes < plan0.ws_bytes()) return ATTN_ERR_INVALID_ARG;
  if (!e4m3 && !split && use_column_split(N, D, causal)) {
    // the column-split kernel (one Q tile per unit)
    CUtensorMap mo;
    if ((st = encode_map_o(&mo, o, (long long)B * Hq, N, D)) != ATTN_OK) return st;
    attn::CsParams cp;
    cp.lse = lse;
    cp.Hq = Hq;
    cp.Hkv = Hkv;
    cp.N = N;
    cp.group = Hq / Hkv;
    cp.num_tiles = p.num_blocks;
    const long long units = (long long)B * Hq * p.num_blocks;
    if (units > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    cp.num_units = (int)units;
    cp.causal = p.causal;
    cp.num_steps = p.causal ? (int)((long long)B * Hq * ((p.num_blocks + 1) / 2)) : cp.num_units;
    cp.div_tiles = attn::make_fast_div((uint32_t)p.num_blocks);
    cp.div_steps = attn::make_fast_div((uint32_t)((p.num_blocks + 1) / 2));
    cp.div_hq = p.div_hq;
    cp.div_group = p.div_group;
    cp.c = p.c;
    cp.idesc_s = p.idesc_s;
    cp.idesc_pv = p.idesc_pv;
    const long long cgrid = cp.num_steps < num_sms ? cp.num_steps : num_sms;
    switch (D) {
      case 32:
        attn::attn_fwd_colsplit_sm100<32><<<(unsigned)cgrid, attn::kCsThreads, attn::CsPlan<32>::kAlloc, s>>>(
            mq, mk, mv, mo, cp);
        break;
      case 64:
        attn::attn_fwd_colsplit_sm100<64><<<(unsigned)cgrid, attn::kCsThreads, attn::CsPlan<64>::kAlloc, s>>>(
            mq, mk, mv, mo, cp);
        break;
      case 96:
        attn::attn_fwd_colsplit_sm100<96><<<(unsigned)cgrid, attn::kCsThreads, attn::CsPlan<96>::kAlloc, s>>>(
            mq, mk, mv, mo, cp);
        break;
      default:
        attn::attn_fwd_colsplit_sm100<128><<<(unsigned)cgrid, attn::kCsThreads, attn::CsPlan<128>::kAlloc, s>>>(
            mq, mk, mv, mo, cp);
        break;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      record_cuda_error("kernel launch", e);
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }
  const Schedule sc = split ? plan0 : plan_schedule(p.num_units, p.num_steps, p.num_blocks, num_sms, p.causal, D, false);
  p.whole_per_cta = sc.whole_per_cta;
  p.tail_units = sc.tail_units;
  p.parts = sc.parts;
  p.ws_cnt = split ? reinterpret_cast<unsigned*>(workspace) : nullptr;
  p.ws_ml = split ? reinterpret_cast<float*>(static_cast<char*>(workspace) + sc.cnt_bytes) : nullptr;
  p.ws_o = split ? reinterpret_cast<float*>(static_cast<char*>(workspace) + sc.cnt_bytes + sc.ml_bytes) : nullptr;
  p.epoch = split ? next_epoch() : 0u;
  const long long grid = sc.grid;
  // O as a TMA store target for the two-tile kernel: bf16, boxes of 64 columns x 128 rows
  CUtensorMap mo;
  if ((st = encode_map(&mo, o, (long long)B * Hq, N, D, 2)) != ATTN_OK) return st;
  if (e4m3) {
    if (D == 32)
      attn::attn_fwd_sm100<32, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<32, true>::kAlloc, s>>>(
          mq, mk, mv, mo, p);
    else if (D == 64)
      attn::attn_fwd_sm100<64, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<64, true>::kAlloc, s>>>(
          mq, mk, mv, mo, p);
    else if (D == 96)
      attn::attn_fwd_sm100<96, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<96, true>::kAlloc, s>>>(
          mq, mk, mv, mo, p);
    else
      attn::attn_fwd_sm100<128, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<128, true>::kAlloc, s>>>(
          mq, mk, mv, mo, p);
  } else switch (D) {
    // non-causal D <= 64: P beside O, one MMA warp per tile (2-7 % faster there; causal units
    // are short, and there it measured 0 to 8 % slower)
    case 32:
      if (!p.causal)
        attn::attn_fwd_sm100<32, false, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<32, false, true>::kAlloc, s>>>(
            mq, mk, mv, mo, p);
      else
        attn::attn_fwd_sm100<32><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<32>::kAlloc, s>>>(mq, mk, mv, mo, p);
      break;
    case 64:
      if (!p.causal)
        attn::attn_fwd_sm100<64, false, true><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<64, false, true>::kAlloc, s>>>(
            mq, mk, mv, mo, p);
      else
        attn::attn_fwd_sm100<64><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<64>::kAlloc, s>>>(mq, mk, mv, mo, p);
      break;
    case 96:
      attn::attn_fwd_sm100<96><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<96>::kAlloc, s>>>(mq, mk, mv, mo, p);
      break;
    default:
      attn::attn_fwd_sm100<128><<<(unsigned)grid, attn::kThreads, attn::SmemPlan<128>::kAlloc, s>>>(mq, mk, mv, mo, p);
      break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("kernel launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------------------
// Entry point for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc: code whose device memory is all owned by another
// allocator (a framework's caching allocator, an embedded runtime that forbids allocation
// after start-up), or latency-critical code that must not risk the device-wide
// synchronisation an allocation can cause.  They cannot provide the workspace attn_fwd_ws
// wants for its split last wave.  attn_fwd_noalloc gives them the same kernel with the
// workspace taken from this file-scope device array instead: it exists once per device
// that loads the library and stays allocated until the process exits.
static __device__ __align__(256) unsigned char g_attn_noalloc_scratch[10u << 20];

namespace {

constexpr size_t kNoallocScratchBytes = sizeof(g_attn_noalloc_scratch);

struct NoallocScratch {
  std::mutex mu;
  void* ptr = nullptr;
};
NoallocScratch g_noalloc[kMaxDevices];

// Device address of the scratch array on `dev` (the current device).  In host code the
// array's name is only a stand-in for it, so the address is looked up once per device with
// that device current.  A failed look-up is not remembered: the next call tries again.
// The array is not cleared: device storage starts at zero when the module loads, and the
// kernel tags its counter words with a per-launch epoch and zeroes them after use, so the
// contents a previous call leaves behind are never taken for the current call's.
void* noalloc_scratch(int dev) {
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "attn_fwd_noalloc: device ordinal %d is beyond the library's limit of %d devices", dev,
                  kMaxDevices);
    return nullptr;
  }
  NoallocScratch& ns = g_noalloc[dev];
  std::lock_guard<std::mutex> lock(ns.mu);
  if (ns.ptr == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_attn_noalloc_scratch);
    if (e != cudaSuccess) {
      record_cuda_error("no-alloc scratch address look-up", e);
      return nullptr;
    }
    ns.ptr = ptr;
  }
  return ns.ptr;
}

}  // namespace

int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int N, int D, int causal, float scale, void* stream) {
  // the same host checks as attn_fwd, before any CUDA call
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0 || !std::isfinite(scale))
    return ATTN_ERR_INVALID_ARG;
  if (!supported_head_dim(D)) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return ATTN_ERR_MISALIGNED;
  const long long need = attn_fwd_workspace_bytes(B, Hq, N, D, causal);
  if (need < 0) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "workspace size query failed");
    return ATTN_ERR_CUDA;
  }
  if ((size_t)need > kNoallocScratchBytes) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "attn_fwd_noalloc: this problem needs %lld bytes of scratch, more than the %zu-byte "
                  "static array; use attn_fwd_ws with a caller workspace",
                  need, kNoallocScratchBytes);
    return ATTN_ERR_UNSUPPORTED;
  }
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error("cudaGetDevice", e);
    return ATTN_ERR_CUDA;
  }
  void* scratch = noalloc_scratch(dev);
  if (scratch == nullptr) return ATTN_ERR_CUDA;
  return launch_forward(q, k, v, o, lse, B, Hq, Hkv, N, D, causal, scale, scratch, kNoallocScratchBytes, stream);
}

size_t attn_fwd_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

int attn_device_status(void* stream, int* site) {
  if (site) *site = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    record_cuda_error("cudaStreamSynchronize", e);
    return ATTN_ERR_CUDA;
  }
  unsigned int value = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&value, attn::g_attn_fault_site, sizeof(value));
  if (e == cudaSuccess && value != 0) e = cudaMemcpyToSymbol(attn::g_attn_fault_site, &zero, sizeof(zero));
  if (e != cudaSuccess) {
    record_cuda_error("fault-site readback", e);
    return ATTN_ERR_CUDA;
  }
  if (site) *site = (int)value;
  return value ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

unsigned int attn_selftest_fast_div(unsigned int n, unsigned int d) {
  if (d == 0u) return 0u;
  const attn::FastDiv f = attn::make_fast_div(d);
  return f.m ? (unsigned int)(((unsigned __int128)n * f.m) >> 64) : n;
}

int attn_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  if (!x || !y) return ATTN_ERR_INVALID_ARG;
  const int pairs = (n + 1) / 2;
  const int threads = 256;
  attn::selftest_exp2_poly<<<(pairs + threads - 1) / threads, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, y, n);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("selftest_exp2_poly launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

int attn_selftest_wait_timeout(unsigned int timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return ATTN_ERR_INVALID_ARG;
  attn::selftest_wait_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)timeout_us * 1000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("selftest_wait_timeout launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Backward pass.

namespace {

struct BwdDeviceInfo {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
};
BwdDeviceInfo g_bwd_dev[kMaxDevices];

template <int D>
cudaError_t bwd_setup_dim() {
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_bwd_sm100<D, true>),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, attn::BwdPlan<D, true>::kAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn::attn_bwd_sm100<D, false>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, attn::BwdPlan<D, false>::kAlloc);
  // the register split (setmaxnreg) needs exactly the launch allocation it was sized for
  if (attn::BwdCfg<D>::kSplit) {
    cudaFuncAttributes fa{};
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(attn::attn_bwd_sm100<D, true>));
    if (e == cudaSuccess && fa.numRegs != attn::kRegsAtLaunch) e = cudaErrorInvalidDeviceFunction;
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(attn::attn_bwd_sm100<D, false>));
    if (e == cudaSuccess && fa.numRegs != attn::kRegsAtLaunch) e = cudaErrorInvalidDeviceFunction;
  }
  return e;
}

bool bwd_device_setup(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  BwdDeviceInfo& d = g_bwd_dev[dev];
  std::call_once(d.once, [&d] {
    cudaError_t e = bwd_setup_dim<32>();
    if (e == cudaSuccess) e = bwd_setup_dim<64>();
    if (e == cudaSuccess) e = bwd_setup_dim<96>();
    if (e == cudaSuccess) e = bwd_setup_dim<128>();
    d.err = e;
  });
  if (d.err != cudaSuccess) {
    record_cuda_error("backward device setup", d.err);
    return false;
  }
  return true;
}

// Workspace layout: -lse2 then -delta, each [B*Hq][Npad] fp32 (Npad = N rounded up to 128),
// each part 256-byte aligned.
size_t bwd_part_bytes(long long B, int Hq, int N) {
  const long long npad = ((long long)N + attn::kBlockN - 1) / attn::kBlockN * attn::kBlockN;
  return ((size_t)B * Hq * npad * sizeof(float) + 255) / 256 * 256;
}

template <int D>
void launch_bwd_dim(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                    const attn::BwdParams& pkv, const attn::BwdParams& pq, long long grid_kv, long long grid_q,
                    cudaStream_t s) {
  attn::attn_bwd_sm100<D, true><<<(unsigned)grid_kv, attn::BwdCfg<D>::kThreads, attn::BwdPlan<D, true>::kAlloc, s>>>(
      mk, mv, mq, mdo, pkv);
  attn::attn_bwd_sm100<D, false><<<(unsigned)grid_q, attn::BwdCfg<D>::kThreads, attn::BwdPlan<D, false>::kAlloc, s>>>(
      mq, mdo, mk, mv, pq);
}

}  // namespace

extern "C" {

long long attn_bwd_workspace_bytes(int B, int Hq, int N) {
  if (B < 0 || Hq < 1 || N < 0) return -1;
  if (B == 0 || N == 0) return 0;
  return (long long)(2 * bwd_part_bytes(B, Hq, N));
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int D, int causal, float scale,
             void* workspace, size_t workspace_bytes, void* stream) {
  // ---- host-side validation (no CUDA call before this block passes)
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0 || !std::isfinite(scale))
    return ATTN_ERR_INVALID_ARG;
  if (!narrow_head_dim(D)) return ATTN_ERR_UNSUPPORTED;  // the backward covers D <= 128
  // the dQ grid has B*Hq*ceil(N/128) CTAs and the prep grid twice that many blocks (< 2^31)
  if ((long long)B * Hq * (((long long)N + attn::kBlockN - 1) / attn::kBlockN) > (1LL << 30))
    return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256))
    return ATTN_ERR_MISALIGNED;
  const size_t part = bwd_part_bytes(B, Hq, N);
  if (workspace_bytes < 2 * part) return ATTN_ERR_INVALID_ARG;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error("cudaGetDevice", e);
    return ATTN_ERR_CUDA;
  }
  if (!bwd_device_setup(dev)) return ATTN_ERR_CUDA;

  CUtensorMap mq, mk, mv, mdo;
  int st;
  if ((st = encode_map(&mq, q, (long long)B * Hq, N, D)) != ATTN_OK) return st;
  if ((st = encode_map(&mk, k, (long long)B * Hkv, N, D)) != ATTN_OK) return st;
  if ((st = encode_map(&mv, v, (long long)B * Hkv, N, D)) != ATTN_OK) return st;
  if ((st = encode_map(&mdo, dout, (long long)B * Hq, N, D)) != ATTN_OK) return st;

  const int nb = (int)(((long long)N + attn::kBlockN - 1) / attn::kBlockN);
  attn::BwdParams p;
  p.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  float* nlse2 = reinterpret_cast<float*>(workspace);
  float* ndelta = reinterpret_cast<float*>(static_cast<char*>(workspace) + part);
  p.nlse2 = nlse2;
  p.ndelta = ndelta;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.Npad = nb * attn::kBlockN;
  p.group = Hq / Hkv;
  p.num_blocks = nb;
  p.causal = causal ? 1 : 0;
  p.c = scale * attn::kLog2e;
  p.scale = scale;
  p.idesc_s = attn::idesc_bf16_f32(attn::kBlockM, attn::kBlockN, false, false, false);
  p.idesc_acc = attn::idesc_bf16_f32(attn::kBlockM, D, false, true, false);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long rows = (long long)B * Hq * p.Npad;
  const int prep_threads = 256;
  const long long rows_per_block = prep_threads / 16 * attn::kPrepRows;
  const long long prep_blocks = (rows + rows_per_block - 1) / rows_per_block;
  attn::attn_bwd_prep<<<(unsigned)prep_blocks, prep_threads, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(dout), lse, nlse2, ndelta,
      rows, N, p.Npad, D);
  // Persistent CTAs (at most one per SM) walk each pass's units, 128-row blocks of a head;
  // causal units pair a head's heaviest and lightest blocks (equal items) when there are at
  // least as many pairs as SMs.
  int num_sms = 0;
  e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess || num_sms < 1) {
    record_cuda_error("cudaDeviceGetAttribute", e);
    return ATTN_ERR_CUDA;
  }
  attn::BwdParams pkv = p, pq = p;
  auto plan_pass = [&](attn::BwdParams& pp, long long heads) -> long long {
    const long long units = heads * nb, pairs = heads * ((nb + 1) / 2);
    pp.pair = (causal && pairs >= num_sms) ? 1 : 0;
    pp.num_items = (int)(pp.pair ? pairs : units);
    return pp.num_items > num_sms ? num_sms : pp.num_items;
  };
  const long long grid_kv = plan_pass(pkv, (long long)B * Hkv), grid_q = plan_pass(pq, (long long)B * Hq);
  switch (D) {
    case 32: launch_bwd_dim<32>(mq, mk, mv, mdo, pkv, pq, grid_kv, grid_q, s); break;
    case 64: launch_bwd_dim<64>(mq, mk, mv, mdo, pkv, pq, grid_kv, grid_q, s); break;
    case 96: launch_bwd_dim<96>(mq, mk, mv, mdo, pkv, pq, grid_kv, grid_q, s); break;
    default: launch_bwd_dim<128>(mq, mk, mv, mdo, pkv, pq, grid_kv, grid_q, s); break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("backward kernel launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Rotary position embedding (RoPE) of Q and K, alone and ahead of the forward pass.

namespace {

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Host checks shared by the RoPE entry points (no CUDA call).
int rope_checks(const void* q, const void* k, const float* cos_t, const float* sin_t, int B, int Hq, int Hkv,
                int N, int D) {
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0) return ATTN_ERR_INVALID_ARG;
  if (!supported_head_dim(D)) return ATTN_ERR_UNSUPPORTED;
  // rows of Q and K together below 2^32 (the kernel indexes rows in 32 bits; a bf16 tensor of
  // 2^32 rows of D >= 32 would take 256 GB): one thread per 8 rotation pairs, < 2^31 blocks
  if ((long long)B * (Hq + Hkv) * (long long)N >= (1LL << 32)) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !cos_t || !sin_t) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(cos_t, 16) || !aligned(sin_t, 16)) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

// sgn = +1: the rotation; -1: its inverse (= transpose), for gradients.
int launch_rope(const void* q, const void* k, const float* cos_t, const float* sin_t, void* q_out, void* k_out,
                int B, int Hq, int Hkv, int N, int D, cudaStream_t s, float sgn = 1.0f) {
  const long long q_rows = (long long)B * Hq * N, k_rows = (long long)B * Hkv * N;
  const long long items = (q_rows + k_rows) * (D / 16);
  const int threads = 256;
  const unsigned grid = (unsigned)((items + threads - 1) / threads);
  const attn::FastDiv div_n = attn::make_fast_div((uint32_t)N);
  const auto qb = reinterpret_cast<const __nv_bfloat16*>(q);
  const auto kb = reinterpret_cast<const __nv_bfloat16*>(k);
  const auto qo = reinterpret_cast<__nv_bfloat16*>(q_out);
  const auto ko = reinterpret_cast<__nv_bfloat16*>(k_out);
  const uint32_t qr = (uint32_t)q_rows, kr = (uint32_t)k_rows, n = (uint32_t)N;
  switch (D) {
    case 32: attn::attn_rope_qk<32><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
    case 64: attn::attn_rope_qk<64><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
    case 96: attn::attn_rope_qk<96><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
    case 128: attn::attn_rope_qk<128><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
    case 192: attn::attn_rope_qk<192><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
    default: attn::attn_rope_qk<256><<<grid, threads, 0, s>>>(qb, kb, cos_t, sin_t, qo, ko, qr, kr, n, div_n, sgn); break;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("rope kernel launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_rope_qk(const void* q, const void* k, const float* cos_t, const float* sin_t, void* q_out, void* k_out,
                 int B, int Hq, int Hkv, int N, int D, void* stream) {
  int st = rope_checks(q, k, cos_t, sin_t, B, Hq, Hkv, N, D);
  if (st != ATTN_OK || B == 0 || N == 0) return st;
  if (!q_out || !k_out) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q_out, 16) || !aligned(k_out, 16)) return ATTN_ERR_MISALIGNED;
  return launch_rope(q, k, cos_t, sin_t, q_out, k_out, B, Hq, Hkv, N, D, reinterpret_cast<cudaStream_t>(stream));
}

int attn_rope_qk_inverse(const void* dq_rot, const void* dk_rot, const float* cos_t, const float* sin_t, void* dq,
                         void* dk, int B, int Hq, int Hkv, int N, int D, void* stream) {
  int st = rope_checks(dq_rot, dk_rot, cos_t, sin_t, B, Hq, Hkv, N, D);
  if (st != ATTN_OK || B == 0 || N == 0) return st;
  if (!dq || !dk) return ATTN_ERR_INVALID_ARG;
  if (!aligned(dq, 16) || !aligned(dk, 16)) return ATTN_ERR_MISALIGNED;
  return launch_rope(dq_rot, dk_rot, cos_t, sin_t, dq, dk, B, Hq, Hkv, N, D, reinterpret_cast<cudaStream_t>(stream),
                     -1.0f);
}

long long attn_bwd_rope_workspace_bytes(int B, int Hq, int Hkv, int N, int D) {
  if (B < 0 || Hq < 1 || Hkv < 1 || N < 0 || !narrow_head_dim(D)) return -1;
  if (B == 0 || N == 0) return 0;
  const long long bwd = attn_bwd_workspace_bytes(B, Hq, N);
  if (bwd < 0) return -1;
  return (long long)(round256((size_t)B * Hq * N * D * 2) + round256((size_t)B * Hkv * N * D * 2)) + bwd;
}

int attn_bwd_rope(const void* q, const void* k, const void* v, const float* cos_t, const float* sin_t, const void* o,
                  const float* lse, const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                  int D, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  int st = rope_checks(q, k, cos_t, sin_t, B, Hq, Hkv, N, D);
  if (st != ATTN_OK) return st;
  if (!narrow_head_dim(D)) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Hq * (((long long)N + attn::kBlockN - 1) / attn::kBlockN) > (1LL << 30))
    return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;
  // every argument of the three steps is checked before the first launch
  if (!v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256))
    return ATTN_ERR_MISALIGNED;
  const size_t q_part = round256((size_t)B * Hq * N * D * 2), k_part = round256((size_t)B * Hkv * N * D * 2);
  const long long need = attn_bwd_workspace_bytes(B, Hq, N);
  if (need < 0 || workspace_bytes < q_part + k_part + (size_t)need) return ATTN_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // RoPE(q), RoPE(k) into the workspace; the attention backward on them gives the gradients with
  // respect to the rotated tensors, which the inverse rotation (the rotation's transpose) maps to
  // q and k, in place
  if ((st = launch_rope(q, k, cos_t, sin_t, ws, ws + q_part, B, Hq, Hkv, N, D, s)) != ATTN_OK) return st;
  if ((st = attn_bwd(ws, ws + q_part, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, causal, scale,
                     ws + q_part + k_part, workspace_bytes - q_part - k_part, stream)) != ATTN_OK)
    return st;
  return launch_rope(dq, dk, cos_t, sin_t, dq, dk, B, Hq, Hkv, N, D, s, -1.0f);
}

long long attn_fwd_rope_workspace_bytes(int B, int Hq, int Hkv, int N, int D) {
  if (B < 0 || Hq < 1 || Hkv < 1 || N < 0 || !supported_head_dim(D)) return -1;
  if (B == 0 || N == 0) return 0;
  const long long split = attn_fwd_workspace_bytes(B, Hq, N, D, 0);
  if (split < 0) return -1;
  return (long long)(round256((size_t)B * Hq * N * D * 2) + round256((size_t)B * Hkv * N * D * 2)) + split;
}

int attn_fwd_rope(const void* q, const void* k, const void* v, const float* cos_t, const float* sin_t, void* o,
                  float* lse, int B, int Hq, int Hkv, int N, int D, int causal, float scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int st = rope_checks(q, k, cos_t, sin_t, B, Hq, Hkv, N, D);
  if (st != ATTN_OK) return st;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return ATTN_OK;
  if (!v || !o || !lse || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) || !aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
  const size_t q_part = round256((size_t)B * Hq * N * D * 2), k_part = round256((size_t)B * Hkv * N * D * 2);
  if (workspace_bytes < q_part + k_part) return ATTN_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error("cudaGetDevice", e);
    return ATTN_ERR_CUDA;
  }
  // the split-tail workspace, if the rest of the caller's workspace holds it
  const long long need = attn_fwd_workspace_bytes(B, Hq, N, D, causal);
  if (need < 0) return ATTN_ERR_CUDA;
  const size_t rest = workspace_bytes - q_part - k_part;
  void* split_ws = (need > 0 && (size_t)need <= rest) ? ws + q_part + k_part : nullptr;
  if ((st = launch_rope(q, k, cos_t, sin_t, ws, ws + q_part, B, Hq, Hkv, N, D, s)) != ATTN_OK) return st;
  return launch_forward(ws, ws + q_part, v, o, lse, B, Hq, Hkv, N, D, causal, scale, split_ws,
                        split_ws ? rest : 0, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// RoPE angle tables, and the forward pass on host buffers.

namespace {

// Independent pieces of a [B, H, ...] problem for the host-buffer call: ranges of batch rows,
// or, for a single batch row with several KV heads, ranges of whole KV-head groups (a KV head
// and the query heads that read it).  Each piece is a contiguous block of every tensor.
struct Piece {
  long long q_off, kv_off, lse_off;  // element offsets of the piece's first q / k,v / lse entry
  int B, Hq, Hkv;                    // the piece's own problem sizes
};

int make_pieces(int B, int Hq, int Hkv, int N, int D, int want, Piece* out) {
  const int g = Hq / Hkv;
  int n = 0;
  if (B >= 2 || Hkv == 1) {
    const int k = want < B ? want : B;
    for (int i = 0; i < k; ++i) {
      const long long b0 = (long long)B * i / k, b1 = (long long)B * (i + 1) / k;
      if (b1 <= b0) continue;
      out[n++] = Piece{b0 * Hq * N * D, b0 * Hkv * N * D, b0 * Hq * N, (int)(b1 - b0), Hq, Hkv};
    }
  } else {
    const int k = want < Hkv ? want : Hkv;
    for (int i = 0; i < k; ++i) {
      const long long h0 = (long long)Hkv * i / k, h1 = (long long)Hkv * (i + 1) / k;
      if (h1 <= h0) continue;
      out[n++] = Piece{h0 * g * N * D, h0 * N * D, h0 * g * N, 1, (int)((h1 - h0) * g), (int)(h1 - h0)};
    }
  }
  return n;
}

constexpr int kMaxPieces = 64;

struct CopyStreams {
  std::mutex mu;
  cudaStream_t in = nullptr, out = nullptr;
};
CopyStreams g_copy_streams[kMaxDevices];

// The two copy streams of the host-buffer call on `dev` (the current device), created once
// (non-blocking, so they never wait for the legacy default stream).  A failure is retried by
// the next call.
bool copy_streams(int dev, cudaStream_t* in, cudaStream_t* out) {
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "device ordinal %d beyond the library's limit", dev);
    return false;
  }
  CopyStreams& cs = g_copy_streams[dev];
  std::lock_guard<std::mutex> lock(cs.mu);
  if (cs.in == nullptr) {
    cudaStream_t a = nullptr, b = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
      if (a) cudaStreamDestroy(a);
      record_cuda_error("copy stream creation", e);
      return false;
    }
    cs.in = a;
    cs.out = b;
  }
  *in = cs.in;
  *out = cs.out;
  return true;
}

}  // namespace

extern "C" {

int attn_rope_tables(float* cos_t, float* sin_t, int N, int D, double base, void* stream) {
  if (N < 0 || D < 2 || (D % 2) != 0 || !std::isfinite(base) || !(base > 0.0)) return ATTN_ERR_INVALID_ARG;
  if ((long long)N * (D / 2) > (1LL << 40)) return ATTN_ERR_UNSUPPORTED;
  if (N == 0) return ATTN_OK;
  if (!cos_t || !sin_t) return ATTN_ERR_INVALID_ARG;
  if (!aligned(cos_t, 16) || !aligned(sin_t, 16)) return ATTN_ERR_MISALIGNED;
  const long long items = (long long)N * (D / 2);
  attn::attn_rope_tables_kernel<<<(unsigned)((items + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      cos_t, sin_t, N, D, base);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error("rope tables kernel launch", e);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

long long attn_fwd_from_host_workspace_bytes(int B, int Hq, int Hkv, int N, int D, int causal, int pieces) {
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0 || pieces < 1 || !supported_head_dim(D)) return -1;
  if (B == 0 || N == 0) return 0;
  Piece pc[kMaxPieces];
  const int n = make_pieces(B, Hq, Hkv, N, D, pieces < kMaxPieces ? pieces : kMaxPieces, pc);
  long long need = 0;
  for (int i = 0; i < n; ++i) {
    const long long b = attn_fwd_workspace_bytes(pc[i].B, pc[i].Hq, N, D, causal);
    if (b < 0) return -1;
    if (b > need) need = b;
  }
  return need;
}

int attn_fwd_from_host(const void* q_host, const void* k_host, const void* v_host, void* o_host, float* lse_host,
                       void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev, void* workspace,
                       size_t workspace_bytes, int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                       int pieces, void* stream) {
  // ---- host-side validation (no CUDA call before this block passes)
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0 || !std::isfinite(scale) || pieces < 1)
    return ATTN_ERR_INVALID_ARG;
  if (!supported_head_dim(D)) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hq > 0x7fffffffLL || attn_num_units(B, Hq, N) > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q_host || !k_host || !v_host || !o_host || !lse_host || !q_dev || !k_dev || !v_dev || !o_dev || !lse_dev)
    return ATTN_ERR_INVALID_ARG;
  if (workspace == nullptr && workspace_bytes != 0) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q_dev, 16) || !aligned(k_dev, 16) || !aligned(v_dev, 16) || !aligned(o_dev, 16) ||
      !aligned(lse_dev, 4) || (workspace != nullptr && !aligned(workspace, 256)))
    return ATTN_ERR_MISALIGNED;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error("cudaGetDevice", e);
    return ATTN_ERR_CUDA;
  }
  cudaStream_t s_in = nullptr, s_out = nullptr;
  if (!copy_streams(dev, &s_in, &s_out)) return ATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  Piece pc[kMaxPieces];
  const int n = make_pieces(B, Hq, Hkv, N, D, pieces < kMaxPieces ? pieces : kMaxPieces, pc);
  // events: start, then per piece "inputs landed" and "outputs ready", then done
  cudaEvent_t ev[2 * kMaxPieces + 2];
  int made = 0;
  for (; made < 2 * n + 2; ++made) {
    e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming);
    if (e != cudaSuccess) break;
  }
  auto release = [&]() {
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  };
  if (e != cudaSuccess) {
    release();
    record_cuda_error("cudaEventCreate", e);
    return ATTN_ERR_CUDA;
  }
  cudaEvent_t ev_start = ev[0], ev_done = ev[1];
  const size_t eb = 2;  // bf16
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(o_host);
  char* lh = reinterpret_cast<char*>(lse_host);
  char* qd = static_cast<char*>(q_dev);
  char* kd = static_cast<char*>(k_dev);
  char* vd = static_cast<char*>(v_dev);
  char* od = static_cast<char*>(o_dev);
  char* ld = reinterpret_cast<char*>(lse_dev);

  int st = ATTN_OK;
  const char* what = nullptr;
  // The uploads wait for the caller's earlier work on `stream`, which may still use the
  // device buffers.
  if ((e = cudaEventRecord(ev_start, s)) != cudaSuccess) what = "cudaEventRecord";
  if (!what && (e = cudaStreamWaitEvent(s_in, ev_start, 0)) != cudaSuccess) what = "cudaStreamWaitEvent";
  for (int i = 0; i < n && !what && st == ATTN_OK; ++i) {
    const Piece& p = pc[i];
    const size_t q_bytes = (size_t)p.B * p.Hq * N * D * eb, kv_bytes = (size_t)p.B * p.Hkv * N * D * eb;
    const size_t l_bytes = (size_t)p.B * p.Hq * N * sizeof(float);
    const size_t qo = (size_t)p.q_off * eb, ko = (size_t)p.kv_off * eb, lo = (size_t)p.lse_off * sizeof(float);
    cudaEvent_t ev_in = ev[2 + 2 * i], ev_c = ev[3 + 2 * i];
    if ((e = cudaMemcpyAsync(qd + qo, qh + qo, q_bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(kd + ko, kh + ko, kv_bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(vd + ko, vh + ko, kv_bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess) {
      what = "host-to-device copy";
      break;
    }
    if ((e = cudaEventRecord(ev_in, s_in)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ev_in, 0)) != cudaSuccess) {
      what = "event record/wait";
      break;
    }
    const long long need = attn_fwd_workspace_bytes(p.B, p.Hq, N, D, causal);
    void* ws = (workspace != nullptr && need > 0 && (size_t)need <= workspace_bytes) ? workspace : nullptr;
    st = launch_forward(qd + qo, kd + ko, vd + ko, od + qo, reinterpret_cast<float*>(ld + lo), p.B, p.Hq, p.Hkv, N,
                        D, causal, scale, ws, ws ? workspace_bytes : 0, stream);
    if (st != ATTN_OK) break;
    if ((e = cudaEventRecord(ev_c, s)) != cudaSuccess || (e = cudaStreamWaitEvent(s_out, ev_c, 0)) != cudaSuccess) {
      what = "event record/wait";
      break;
    }
    if ((e = cudaMemcpyAsync(oh + qo, od + qo, q_bytes, cudaMemcpyDeviceToHost, s_out)) != cudaSuccess ||
        (e = cudaMemcpyAsync(lh + lo, ld + lo, l_bytes, cudaMemcpyDeviceToHost, s_out)) != cudaSuccess) {
      what = "device-to-host copy";
      break;
    }
  }
  if (!what && st == ATTN_OK) {
    if ((e = cudaEventRecord(ev_done, s_out)) != cudaSuccess || (e = cudaEventSynchronize(ev_done)) != cudaSuccess)
      what = "waiting for the downloads";
  } else {
    // leave nothing of this call in flight: its copies and kernels read and write the
    // caller's buffers
    cudaStreamSynchronize(s_in);
    cudaStreamSynchronize(s);
    cudaStreamSynchronize(s_out);
  }
  release();
  if (what) {
    record_cuda_error(what, e);
    return ATTN_ERR_CUDA;
  }
  return st;
}

}  // extern "C"
