// attn_rope_kernel.cuh -- rotary position embedding of Q and K for B200 (sm_100a).
//
// The pages list a rotary kernel among those built with the tile library ("HipKittens: fast
// and furious AMD kernels", section "Performance results") without its formula.  This one
// uses the rotate-half pairing: for the row of position p and d < D/2,
//
//   x'_d       = x_d cos(theta_pd) - x_{d+D/2} sin(theta_pd)
//   x'_{d+D/2} = x_{d+D/2} cos(theta_pd) + x_d sin(theta_pd)
//
// with cos(theta), sin(theta) taken from caller tables [N][D/2] (fp32), so that any angle
// schedule (base, scaling) can be used; the binding builds the usual
// theta_pd = p * base^(-2d/D).
//
// One pass over HBM: every row of Q [B*Hq*N] and K [B*Hkv*N] is read once and written once,
// in fp32 arithmetic rounded to bf16 (nearest even).  A thread turns 8 pairs: one 16-byte
// piece of each half of its row and the matching 32 bytes of each table row (the tables
// stay in L2: every head reads them).  The output may alias the input.
//
// With sgn = -1 the kernel applies the inverse rotation (by -theta), which is also its
// transpose: it maps gradients with respect to RoPE(q), RoPE(k) to gradients with respect to
// q, k (the backward of the rotation; sgn = +1 multiplies sin by exactly 1).
#pragma once

#include <cuda_bf16.h>

#include "attn_fwd_kernel.cuh"  // FastDiv, and the PTX wrappers

namespace attn {

// Work item = one 8-pair piece of one row, one per thread (all loads issued before any use).
// The row and the piece come from the item by a division by the compile-time piece count, the
// position in the sequence from the row by a multiply-high division by N (rows < 2^32, checked
// on the host).  Measured on B200 (B4 H16 N2048 D128): 4.96 TB/s, against 4.7 TB/s with 64-bit
// divisions by runtime values here; two items per thread measured 4.0 TB/s.
template <int D>
__global__ void __launch_bounds__(256) attn_rope_qk(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                    const float* __restrict__ cos_t,
                                                    const float* __restrict__ sin_t, __nv_bfloat16* q_out,
                                                    __nv_bfloat16* k_out, uint32_t q_rows, uint32_t k_rows,
                                                    uint32_t N, FastDiv div_n, float sgn) {
  constexpr int kPieces = D / 16;  // 8-pair pieces per row
  constexpr int kHalf = D / 2;
  const unsigned long long q_items = (unsigned long long)q_rows * kPieces;
  const unsigned long long total = q_items + (unsigned long long)k_rows * kPieces;
  const unsigned long long item = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= total) return;
  const bool is_q = item < q_items;
  const unsigned long long it = is_q ? item : item - q_items;
  const uint32_t row = (uint32_t)(it / kPieces);
  const int d = (int)(it - (unsigned long long)row * kPieces) * 8;
  const uint32_t pos = row - fast_div(row, div_n) * N;
  const __nv_bfloat16* src = (is_q ? q : k) + (size_t)row * D;
  const uint4 ua = *reinterpret_cast<const uint4*>(src + d);
  const uint4 ub = *reinterpret_cast<const uint4*>(src + kHalf + d);
  const float4* ct = reinterpret_cast<const float4*>(cos_t + (size_t)pos * kHalf + d);
  const float4* st = reinterpret_cast<const float4*>(sin_t + (size_t)pos * kHalf + d);
  const float4 c0 = ct[0], c1 = ct[1], s0 = st[0], s1 = st[1];
  __nv_bfloat16* dst = (is_q ? q_out : k_out) + (size_t)row * D;
  const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&ua);
  const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&ub);
  uint32_t oa[4], ob[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 a = __bfloat1622float2(pa[e]);
    const float2 b = __bfloat1622float2(pb[e]);
    const float c_lo = cs[2 * e], c_hi = cs[2 * e + 1], s_lo = sgn * sn[2 * e], s_hi = sgn * sn[2 * e + 1];
    oa[e] = pack_bf16x2(fmaf(a.x, c_lo, -b.x * s_lo), fmaf(a.y, c_hi, -b.y * s_hi));
    ob[e] = pack_bf16x2(fmaf(b.x, c_lo, a.x * s_lo), fmaf(b.y, c_hi, a.y * s_hi));
  }
  *reinterpret_cast<uint4*>(dst + d) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
  *reinterpret_cast<uint4*>(dst + kHalf + d) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
}

}  // namespace attn

namespace attn {

// The usual angle schedule for the tables above: theta_pd = p * base^(-2d/D) for p < N and
// d < D/2, evaluated in fp64 and stored as fp32 cos / sin.  One thread per (p, d).
__global__ void __launch_bounds__(256) attn_rope_tables_kernel(float* __restrict__ cos_t, float* __restrict__ sin_t,
                                                               int N, int D, double base) {
  const int half = D / 2;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)N * half) return;
  const int p = (int)(i / half);
  const int d = (int)(i - (long long)p * half);
  const double theta = (double)p * pow(base, -2.0 * (double)d / (double)D);
  double s, c;
  sincos(theta, &s, &c);
  cos_t[i] = (float)c;
  sin_t[i] = (float)s;
}

}  // namespace attn
