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

#include "sm100_ptx.cuh"

namespace attn {

// Work item = one 8-pair piece of one row; each thread takes kRopeItems items (grid-strided
// by the thread count, so a warp's accesses stay contiguous) and issues all their loads first.
// Measured on B200 (B4 H16 N2048 D128): one item per thread 4.7 TB/s, two 4.0 TB/s.
constexpr int kRopeItems = 1;
__global__ void __launch_bounds__(256) attn_rope_qk(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                    const float* __restrict__ cos_t,
                                                    const float* __restrict__ sin_t, __nv_bfloat16* q_out,
                                                    __nv_bfloat16* k_out, long long q_rows, long long k_rows,
                                                    int N, int D, float sgn) {
  const int pieces = D / 16;  // 8-pair pieces per row
  const int half = D / 2;
  const long long q_items = q_rows * pieces;
  const long long total = q_items + k_rows * pieces;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long first = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  uint4 ua[kRopeItems], ub[kRopeItems];
  float4 cv[kRopeItems][2], sv[kRopeItems][2];
#pragma unroll
  for (int u = 0; u < kRopeItems; ++u) {
    const long long item = first + u * stride;
    if (item >= total) continue;
    const bool is_q = item < q_items;
    const long long it = is_q ? item : item - q_items;
    const long long row = it / pieces;
    const int d = (int)(it - row * pieces) * 8;
    const int pos = (int)(row % N);
    const __nv_bfloat16* src = (is_q ? q : k) + row * D;
    ua[u] = *reinterpret_cast<const uint4*>(src + d);
    ub[u] = *reinterpret_cast<const uint4*>(src + half + d);
    const float4* ct = reinterpret_cast<const float4*>(cos_t + (size_t)pos * half + d);
    const float4* st = reinterpret_cast<const float4*>(sin_t + (size_t)pos * half + d);
    cv[u][0] = ct[0];
    cv[u][1] = ct[1];
    sv[u][0] = st[0];
    sv[u][1] = st[1];
  }
#pragma unroll
  for (int u = 0; u < kRopeItems; ++u) {
    const long long item = first + u * stride;
    if (item >= total) continue;
    const bool is_q = item < q_items;
    const long long it = is_q ? item : item - q_items;
    const long long row = it / pieces;
    const int d = (int)(it - row * pieces) * 8;
    __nv_bfloat16* dst = (is_q ? q_out : k_out) + row * D;
    const float cs[8] = {cv[u][0].x, cv[u][0].y, cv[u][0].z, cv[u][0].w, cv[u][1].x, cv[u][1].y, cv[u][1].z, cv[u][1].w};
    const float sn[8] = {sv[u][0].x, sv[u][0].y, sv[u][0].z, sv[u][0].w, sv[u][1].x, sv[u][1].y, sv[u][1].z, sv[u][1].w};
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&ua[u]);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&ub[u]);
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
    *reinterpret_cast<uint4*>(dst + half + d) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
  }
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
