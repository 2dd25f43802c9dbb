// Gated delta-rule update of a multi-head linear-attention state.
//
// The web pages about Flash-MoE name only the routines of this step: the
// GatedDeltaNet recurrence updates a 64-head x 128x128 state matrix with
// single-precision scale, matrix-vector and rank-1-update calls ([P2]
// "Accelerate-BLAS für lineare Aufmerksamkeit", [P3] "Uso do Accelerate
// BLAS").  Per head and token, in that order:
//   S <- alpha S;   u <- S k;   S <- S + beta (v - u) k^T;   o <- S q.
// Every row i of a head's state (the dk key coefficients of value i) is
// updated on its own: u_i = S_i . k, S_i += beta (v_i - u_i) k, o_i = S_i . q.
// So a warp owns one or two rows, holds their dk coefficients in registers
// (dk / 128 float4 per lane each) for all T tokens, and reads and writes
// each row once per call: the step is a single stream over the state
// (HBM-bound, 8 bytes per state element per call).
#pragma once

#include "common.cuh"

namespace fmoe {

struct DeltaArgs {
  float* state;        // [heads][dv][dk], updated in place
  const float* q;      // [T][heads][dk]
  const float* k;      // [T][heads][dk]
  const float* v;      // [T][heads][dv]
  const float* alpha;  // [T][heads]
  const float* beta;   // [T][heads]
  float* o;            // [T][heads][dv]
  int heads, dk, dv, T;
};

constexpr int kDeltaWarps = 8;  // warps per CTA

// State rows per warp: two at dk = 128 (both rows' loads in flight together,
// and the pages' 8,192 rows of a 64 x 128 x 128 state fit one wave of CTAs at
// 4 CTAs per SM); one for wider rows, whose registers would not hold two.
__host__ __device__ constexpr int delta_rows_per_warp(int nv4) { return nv4 == 1 ? 2 : 1; }

template <int NV4>  // float4 per lane: dk / 128
__global__ void __launch_bounds__(kDeltaWarps * 32, NV4 == 4 ? 3 : 4)
    delta_update_kernel(const __grid_constant__ DeltaArgs a) {
  constexpr int kDeltaRows = delta_rows_per_warp(NV4);
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)a.heads * a.dv;
  const long long row0 = ((long long)blockIdx.x * kDeltaWarps + (threadIdx.x >> 5)) * kDeltaRows;
  if (row0 >= rows) return;  // (warp-uniform)
  const int nr = rows - row0 >= kDeltaRows ? kDeltaRows : (int)(rows - row0);
  float4 s[kDeltaRows][NV4];
  int hh[kDeltaRows], ii[kDeltaRows];
#pragma unroll
  for (int r = 0; r < kDeltaRows; ++r) {
    const long long row = row0 + (r < nr ? r : 0);  // a missing second row repeats the first, unwritten
    hh[r] = (int)(row / a.dv);
    ii[r] = (int)(row - (long long)hh[r] * a.dv);
    const float4* srow = reinterpret_cast<const float4*>(a.state + row * a.dk);
#pragma unroll
    for (int n = 0; n < NV4; ++n) s[r][n] = __ldcs(srow + lane + 32 * n);  // read once: evict first
  }
  for (int t = 0; t < a.T; ++t) {
    float u[kDeltaRows], c[kDeltaRows], oi[kDeltaRows];
    float4 kk[kDeltaRows][NV4], qq[kDeltaRows][NV4];
    float al[kDeltaRows], be[kDeltaRows], vi[kDeltaRows];
#pragma unroll
    for (int r = 0; r < kDeltaRows; ++r) {
      const long long th = (long long)t * a.heads + hh[r];
      al[r] = __ldg(a.alpha + th);
      be[r] = __ldg(a.beta + th);
      vi[r] = __ldg(a.v + th * a.dv + ii[r]);
      const float4* kv = reinterpret_cast<const float4*>(a.k + th * a.dk);
      const float4* qv = reinterpret_cast<const float4*>(a.q + th * a.dk);
#pragma unroll
      for (int n = 0; n < NV4; ++n) {
        kk[r][n] = __ldg(kv + lane + 32 * n);  // shared by the dv rows of the head
        qq[r][n] = __ldg(qv + lane + 32 * n);
      }
    }
    // scale, then u = S_i . k
#pragma unroll
    for (int r = 0; r < kDeltaRows; ++r) {
      u[r] = 0.f;
#pragma unroll
      for (int n = 0; n < NV4; ++n) {
        s[r][n].x *= al[r];
        s[r][n].y *= al[r];
        s[r][n].z *= al[r];
        s[r][n].w *= al[r];
        u[r] = fmaf(s[r][n].x, kk[r][n].x, u[r]);
        u[r] = fmaf(s[r][n].y, kk[r][n].y, u[r]);
        u[r] = fmaf(s[r][n].z, kk[r][n].z, u[r]);
        u[r] = fmaf(s[r][n].w, kk[r][n].w, u[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kDeltaRows; ++r) u[r] = warp_sum(u[r]);
    // rank-1 update of the row, then o_i = S_i . q
#pragma unroll
    for (int r = 0; r < kDeltaRows; ++r) {
      c[r] = be[r] * (vi[r] - u[r]);
      oi[r] = 0.f;
#pragma unroll
      for (int n = 0; n < NV4; ++n) {
        s[r][n].x = fmaf(c[r], kk[r][n].x, s[r][n].x);
        s[r][n].y = fmaf(c[r], kk[r][n].y, s[r][n].y);
        s[r][n].z = fmaf(c[r], kk[r][n].z, s[r][n].z);
        s[r][n].w = fmaf(c[r], kk[r][n].w, s[r][n].w);
        oi[r] = fmaf(s[r][n].x, qq[r][n].x, oi[r]);
        oi[r] = fmaf(s[r][n].y, qq[r][n].y, oi[r]);
        oi[r] = fmaf(s[r][n].z, qq[r][n].z, oi[r]);
        oi[r] = fmaf(s[r][n].w, qq[r][n].w, oi[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kDeltaRows; ++r) oi[r] = warp_sum(oi[r]);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < kDeltaRows; ++r)
        if (r < nr) a.o[((long long)t * a.heads + hh[r]) * a.dv + ii[r]] = oi[r];
    }
  }
#pragma unroll
  for (int r = 0; r < kDeltaRows; ++r) {
    if (r < nr) {
      float4* srow = reinterpret_cast<float4*>(a.state + (row0 + r) * a.dk);
#pragma unroll
      for (int n = 0; n < NV4; ++n) __stcs(srow + lane + 32 * n, s[r][n]);
    }
  }
}

}  // namespace fmoe
