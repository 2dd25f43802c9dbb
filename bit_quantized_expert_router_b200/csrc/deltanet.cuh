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
// So one warp owns one row, holds its dk coefficients in registers (dk / 128
// float4 per lane) for all T tokens, and reads and writes the row once per
// call: the step is a single stream over the state (HBM-bound, 8 bytes per
// state element per call).
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

constexpr int kDeltaWarps = 8;  // state rows per CTA

// dk = 128 fits 48 registers without spilling: 5 CTAs (40 warps) per SM,
// 5,920 of the pages' 8,192 state rows in flight at once; wider rows take 4
// CTAs per SM.
template <int NV4>  // float4 per lane: dk / 128
__global__ void __launch_bounds__(kDeltaWarps * 32, NV4 == 1 ? 5 : 4)
    delta_update_kernel(const __grid_constant__ DeltaArgs a) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kDeltaWarps + (threadIdx.x >> 5);
  if (row >= (long long)a.heads * a.dv) return;  // (warp-uniform)
  const int h = (int)(row / a.dv), i = (int)(row - (long long)h * a.dv);
  float4* srow = reinterpret_cast<float4*>(a.state + row * a.dk);
  float4 s[NV4];
#pragma unroll
  for (int n = 0; n < NV4; ++n) s[n] = __ldcs(srow + lane + 32 * n);  // read once: evict first
  for (int t = 0; t < a.T; ++t) {
    const long long th = (long long)t * a.heads + h;
    const float al = __ldg(a.alpha + th), be = __ldg(a.beta + th);
    const float vi = __ldg(a.v + th * a.dv + i);
    const float4* kv = reinterpret_cast<const float4*>(a.k + th * a.dk);
    const float4* qv = reinterpret_cast<const float4*>(a.q + th * a.dk);
    float4 kk[NV4], qq[NV4];
#pragma unroll
    for (int n = 0; n < NV4; ++n) {
      kk[n] = __ldg(kv + lane + 32 * n);  // shared by the dv rows of the head
      qq[n] = __ldg(qv + lane + 32 * n);
    }
    // scale, then u = S_i . k
    float u = 0.f;
#pragma unroll
    for (int n = 0; n < NV4; ++n) {
      s[n].x *= al;
      s[n].y *= al;
      s[n].z *= al;
      s[n].w *= al;
      u = fmaf(s[n].x, kk[n].x, u);
      u = fmaf(s[n].y, kk[n].y, u);
      u = fmaf(s[n].z, kk[n].z, u);
      u = fmaf(s[n].w, kk[n].w, u);
    }
    u = warp_sum(u);
    // rank-1 update of the row, then o_i = S_i . q
    const float c = be * (vi - u);
    float oi = 0.f;
#pragma unroll
    for (int n = 0; n < NV4; ++n) {
      s[n].x = fmaf(c, kk[n].x, s[n].x);
      s[n].y = fmaf(c, kk[n].y, s[n].y);
      s[n].z = fmaf(c, kk[n].z, s[n].z);
      s[n].w = fmaf(c, kk[n].w, s[n].w);
      oi = fmaf(s[n].x, qq[n].x, oi);
      oi = fmaf(s[n].y, qq[n].y, oi);
      oi = fmaf(s[n].z, qq[n].z, oi);
      oi = fmaf(s[n].w, qq[n].w, oi);
    }
    oi = warp_sum(oi);
    if (lane == 0) a.o[th * a.dv + i] = oi;
  }
#pragma unroll
  for (int n = 0; n < NV4; ++n) __stcs(srow + lane + 32 * n, s[n]);
}

}  // namespace fmoe
