// Stand-alone router (T tokens) and the offline quantiser.
#pragma once
#include "layer_kernel.cuh"

namespace fmoe {

// logits[t][e] = W_r[e] . x[t] for e < E, and logits[t][E] = w_sg . x[t] when a
// shared-gate vector is given.  One warp per router row, all tokens; the row is
// held in registers and reused across tokens.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ w_router,
                                                            const uint16_t* __restrict__ w_sgate,
                                                            const float* __restrict__ x, int T, int H,
                                                            int E, float* __restrict__ logits) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int n_rows = E + (w_sgate ? 1 : 0);
  if (row >= n_rows) return;
  const uint16_t* r = (row < E) ? w_router + (long long)row * H : w_sgate;
  const uint4* rv = reinterpret_cast<const uint4*>(r);
  const int nv = H / 8;
  float acc[16];
  for (int t = 0; t < 16; ++t) acc[t] = 0.f;
  for (int base = 0; base < nv; base += 32 * 8) {
    uint4 w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = base + lane + 32 * i;
      if (v < nv) w[i] = ld_stream_u4(rv + v);
    }
    for (int t = 0; t < T; ++t) {
      const float4* xt = reinterpret_cast<const float4*>(x + (long long)t * H);
      float s = acc[t];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = base + lane + 32 * i;
        if (v < nv) {
          const float4 xa = __ldg(xt + 2 * v), xb = __ldg(xt + 2 * v + 1);
          s = fmaf(bf16_lo(w[i].x), xa.x, s);
          s = fmaf(bf16_hi(w[i].x), xa.y, s);
          s = fmaf(bf16_lo(w[i].y), xa.z, s);
          s = fmaf(bf16_hi(w[i].y), xa.w, s);
          s = fmaf(bf16_lo(w[i].z), xb.x, s);
          s = fmaf(bf16_hi(w[i].z), xb.y, s);
          s = fmaf(bf16_lo(w[i].w), xb.z, s);
          s = fmaf(bf16_hi(w[i].w), xb.w, s);
        }
      }
      acc[t] = s;
    }
  }
  for (int t = 0; t < T; ++t) {
    const float s = warp_sum(acc[t]);
    if (lane == 0) logits[(long long)t * (E + 1) + row] = s;
  }
}

// One warp per token: top-K, renormalised weights, shared gate.
__global__ void topk_kernel(const float* __restrict__ logits, int T, int E, int K, bool has_sgate,
                            int* __restrict__ idx, float* __restrict__ w, float* __restrict__ sgate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* lt = logits + (long long)t * (E + 1);
  warp_topk<false>(lt, E, K, lane, idx + (long long)t * K, w + (long long)t * K);
  if (lane == 0 && sgate) sgate[t] = has_sgate ? sigmoidf_(__ldcg(lt + E)) : 1.0f;
}

// Copy logits [T][E+1] -> [T][E] (drops the shared-gate column).
__global__ void copy_logits_kernel(const float* __restrict__ src, int T, int E, float* __restrict__ dst) {
  const long long n = (long long)T * E;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / E, e = i % E;
    dst[i] = src[t * (E + 1) + e];
  }
}

// Affine min/max quantiser, one thread per (row, group of 64).  Every step is
// an IEEE fp32 operation in a fixed order, so the codes are reproducible
// bit for bit: s = bf16(fl(fl(mx - mn) / (2^b - 1))), bias = bf16(mn),
// q = clamp(rint(fl(fl(w - bias) / s)), 0, 2^b - 1), q = 0 when s == 0.
__global__ void quantize_kernel(const float* __restrict__ w, int rows, int n_in, int bits,
                                uint32_t* __restrict__ codes, uint32_t* __restrict__ sb) {
  const int ng = n_in / 64;
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (gid >= (long long)rows * ng) return;
  const long long r = gid / ng;
  const int g = (int)(gid % ng);
  const float* p = w + r * n_in + (long long)g * 64;
  float mn = p[0], mx = p[0];
  for (int i = 1; i < 64; ++i) {
    mn = fminf(mn, p[i]);
    mx = fmaxf(mx, p[i]);
  }
  const float levels = (float)((1 << bits) - 1);
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), levels);
  const uint32_t sbits = f32_to_bf16_rne(s32), bbits = f32_to_bf16_rne(mn);
  const float s = __uint_as_float(sbits << 16), bb = __uint_as_float(bbits << 16);
  const int cpw = 32 / bits;
  uint32_t* crow = codes + r * (n_in * bits / 32) + (long long)g * (64 / cpw);
  for (int j = 0; j < 64 / cpw; ++j) {
    uint32_t word = 0;
    for (int n = 0; n < cpw; ++n) {
      uint32_t q = 0;
      if (s != 0.f) {
        float t = rintf(__fdiv_rn(__fsub_rn(p[j * cpw + n], bb), s));
        t = fminf(fmaxf(t, 0.f), levels);
        q = (uint32_t)t;
      }
      word |= q << (bits * n);
    }
    crow[j] = word;
  }
  sb[r * ng + g] = sbits | (bbits << 16);
}

}  // namespace fmoe
