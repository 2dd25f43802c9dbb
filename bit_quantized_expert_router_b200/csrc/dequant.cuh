// Packed expert format and the dequantising dot-product primitives.
//
// Format (the pages fix only "weight = nibble * scale + bias", see
// "Flash-MoE: Ausführen eines 397B-Parameter-Qwen-Modells ...", section
// "FMA-optimierter Dequant-Kernel"; the rest is this library's layout):
//   * a matrix W[N][K] stores codes as uint32 words, row-major, element k in
//     word k / (32/b) at bit b * (k mod 32/b), least significant bits first;
//   * then one 32-bit word per (row, group of 64 inputs): bf16 scale in bits
//     0..15, bf16 bias in bits 16..31;
//   * an expert blob = [gate codes | gate sb | up codes | up sb | down codes |
//     down sb]; gate and up are [I][H], down is [H][I].
//
// Evaluation.  For one row and one group G the pages rewrite
// (q*s + b) * x as fma(q, s*x, b*x); summed over the group this is
// s * sum_k q_k x_k + b * sum_k x_k.  The engine evaluates exactly that: the
// code-dependent part sum_k q_k x_k with one fused multiply-add per code, and
// the bias part with a per-vector sum of x computed once when x is staged.
//
// Decoding a code costs one bitwise AND.  A code q at bit position p of a word,
// masked in place and read as an fp32 bit pattern, is the (subnormal) number
// q * 2^(p - 149).  Staging x multiplies element k by 2^(S_v - p(k)) (exact
// powers of two, with S_v chosen per 16-byte vector from max|x|), so every
// product q * 2^(p-149) * x * 2^(S_v-p) equals q * x * 2^(S_v - 149) with one
// common scale per vector, and the FMA (which keeps subnormal operands)
// computes it with ordinary fp32 rounding.  Codes in the top byte of a word are
// first shifted down by 8 so that every masked value stays below bit 24.
#pragma once
#include "common.cuh"

namespace fmoe {

struct BlobOff {
  long long gc, gsb, uc, usb, dc, dsb, total;
};

__host__ __device__ inline BlobOff blob_offsets(int H, int I, int bits) {
  const long long cb = (long long)I * H * bits / 8;
  const long long sb = (long long)I * (H / 64) * 4;
  BlobOff o;
  o.gc = 0;
  o.gsb = cb;
  o.uc = cb + sb;
  o.usb = o.uc + cb;
  o.dc = o.usb + sb;
  o.dsb = o.dc + cb;
  o.total = o.dsb + sb;
  return o;
}

// Bit position at which code n (0 <= n < 32/b) of a word is read.
__host__ __device__ inline int code_bitpos(int bits, int n) {
  if (bits == 4) return n < 6 ? 4 * n : 4 * (n - 2);
  return n < 12 ? 2 * n : 2 * (n - 4);
}

// Eight 4-bit codes of word w against eight staged inputs (pairs xa.x, xa.y,
// xb.x, xb.y hold inputs 0-1, 2-3, 4-5, 6-7 of the word).
__device__ __forceinline__ void dot_word4(uint64_t& acc, uint32_t w, ulonglong2 xa, ulonglong2 xb) {
  const uint32_t w8 = w >> 8;
  ffma2(acc, pk_u32(w & 0xFu, w & 0xF0u), xa.x);
  ffma2(acc, pk_u32(w & 0xF00u, w & 0xF000u), xa.y);
  ffma2(acc, pk_u32(w & 0xF0000u, w & 0xF00000u), xb.x);
  ffma2(acc, pk_u32(w8 & 0xF0000u, w8 & 0xF00000u), xb.y);
}

// Sixteen 2-bit codes of word w against sixteen staged inputs.
__device__ __forceinline__ void dot_word2(uint64_t& acc, uint32_t w, ulonglong2 x0, ulonglong2 x1,
                                          ulonglong2 x2, ulonglong2 x3) {
  const uint32_t w8 = w >> 8;
  ffma2(acc, pk_u32(w & 0x3u, w & 0xCu), x0.x);
  ffma2(acc, pk_u32(w & 0x30u, w & 0xC0u), x0.y);
  ffma2(acc, pk_u32(w & 0x300u, w & 0xC00u), x1.x);
  ffma2(acc, pk_u32(w & 0x3000u, w & 0xC000u), x1.y);
  ffma2(acc, pk_u32(w & 0x30000u, w & 0xC0000u), x2.x);
  ffma2(acc, pk_u32(w & 0x300000u, w & 0xC00000u), x2.y);
  ffma2(acc, pk_u32(w8 & 0x30000u, w8 & 0xC0000u), x3.x);
  ffma2(acc, pk_u32(w8 & 0x300000u, w8 & 0xC00000u), x3.y);
}

// Bit position at which code n of a word is read, for a compile-time width.
template <int BITS>
__device__ __forceinline__ int code_bitpos_t(int n) {
  if (BITS == 4) return n < 6 ? 4 * n : 4 * (n - 2);
  return n < 12 ? 2 * n : 2 * (n - 4);
}

// Staged input for BITS-wide codes over n inputs (n a multiple of 128/BITS):
//   xs: float4 array [F4][NV] with NV = n / CPV vectors of CPV = 128/BITS
//       inputs: xs[j*NV + v] = inputs 4j..4j+3 of vector v, input k of the
//       vector multiplied by 2^(S_v - code_bitpos(k mod 32/BITS));
//   sf: float2 per vector: {sum of the vector's inputs, 2^(149 - S_v)}.
// S_v is chosen per vector from max|x| so that every staged value and every
// product with a decoded code stays a finite normal float.  The transposed
// [F4][NV] order makes lane-consecutive vectors hit consecutive shared-memory
// banks in the dot-product loops.  Several same-width inputs that lie back to
// back in memory (the routed experts' activations) can be staged in one call;
// input s's vectors are then columns s*(n_s/CPV) ... of one [F4][NV] array.
//
// Stage float4 j of vector v (q = v*F4 + j < total, else only the shuffles)
// from its four inputs `val`.  The F4 lanes of a vector are consecutive lanes
// of one warp and combine their max and sum with shuffles, so the whole warp
// calls this together.
template <int BITS>
__device__ __forceinline__ void stage_f4(float4 val, int q, int total, int NV, float4* xs, float2* sf) {
  constexpr int CPV = 128 / BITS, CPW = 32 / BITS, F4 = CPV / 4;
  const bool on = q < total;
  const int v = q / F4, j = q % F4;
  float mx = fmaxf(fmaxf(fabsf(val.x), fabsf(val.y)), fmaxf(fabsf(val.z), fabsf(val.w)));
  float sum = (val.x + val.y) + (val.z + val.w);
#pragma unroll
  for (int o = 1; o < F4; o <<= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  // max|x| * 2^S < 2^125; S in [22, 249] keeps 2^(149 - S) and 2^(S - p) finite.
  int S = 109;
  if (mx > 0.f) {
    int e;
    frexpf(mx, &e);  // mx < 2^e
    S = 125 - e;
    S = S < 22 ? 22 : (S > 249 ? 249 : S);
  }
  const float* in = &val.x;
  float4 o;
  float* out = &o.x;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    int e = S - code_bitpos_t<BITS>((4 * j + c) % CPW);  // in [0, 249]
    float t = in[c];
    if (e > 126) {
      t *= pow2f(126);
      e -= 126;
    }
    out[c] = t * pow2f(e);
  }
  if (on) {
    xs[j * NV + v] = o;
    if (j == 0) {
      const int fe = 149 - S;  // in [-100, 127]
      sf[v] = make_float2(sum, pow2f(fe));
    }
  }
}

// All threads of the CTA call this; thread q of each pass handles float4 j of
// vector v (q = v*F4 + j), so a pass costs one 16-byte load per thread.  With
// kGlobal, src is global memory read through L2 (other CTAs of the grid may
// have written it); otherwise src is this CTA's shared memory.
template <int BITS, bool kGlobal>
__device__ inline void stage_inputs(const float* __restrict__ src, int n, float4* xs, float2* sf, int tid,
                                    int nthreads) {
  constexpr int CPV = 128 / BITS, F4 = CPV / 4;
  // passes whose loads are all issued before any is used (their latencies,
  // and those of their shuffles, overlap)
  constexpr int kBatch = kGlobal ? 4 : 2;
  const int NV = n / CPV, total = NV * F4;
  const int lane = tid & 31;
  for (int base0 = tid - lane; base0 < total; base0 += kBatch * nthreads) {
    float4 val[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int q = base0 + b * nthreads + lane;
      val[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (q < total)
        val[b] = kGlobal ? __ldcg(reinterpret_cast<const float4*>(src) + q) : reinterpret_cast<const float4*>(src)[q];
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int base = base0 + b * nthreads;
      if (base >= total) break;  // warp-uniform
      stage_f4<BITS>(val[b], base + lane, total, NV, xs, sf);
    }
  }
}

// stage_inputs from a tagged source written by other CTAs of the running
// grid: word k is {tag (high 32 bits), fp32 bits of input k}.  Each thread
// issues the loads of all its float4s (two 16-byte loads each) at once, then
// re-reads those whose four words do not all carry `tag` yet, until they do
// or limit_ns has passed since the first re-read; then the warp stages them.
// Returns false if the wait ran out (the values staged are then whatever was
// read; the caller poisons its results).
template <int BITS>
__device__ inline bool stage_tagged(const unsigned long long* src, int n, float4* xs, float2* sf, int tid,
                                    int nthreads, unsigned tag, uint64_t limit_ns) {
  constexpr int CPV = 128 / BITS, F4 = CPV / 4;
  constexpr int kBatch = 4;
  const int NV = n / CPV, total = NV * F4;
  const int lane = tid & 31;
  bool ok = true;
  for (int base0 = tid - lane; base0 < total; base0 += kBatch * nthreads) {
    unsigned long long w[kBatch][4];
    unsigned pend = 0;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int q = base0 + b * nthreads + lane;
      w[b][0] = w[b][1] = w[b][2] = w[b][3] = 0ull;
      if (q < total) {
        ld_relaxed_gpu_v2u64(src + 4 * (long long)q, w[b][0], w[b][1]);
        ld_relaxed_gpu_v2u64(src + 4 * (long long)q + 2, w[b][2], w[b][3]);
        pend |= 1u << b;
      }
    }
    uint64_t t0 = 0;
    while (true) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if ((pend >> b & 1u) && (unsigned)(w[b][0] >> 32) == tag && (unsigned)(w[b][1] >> 32) == tag &&
            (unsigned)(w[b][2] >> 32) == tag && (unsigned)(w[b][3] >> 32) == tag)
          pend &= ~(1u << b);
      if (!pend) break;
      FMOE_SPIN(1);
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        ok = false;
        break;
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (pend >> b & 1u) {
          const long long q = base0 + b * nthreads + lane;
          ld_relaxed_gpu_v2u64(src + 4 * q, w[b][0], w[b][1]);
          ld_relaxed_gpu_v2u64(src + 4 * q + 2, w[b][2], w[b][3]);
        }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int base = base0 + b * nthreads;
      if (base >= total) break;  // warp-uniform
      const float4 val = make_float4(__uint_as_float((unsigned)w[b][0]), __uint_as_float((unsigned)w[b][1]),
                                     __uint_as_float((unsigned)w[b][2]), __uint_as_float((unsigned)w[b][3]));
      stage_f4<BITS>(val, base + lane, total, NV, xs, sf);
    }
  }
  return ok;
}

}  // namespace fmoe
