// The shared expert of a multi-token step on the tensor cores.
//
// With T tokens every token uses the shared expert, so its three matrices are
// real small GEMMs: [rows x K] times [K x T].  Each CTA computes one tile of
// 128 matrix rows over 512 inputs (8 groups of 64) for all tokens:
//   part[t][row] = sum over the tile's groups G of
//                  s[row,G] * sum_{k in G} q[row,k] x[t][k]  +  b[row,G] * sum_{k in G} x[t][k],
// which is the pages' fma(q, s*x, b*x) summed over the group with s and b
// taken out of the sum ("Flash-MoE: Ausführen eines 397B-Parameter-Qwen-
// Modells ...", section "FMA-optimierter Dequant-Kernel").
//
// The code-dependent sums run on tcgen05: A = the codes as bf16 (integers
// 0..15 are exact in bf16), B = each input split into a bf16 high part and a
// bf16 low part (x = hi + lo to about 2^-17 relative), N = 32 columns (16
// token slots for hi, 16 for lo), M = 128, one K = 64 accumulation per group
// into its own 32 TMEM columns (fp32).  The epilogue reads each group's
// columns, adds the hi and lo halves, and applies the group's scale and bias
// in fp32: the weights are never rounded.
//
// Partial results per input tile are summed later in a fixed order: the gate
// and up partials where the down tiles build their input (silu(g) * u), the
// down partials in the combine.
#pragma once
#include "grouped_kernels.cuh"
#include "tc.cuh"

namespace fmoe {

constexpr int kTcRows = 128;                       // M
constexpr int kTcN = 2 * kMaxTokens;               // N
constexpr int kTcGroups = 8;                       // groups of 64 inputs per tile
constexpr int kTcK = kTcGroups * 64;               // inputs per tile
constexpr int kTcTmemCols = kTcGroups * kTcN;      // 256 fp32 columns
constexpr int kTcA = 0;                                      // [groups][128 rows x 128 B]
constexpr int kTcB = kTcA + kTcGroups * kTcRows * 128;       // [groups][32 rows x 128 B]
constexpr int kTcXsum = kTcB + kTcGroups * kTcN * 128;       // [groups][16] fp32
constexpr int kTcBar = kTcXsum + kTcGroups * kMaxTokens * 4;
constexpr int kTcTmemSlot = kTcBar + 8;
constexpr int kTcSmemBytes = kTcTmemSlot + 8 + 1024;         // + alignment slack of the dynamic base

// Two small integers (< 128) as a bf16 pair {lo, hi}, exactly: 128 + q is
// representable (bit pattern 0x4300 | q), and subtracting 128 is exact.
__device__ __forceinline__ uint32_t ints_to_bf16x2(uint32_t lo, uint32_t hi) {
  const uint32_t biased = lo | (hi << 16) | 0x43004300u;
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&biased);
  v = __hsub2(v, __floats2bfloat162_rn(128.f, 128.f));
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t floats_to_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// One tile.  All threads of the CTA call it (kThreads = 512 = 16 warps).
//   codes, row_bytes: the matrix's packed codes, row 0 input 0, bytes per row;
//   sbw, sb_row_words: its scale/bias words, words per row;
//   r0, k0: first row and first input of the tile;
//   src(t, k, v): fills v[0..15] with inputs k .. k+15 of token t (t < T);
//   out[t * ldo + r0 + r]: the tile's results, t < T.
template <int BITS, class Src>
__device__ __noinline__ void tc_tile(char* sbase, const char* __restrict__ codes, long long row_bytes,
                                     const uint32_t* __restrict__ sbw, int sb_row_words, int r0, int k0, int T,
                                     Src src, float* __restrict__ out, long long ldo, unsigned long long timeout_ns) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sbase + kTcBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sbase + kTcTmemSlot);
  float* xsum = reinterpret_cast<float*>(sbase + kTcXsum);
  if (warp == 0) {
    tmem_alloc(tslot, kTcTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_proxy_async_smem();
  }

  // A: codes -> bf16, 128-byte-swizzled K-major, one 16 KB tile per group.
  // Each thread converts kPer (row, group) blocks; all their loads are issued
  // before the first conversion.
  {
    constexpr int kPer = kTcRows * kTcGroups / kThreads;  // 2
    constexpr int kWords = 64 * BITS / 32;                // code words per block
    uint32_t w[kPer][kWords];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kThreads, g = idx % kTcGroups, r = idx / kTcGroups;
      const uint4* p = reinterpret_cast<const uint4*>(codes + (long long)(r0 + r) * row_bytes +
                                                      (long long)(k0 + g * 64) * BITS / 8);
#pragma unroll
      for (int u = 0; u < kWords / 4; ++u) {
        const uint4 v = __ldg(p + u);
        w[q][4 * u] = v.x;
        w[q][4 * u + 1] = v.y;
        w[q][4 * u + 2] = v.z;
        w[q][4 * u + 3] = v.w;
      }
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kThreads, g = idx % kTcGroups, r = idx / kTcGroups;
      char* dst = sbase + kTcA + g * (kTcRows * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // chunk c = codes 8c .. 8c+7
        uint4 o;
        if (BITS == 4) {
          const uint32_t x = w[q][c];
          o.x = ints_to_bf16x2(x & 0xFu, (x >> 4) & 0xFu);
          o.y = ints_to_bf16x2((x >> 8) & 0xFu, (x >> 12) & 0xFu);
          o.z = ints_to_bf16x2((x >> 16) & 0xFu, (x >> 20) & 0xFu);
          o.w = ints_to_bf16x2((x >> 24) & 0xFu, (x >> 28) & 0xFu);
        } else {  // half c % 2 of word c / 2
          const uint32_t x = w[q][c >> 1] >> (16 * (c & 1));
          o.x = ints_to_bf16x2(x & 3u, (x >> 2) & 3u);
          o.y = ints_to_bf16x2((x >> 4) & 3u, (x >> 6) & 3u);
          o.z = ints_to_bf16x2((x >> 8) & 3u, (x >> 10) & 3u);
          o.w = ints_to_bf16x2((x >> 12) & 3u, (x >> 14) & 3u);
        }
        *reinterpret_cast<uint4*>(dst + sw128_offset(r, 8 * c)) = o;
      }
    }
  }

  // B: warp t = token t (rows t: high parts, 16 + t: low parts), lane j =
  // inputs 16j .. 16j+15 of the tile; per-group input sums for the bias term.
  {
    const int t = warp, j = lane, g = j >> 2, ko = 16 * (j & 3);
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
    if (t < T) src(t, k0 + 16 * j, v);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) s += v[i];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if ((j & 3) == 0) xsum[g * kMaxTokens + t] = s;
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      hi[i] = *reinterpret_cast<const uint32_t*>(&h);
      const float2 hf = __bfloat1622float2(h);
      lo[i] = floats_to_bf16x2(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
    }
    char* bt = sbase + kTcB + g * (kTcN * 128);
    *reinterpret_cast<uint4*>(bt + sw128_offset(t, ko)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(bt + sw128_offset(t, ko + 8)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    *reinterpret_cast<uint4*>(bt + sw128_offset(kMaxTokens + t, ko)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(bt + sw128_offset(kMaxTokens + t, ko + 8)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
  }

  // The tensor core reads A and B through the async proxy.
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *tslot;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32<kTcRows, kTcN>();
#pragma unroll 1
    for (int g = 0; g < kTcGroups; ++g) {
      const uint64_t ad = sw128_kmajor_desc(smem_u32(sbase + kTcA + g * (kTcRows * 128)));
      const uint64_t bd = sw128_kmajor_desc(smem_u32(sbase + kTcB + g * (kTcN * 128)));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // K = 16 per instruction, 32 B along the swizzled row
        tc_mma_bf16(tbase + (uint32_t)(g * kTcN), ad + 2 * kk, bd + 2 * kk, idesc, kk > 0 ? 1u : 0u);
    }
    tc_commit(bar);
  }

  bool done = true;
  if (warp < 4) {
    const int r = warp * 32 + lane;  // tile row = TMEM lane
    uint32_t sbv[kTcGroups];
    const uint4* sp = reinterpret_cast<const uint4*>(sbw + (long long)(r0 + r) * sb_row_words + k0 / 64);
    const uint4 s0 = __ldg(sp), s1 = __ldg(sp + 1);
    sbv[0] = s0.x; sbv[1] = s0.y; sbv[2] = s0.z; sbv[3] = s0.w;
    sbv[4] = s1.x; sbv[5] = s1.y; sbv[6] = s1.z; sbv[7] = s1.w;
    done = __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0, timeout_ns));
    if (!done && lane == 0) set_status(kStatusMmaTimeout);
    tc_fence_after_sync();
    float acc[kMaxTokens];
#pragma unroll
    for (int t = 0; t < kMaxTokens; ++t) acc[t] = 0.f;
#pragma unroll 1
    for (int g = 0; g < kTcGroups; ++g) {
      uint32_t d[32];
      tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)(g * kTcN), d);
      tmem_wait_ld();
      const float sc = bf16_lo(sbv[g]), bi = bf16_hi(sbv[g]);
#pragma unroll
      for (int t = 0; t < kMaxTokens; ++t)
        acc[t] = fmaf(sc, __uint_as_float(d[t]) + __uint_as_float(d[kMaxTokens + t]),
                      fmaf(bi, xsum[g * kMaxTokens + t], acc[t]));
    }
    // results of MMAs not known complete are NaN (they reach every token)
#pragma unroll
    for (int t = 0; t < kMaxTokens; ++t)
      if (t < T) out[(long long)t * ldo + r0 + r] = done ? acc[t] : quiet_nan();
  }
  // TMEM is freed only once the MMAs are known complete (a second bounded
  // wait if the first one ran out).
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    bool ok = mbar_wait_bounded(bar, 0, timeout_ns);
    if (!ok && lane == 0) set_status(kStatusMmaTimeout);
    tc_fence_after_sync();
    tmem_dealloc(tbase, kTcTmemCols);
  }
  (void)done;
}

__device__ __forceinline__ char* align1024(char* p) {
  const uint32_t s = smem_u32(p);
  return p + ((1024u - (s & 1023u)) & 1023u);
}

// Step 1 with a tensor-core shared expert: router rows of this CTA for all
// tokens, then (CTAs below 2 * (I/128) * (H/512)) one gate or up tile.
template <int BS>
__global__ void __launch_bounds__(kThreads, 1) router_shared_gu_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];  // (aligned to 1024 below)
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  char* sbase = align1024(smem_raw);
  const int b = blockIdx.x;
  const int rows = a.E + (a.w_sgate ? 1 : 0);
  if (b * kRouterRows < rows)
    router_rows_tokens(a.w_router, a.w_sgate, a.x, a.T, a.H, a.E, b * kRouterRows, const_cast<float*>(a.logits));
  const int KSg = a.H / kTcK, nrt = a.I / kTcRows;
  if (b < 2 * nrt * KSg) {
    const int m = b / (nrt * KSg), rt = (b / KSg) % nrt, ks = b % KSg;
    const char* codes = a.shared + a.off_s[m == 0 ? 0 : 2];
    const uint32_t* sbw = reinterpret_cast<const uint32_t*>(a.shared + a.off_s[m == 0 ? 1 : 3]);
    const float* x = a.x;
    const int H = a.H;
    auto src = [x, H](int t, int k, float (&v)[16]) {
      const float4* p = reinterpret_cast<const float4*>(x + (long long)t * H + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 q = __ldg(p + i);
        v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
      }
    };
    float* out = a.sh_gu + ((long long)(m * KSg + ks) * kMaxTokens) * a.I;
    tc_tile<BS>(sbase, codes, (long long)a.H * BS / 8, sbw, a.H / 64, rt * kTcRows, ks * kTcK, a.T, src, out, a.I,
                a.timeout_ns);
  }
}

// Step 2 with a tensor-core shared expert: CTAs 0..T as the prep step, the
// others one down tile each, whose input is silu(g) * u from the gate/up
// partials (summed over the input tiles in order).
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) prep_shared_down_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];  // (aligned to 1024 below)
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  const int b = blockIdx.x;
  if (b <= a.T) {
    prep_cta<BR, BS>(a, b);
    return;
  }
  char* sbase = align1024(smem_raw);
  const int j = b - (a.T + 1), KSd = a.I / kTcK, KSg = a.H / kTcK;
  const int rt = j / KSd, ks = j % KSd;
  const float* gp = a.sh_gu;
  const float* up = a.sh_gu + (long long)KSg * kMaxTokens * a.I;
  const int I = a.I;
  // (per float4 of inputs, the partials of all input tiles are loaded together
  // and then summed in tile order)
  auto src = [gp, up, I, KSg](int t, int k, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
#pragma unroll 8
      for (int s = 0; s < KSg; ++s) {
        const long long off = ((long long)s * kMaxTokens + t) * I + k;
        const float4 a4 = __ldcg(reinterpret_cast<const float4*>(gp + off) + i);
        const float4 b4 = __ldcg(reinterpret_cast<const float4*>(up + off) + i);
        g.x += a4.x; g.y += a4.y; g.z += a4.z; g.w += a4.w;
        u.x += b4.x; u.y += b4.y; u.z += b4.z; u.w += b4.w;
      }
      v[4 * i] = g.x * sigmoidf_(g.x) * u.x;
      v[4 * i + 1] = g.y * sigmoidf_(g.y) * u.y;
      v[4 * i + 2] = g.z * sigmoidf_(g.z) * u.z;
      v[4 * i + 3] = g.w * sigmoidf_(g.w) * u.w;
    }
  };
  const char* codes = a.shared + a.off_s[4];
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(a.shared + a.off_s[5]);
  float* out = a.sh_y + (long long)ks * kMaxTokens * a.H;
  tc_tile<BS>(sbase, codes, (long long)a.I * BS / 8, sbw, a.I / 64, rt * kTcRows, ks * kTcK, a.T, src, out, a.H,
              a.timeout_ns);
}

}  // namespace fmoe
