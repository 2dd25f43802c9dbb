// The single-token MoE layer as one persistent kernel (one CTA per SM).
//
// What it computes (the Flash-MoE pages): a router GEMV over the experts, then
// softmax, top-K and renormalised weights ("Flash-MoE: Ausführen eines
// 397B-Parameter-Qwen-Modells ...", section "Pipeline-Leistung"); the selected
// experts plus one shared expert as dequantised GEMVs, gate and up, fused
// SwiGLU, then down (section "Metal-Compute-Shader"); and a fused end step,
// out = residual + sum_k w_k y_k + sigmoid(w_sg . x) * y_shared (same section,
// "MoE-Kombination + Rest + Sigmoid-Gate").  The weights are affine
// group-quantised and evaluated in the pages' FMA form (dequant.cuh).
//
// How it runs on B200.
//   Input-stationary warps.  A row of n inputs is cut into slices of 1024
//   inputs; lane L of the warp that owns slice q holds inputs
//   [1024 q + 32 L, +32) of x in registers, staged once for the code width,
//   and reads the codes of those inputs straight from memory into registers
//   (one 16-byte load per row at 4 bits, 8 bytes at 2 bits).  Neither the
//   inputs nor the codes pass through shared memory, so its bandwidth is not
//   a limit.  The P slices of a row are computed by a group of P warps; the
//   last of them to finish (a shared-memory counter) adds the slice sums in
//   slice order.
//   Balanced units.  The gate/up rows of each expert ("units") are dealt
//   round-robin over the CTAs, and inside a CTA round-robin over its warp
//   groups, so every CTA gets the same number of units to within one and
//   every group to within one of those.
//   Hand-offs without barriers.  Router logits and SwiGLU activations are
//   published as 64-bit words {tag, fp32 bits} in the workspace, the tag being
//   this launch's number (the workspace's epoch + 1); a consumer polls the
//   words it needs until they carry the tag, so each hand-off costs one
//   round trip through L2 and no grid barrier.
//   Order of work in a CTA:
//     before the previous kernel on the stream has finished (a programmatic
//     dependent launch): its router row slices and first shared-expert units
//     are loaded into registers, and L2 is asked for the rest of its shared
//     expert rows;
//     x -> router dot products -> logits published; the shared expert's
//     gate/up units -> activations published;
//     the first warp through its shared units takes the routing decision
//     (polls all logits, top-K, weights) for its CTA;
//     L2 is asked for this CTA's routed gate/up rows and down rows;
//     while they stream: the shared expert's down rows (its activations are
//     already published);
//     the routed gate/up units (a register ring of loads ahead) -> activations;
//     each routed expert's down rows as soon as its activations are all
//     published; the combine over this CTA's block of output rows.
//   Every wait is time-limited: on expiry a status bit is set, the CTA
//   publishes and writes NaN from then on (so no output built on a missing
//   value looks plausible) and carries on to its end.  No float atomics: every
//   sum has a fixed order, so results are bitwise reproducible.
#pragma once
#include "routing.cuh"

namespace fmoe {

constexpr int kRing = 3;       // gate/up units whose codes a warp holds in registers ahead
constexpr int kDownChunk = 4;  // down rows a warp loads at once
constexpr unsigned kEpochLimit = 0x7FFFFFFFu;  // valid epochs are below this; tags are epoch + 1

// Optional phase trace (compile with -DFMOE_TRACE_BUILD): per CTA, the latest
// %globaltimer over its warps at fixed points of the kernel.
#ifdef FMOE_TRACE_BUILD
constexpr int kTracePoints = 16;
__device__ unsigned long long g_fmoe_trace[1024][kTracePoints];
#define FMOE_TRACE_WARP(i) \
  do { if ((threadIdx.x & 31) == 0 && blockIdx.x < 1024) \
    atomicMax(&g_fmoe_trace[blockIdx.x][i], (unsigned long long)globaltimer_ns()); } while (0)
#else
#define FMOE_TRACE_WARP(i) do { } while (0)
#endif

struct DecodeArgs {
  const uint16_t* w_router;  // [E][H] bf16 bits (null when the routing is given)
  const uint16_t* w_sgate;   // [H] bf16 bits, or null (ungated shared expert)
  const char* experts;       // E routed blobs, blob e at experts + e * expert_stride
  long long expert_stride;
  const char* shared;        // shared expert blob (or the single expert), or null
  const float* x;            // [H]
  const float* residual;     // [H] or null
  float* out;                // [H]
  const uint16_t* norm_w;    // [H] bf16 RMS-norm weight of the input, or null
  float norm_eps;
  unsigned* bar;             // workspace counters: [0] launch epoch, [2] done ticket
  unsigned long long* tlog;  // workspace: tagged router logits [n_router]
  unsigned long long* tact;  // workspace: tagged activations [K + 1][I] (slot K = shared)
  int* idx_out;              // optional [K]
  float* w_out;              // optional [K]
  float* sg_out;             // optional [1]
  // Given routing (no router): the blob and weight of each routed slot and
  // the shared gate.
  const char* fixed_blob[kMaxTopK];
  float fixed_w[kMaxTopK];
  float fixed_sg;
  int fixed_route;
  int H, I, E, K, bits_r, bits_s;
  int n_router;              // router rows: E (+1 with w_sgate); 0 with a given routing or one expert
  int has_shared;
  int off_sh, off_ro;        // CTA offsets of the round-robin shared and routed unit lists
  long long off_r[6], off_s[6];  // blob section offsets for the routed / shared code width
  // dynamic shared memory layout (byte offsets) and its sizes
  int sm_norm, sm_abuf, sm_abuf_stride, sm_upart, sm_ucnt, sm_rpart, sm_rcnt, sm_ysp;
  int max_units, max_rrows, max_drows;
  unsigned long long timeout_ns;
};

// Per-CTA state (static shared memory).
struct DecodeShared {
  uint64_t x_bar;      // completes once x (and the norm weight) is in shared memory
  uint64_t route_bar;  // completes once the routing decision is in idx / w / sg / blob
  int route_claim;     // the first warp through its shared units takes the routing decision
  int poison;          // a wait of this CTA ran out: what it publishes or writes is NaN
  int last;            // this CTA took the launch's last ticket
  float red[kWarps];
  int idx[kMaxTopK];
  float w[kMaxTopK];
  float sg;
  const char* blob[kMaxSlots];
};

// ---------------------------------------------------------------------------
// Small pieces
// ---------------------------------------------------------------------------

__device__ __forceinline__ int mod_pos(int a, int m) {
  const int r = a % m;
  return r < 0 ? r + m : r;
}
// Items of a round-robin list of n items, item u to CTA (u + off) mod G: the
// first item of CTA c is (c - off) mod G and there are count_from(n, first, G).
__device__ __forceinline__ int count_from(int n, int first, int G) { return n > first ? (n - first - 1) / G + 1 : 0; }

__device__ __forceinline__ uint2 ld_stream_u2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ void ld_relaxed_gpu_v2u64(const unsigned long long* p, unsigned long long& a,
                                                     unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0,%1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
// L2 prefetch of [p, p + bytes) widened to 16-byte boundaries inside
// [lo, hi) (the section the range lies in, itself 16-byte aligned).
__device__ __forceinline__ void prefetch_l2_in(const char* p, long long bytes, const char* lo, const char* hi) {
  const char* a = reinterpret_cast<const char*>(reinterpret_cast<uintptr_t>(p) & ~uintptr_t(15));
  const char* b = reinterpret_cast<const char*>((reinterpret_cast<uintptr_t>(p + bytes) + 15) & ~uintptr_t(15));
  if (a < lo) a = lo;
  if (b > hi) b = hi;
  while (b - a > 0) {
    const long long n = (b - a) > (1 << 20) ? (1 << 20) : (b - a);
    bulk_prefetch_l2(a, (uint32_t)n);
    a += n;
  }
}
__device__ __forceinline__ float quiet_nan() { return __uint_as_float(0x7FC00000u); }

// Exponent e with |v| < 2^e for a positive finite v (subnormals: e = -126).
__device__ __forceinline__ int exp_above(float v) {
  const int E = (int)((__float_as_uint(v) >> 23) & 0xFF);
  return E == 0 ? -126 : E - 126;
}

// One vector of 32 inputs staged for BITS-wide codes (see dequant.cuh):
// xp[m] = {in[2m], in[2m+1]} with in[k] = x[k] * 2^(S - bitpos(k)), S from
// max|x| over the vector; f = 2^(149 - S); sum = the plain sum of the inputs.
struct LaneX {
  uint64_t xp[16];
  float f, sum;
};

template <int BITS>
__device__ __forceinline__ void stage_lane(const float (&x)[32], LaneX& s) {
  float mx = 0.f, p[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    p[m] = x[2 * m] + x[2 * m + 1];
    mx = fmaxf(mx, fmaxf(fabsf(x[2 * m]), fabsf(x[2 * m + 1])));
  }
#pragma unroll
  for (int w = 8; w > 0; w >>= 1)
#pragma unroll
    for (int m = 0; m < w; ++m) p[m] += p[m + w];
  int S = 109;
  if (mx > 0.f) {
    S = 125 - exp_above(mx);
    S = S < 22 ? 22 : (S > 249 ? 249 : S);
  }
  float st[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    int e = S - code_bitpos_t<BITS>(k % (32 / BITS));  // in [0, 249]
    float t = x[k];
    if (e > 126) {
      t *= pow2f(126);
      e -= 126;
    }
    st[k] = t * pow2f(e);
  }
#pragma unroll
  for (int m = 0; m < 16; ++m) s.xp[m] = pk_u32(__float_as_uint(st[2 * m]), __float_as_uint(st[2 * m + 1]));
  s.f = pow2f(149 - S);
  s.sum = p[0];
}

// Dot product of one vector's codes with its staged inputs (unscaled: times
// 2^(S - 149) in the staged scale).  Two accumulators halve the chain.
template <int BITS>
__device__ __forceinline__ float vec_dot(const uint4& c, const LaneX& X) {
  uint64_t a0 = 0, a1 = 0;
  if (BITS == 4) {
    dot_word4(a0, c.x, make_ulonglong2(X.xp[0], X.xp[1]), make_ulonglong2(X.xp[2], X.xp[3]));
    dot_word4(a1, c.y, make_ulonglong2(X.xp[4], X.xp[5]), make_ulonglong2(X.xp[6], X.xp[7]));
    dot_word4(a0, c.z, make_ulonglong2(X.xp[8], X.xp[9]), make_ulonglong2(X.xp[10], X.xp[11]));
    dot_word4(a1, c.w, make_ulonglong2(X.xp[12], X.xp[13]), make_ulonglong2(X.xp[14], X.xp[15]));
  } else {
    dot_word2(a0, c.x, make_ulonglong2(X.xp[0], X.xp[1]), make_ulonglong2(X.xp[2], X.xp[3]),
              make_ulonglong2(X.xp[4], X.xp[5]), make_ulonglong2(X.xp[6], X.xp[7]));
    dot_word2(a1, c.y, make_ulonglong2(X.xp[8], X.xp[9]), make_ulonglong2(X.xp[10], X.xp[11]),
              make_ulonglong2(X.xp[12], X.xp[13]), make_ulonglong2(X.xp[14], X.xp[15]));
  }
  const float2 d0 = unpk_f32(a0), d1 = unpk_f32(a1);
  return (d0.x + d0.y) + (d1.x + d1.y);
}

// The lane's share of one row: s * (sum_k q_k x_k) + b * (sum_k x_k) over its
// 32 inputs, with (s, b) the bf16 pair of the inputs' quantisation group.
template <int BITS>
__device__ __forceinline__ float vec_row(const uint4& c, uint32_t sb, const LaneX& X) {
  return fmaf(bf16_lo(sb) * X.f, vec_dot<BITS>(c, X), bf16_hi(sb) * X.sum);
}

// Codes (16 bytes at 4 bits, 8 at 2 bits) and the (s, b) word of vector v of
// a row whose codes start at `codes` and whose (s, b) words start at `sbw`.
template <int BITS>
__device__ __forceinline__ void load_vec(const char* codes, const char* sbw, int v, uint4& c, uint32_t& sb) {
  if (BITS == 4) {
    c = ld_stream_u4(codes + (long long)v * 16);
  } else {
    const uint2 t = ld_stream_u2(codes + (long long)v * 8);
    c = make_uint4(t.x, t.y, 0u, 0u);
  }
  sb = ld_stream_u32(sbw + (long long)(v >> 1) * 4);
}

struct UnitRegs {
  uint4 cg, cu;
  uint32_t sg, su;
};

// ---------------------------------------------------------------------------
// Geometry of one CTA's work (the same for all warps of a launch)
// ---------------------------------------------------------------------------
struct Geo {
  int G, c, warp, lane, tid;
  int P, n_grp, grp, q, vx;  // gate/up and router: slices per row, groups, my group and slice, my vector
  bool gon, xon;             // my warp has a group; my lane's vector exists
  int n_sh_c, sh_first, n_ro_c, ro_first, n_rr_c;
  int r0, nrow;              // this CTA's block of output rows
};

__device__ __forceinline__ Geo make_geo(const DecodeArgs& a) {
  Geo g;
  g.G = gridDim.x;
  g.c = blockIdx.x;
  g.tid = threadIdx.x;
  g.lane = g.tid & 31;
  g.warp = g.tid >> 5;
  const int nv = a.H / 32;
  g.P = (nv + 31) / 32;
  g.n_grp = kWarps / g.P;
  g.grp = g.warp / g.P;
  g.q = g.warp % g.P;
  g.gon = g.grp < g.n_grp;
  g.vx = g.q * 32 + g.lane;
  g.xon = g.gon && g.vx < nv;
  g.sh_first = mod_pos(g.c - a.off_sh, g.G);
  g.n_sh_c = count_from(a.has_shared ? a.I : 0, g.sh_first, g.G);
  g.ro_first = mod_pos(g.c - a.off_ro, g.G);
  g.n_ro_c = count_from(a.K * a.I, g.ro_first, g.G);
  g.n_rr_c = count_from(a.n_router, g.c, g.G);
  g.r0 = (int)((long long)g.c * a.H / g.G);
  g.nrow = (int)((long long)(g.c + 1) * a.H / g.G) - g.r0;
  return g;
}

// ---------------------------------------------------------------------------
// Gate/up units
// ---------------------------------------------------------------------------

// (blob, row, slot) of unit i of my warp's shared list or routed list, and
// its CTA-local index (for the slice partials).
struct UnitRef {
  const char* blob;
  int row, slot, j;
};
__device__ __forceinline__ UnitRef shared_unit(const DecodeArgs& a, const DecodeShared& cs, const Geo& g, int i) {
  UnitRef u;
  u.j = g.grp + g.n_grp * i;
  u.row = g.sh_first + g.G * u.j;
  u.slot = a.K;
  u.blob = cs.blob[a.K];
  return u;
}
__device__ __forceinline__ int routed_base(const Geo& g) { return mod_pos(g.grp - g.n_sh_c, g.n_grp); }
__device__ __forceinline__ UnitRef routed_unit(const DecodeArgs& a, const DecodeShared& cs, const Geo& g, int i) {
  UnitRef u;
  const int jr = routed_base(g) + g.n_grp * i;
  const int uu = g.ro_first + g.G * jr;
  u.slot = uu / a.I;
  u.row = uu - u.slot * a.I;
  u.j = g.n_sh_c + jr;
  u.blob = cs.blob[u.slot];
  return u;
}
__device__ __forceinline__ int my_shared_units(const Geo& g) {
  return g.gon ? count_from(g.n_sh_c, g.grp, g.n_grp) : 0;
}
__device__ __forceinline__ int my_routed_units(const Geo& g) {
  return g.gon ? count_from(g.n_ro_c, routed_base(g), g.n_grp) : 0;
}

template <int BITS>
__device__ __forceinline__ void load_unit(const DecodeArgs& a, const UnitRef& u, const long long* o, const Geo& g,
                                          UnitRegs& R) {
  R.cg = R.cu = make_uint4(0u, 0u, 0u, 0u);
  R.sg = R.su = 0u;
  if (!g.xon) return;
  const long long cb = (long long)a.H * BITS / 8, sbr = a.H / 16;
  load_vec<BITS>(u.blob + o[0] + u.row * cb, u.blob + o[1] + u.row * sbr, g.vx, R.cg, R.sg);
  load_vec<BITS>(u.blob + o[2] + u.row * cb, u.blob + o[3] + u.row * sbr, g.vx, R.cu, R.su);
}

// Publish one tagged 64-bit word {tag, value}.
__device__ __forceinline__ void publish(unsigned long long* p, unsigned tag, float v) {
  st_relaxed_gpu_u64(p, ((unsigned long long)tag << 32) | __float_as_uint(v));
}

// One gate/up unit of my slice: the slice's gate and up sums; the last slice
// warp of the group to finish adds all slices in slice order and publishes
// silu(g) * u.
template <int BITS>
__device__ __forceinline__ void unit_compute(const DecodeArgs& a, DecodeShared& cs, const Geo& g, char* smem,
                                             const UnitRef& u, const UnitRegs& R, const LaneX& X, unsigned tag) {
  float gv = 0.f, uv = 0.f;
  if (g.xon) {
    gv = vec_row<BITS>(R.cg, R.sg, X);
    uv = vec_row<BITS>(R.cu, R.su, X);
  }
  const float v = warp_sum2_split(gv, uv, g.lane);  // g on lanes 0..15, u on 16..31
  const float ut = __shfl_sync(0xffffffffu, v, 16);
  if (g.lane == 0) {
    float gs = v, us = ut;
    bool last = true;
    if (g.P > 1) {
      float2* part = reinterpret_cast<float2*>(smem + a.sm_upart) + u.j * g.P;
      int* cnt = reinterpret_cast<int*>(smem + a.sm_ucnt) + u.j;
      part[g.q] = make_float2(gs, us);
      __threadfence_block();
      last = atomicAdd(cnt, 1) == g.P - 1;
      if (last) {
        __threadfence_block();
        gs = 0.f;
        us = 0.f;
        const volatile float* pv = reinterpret_cast<const volatile float*>(part);
        for (int s = 0; s < g.P; ++s) {
          gs += pv[2 * s];
          us += pv[2 * s + 1];
        }
      }
    }
    if (last) {
      const float act = cs.poison ? quiet_nan() : gs * sigmoidf_(gs) * us;
      publish(a.tact + (long long)u.slot * a.I + u.row, tag, act);
    }
  }
}

// The units of one list (shared or routed), with kRing of them loaded ahead
// in registers.  R holds the first kRing units' loads on entry.
template <int BITS, bool kRouted>
__device__ __forceinline__ void unit_loop(const DecodeArgs& a, DecodeShared& cs, const Geo& g, char* smem, int n,
                                          UnitRegs (&R)[kRing], const LaneX& X, unsigned tag) {
  const long long* o = (kRouted && a.K > 0) ? a.off_r : a.off_s;
  for (int base = 0; base < n; base += kRing) {
#pragma unroll
    for (int d = 0; d < kRing; ++d) {
      const int i = base + d;
      if (i < n) {
        const UnitRef u = kRouted ? routed_unit(a, cs, g, i) : shared_unit(a, cs, g, i);
        unit_compute<BITS>(a, cs, g, smem, u, R[d], X, tag);
        if (i + kRing < n) {
          const UnitRef un = kRouted ? routed_unit(a, cs, g, i + kRing) : shared_unit(a, cs, g, i + kRing);
          load_unit<BITS>(a, un, o, g, R[d]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Router rows
// ---------------------------------------------------------------------------

// The lane's 32 bf16 router weights against its 32 raw inputs.
__device__ __forceinline__ float router_lane_dot(const uint4 (&w)[4], const float (&x)[32]) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t* ww = &w[i].x;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      s0 = fmaf(bf16_lo(ww[h]), x[8 * i + 2 * h], s0);
      s1 = fmaf(bf16_hi(ww[h]), x[8 * i + 2 * h + 1], s1);
    }
  }
  return s0 + s1;
}

__device__ __forceinline__ const uint16_t* router_row(const DecodeArgs& a, int e) {
  return e < a.E ? a.w_router + (long long)e * a.H : a.w_sgate;
}
__device__ __forceinline__ void load_router(const DecodeArgs& a, const Geo& g, int e, uint4 (&w)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
  if (!g.xon) return;
  const uint4* p = reinterpret_cast<const uint4*>(router_row(a, e) + (long long)g.vx * 32);
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = ld_stream_u4(p + i);
}

// My group's router rows (CTA-local rows grp, grp + n_grp, ...): each slice
// sum goes to shared memory; the last slice warp adds them in slice order and
// publishes the logit.  w0 holds the first row's weights (loaded early).
__device__ __forceinline__ void router_rows(const DecodeArgs& a, DecodeShared& cs, const Geo& g, char* smem,
                                            uint4 (&w)[4], const float (&x)[32], unsigned tag) {
  if (!g.gon) return;
  for (int jr = g.grp; jr < g.n_rr_c; jr += g.n_grp) {
    const int e = g.c + g.G * jr;
    if (jr != g.grp) load_router(a, g, e, w);
    const float s = warp_sum(router_lane_dot(w, x));
    if (g.lane == 0) {
      float tot = s;
      bool last = true;
      if (g.P > 1) {
        float* part = reinterpret_cast<float*>(smem + a.sm_rpart) + jr * g.P;
        int* cnt = reinterpret_cast<int*>(smem + a.sm_rcnt) + jr;
        part[g.q] = s;
        __threadfence_block();
        last = atomicAdd(cnt, 1) == g.P - 1;
        if (last) {
          __threadfence_block();
          tot = 0.f;
          for (int q = 0; q < g.P; ++q) tot += *reinterpret_cast<volatile float*>(part + q);
        }
      }
      if (last) publish(a.tlog + e, tag, cs.poison ? quiet_nan() : tot);
    }
  }
}

// ---------------------------------------------------------------------------
// Routing decision (one warp)
// ---------------------------------------------------------------------------

// Order-preserving 32-bit key of a logit: larger key = larger logit; NaN
// (a poisoned logit) orders above every number.
__device__ __forceinline__ uint32_t logit_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Poll the E router logits (NK per lane: expert i * 32 + lane) and, on lane 0,
// the shared gate's logit; take the top K (descending logit, lower index on
// exact ties); weights exp(l_k - l_0) / sum_j exp(l_j - l_0) (softmax over
// the selected experts, equal to softmax then renormalise); sigmoid gate.
template <int NK>
__device__ void route_warp(const DecodeArgs& a, DecodeShared& cs, const Geo& g, unsigned tag) {
  const int lane = g.lane;
  uint32_t key[NK];
  uint64_t pend = 0;  // bit i: word i still to come (bit NK: the shared gate's)
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    key[i] = 0u;
    if (i * 32 + lane < a.E) pend |= 1ull << i;
  }
  const bool has_gate = a.w_sgate != nullptr;
  if (lane == 0 && has_gate) pend |= 1ull << NK;
  float gate_logit = 0.f;
  bool timed_out = cs.poison != 0;  // (a poisoned CTA does not wait again)
  uint64_t t0 = 0;
  while (pend && !timed_out) {
    unsigned long long v[NK + 1];
#pragma unroll
    for (int i = 0; i <= NK; ++i) {
      const int e = i < NK ? i * 32 + lane : a.E;
      v[i] = (pend >> i & 1ull) ? ld_relaxed_gpu_u64(a.tlog + e) : 0ull;
    }
#pragma unroll
    for (int i = 0; i <= NK; ++i) {
      if ((pend >> i & 1ull) && tag != 0u && (unsigned)(v[i] >> 32) == tag) {
        const float l = __uint_as_float((unsigned)v[i]);
        if (i < NK) key[i] = logit_key(l); else gate_logit = l;
        pend &= ~(1ull << i);
      }
    }
    if (!pend) break;
    const uint64_t now = globaltimer_ns();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > a.timeout_ns) {
      timed_out = true;
      break;
    }
  }
  if (__any_sync(0xffffffffu, timed_out)) {
    if (lane == 0) {
      set_status(kStatusGridBarrierTimeout);
      cs.poison = 1;
    }
  }
  // Top-K: per round the largest key, and among equal keys the lowest expert
  // index; only the lane that holds the winner rescans its keys.
  uint32_t mk = key[0];
  int mp = 0;
#pragma unroll
  for (int i = 1; i < NK; ++i)
    if (key[i] > mk) { mk = key[i]; mp = i; }
  uint32_t out_key = 0u, out_idx = 0u;
  for (int kk = 0; kk < a.K; ++kk) {
    const uint32_t h = __reduce_max_sync(0xffffffffu, mk);
    const uint32_t e = __reduce_min_sync(0xffffffffu, mk == h ? (uint32_t)(mp * 32 + lane) : 0xffffffffu);
    if (mk == h && (uint32_t)(mp * 32 + lane) == e) {
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (i == mp) key[i] = 0u;
      mk = key[0];
      mp = 0;
#pragma unroll
      for (int i = 1; i < NK; ++i)
        if (key[i] > mk) { mk = key[i]; mp = i; }
    }
    if (lane == kk) {
      out_key = h;
      out_idx = e;
    }
  }
  const float val = lane < a.K ? __uint_as_float((out_key & 0x80000000u) ? (out_key & 0x7FFFFFFFu) : ~out_key) : 0.f;
  const float l0 = __shfl_sync(0xffffffffu, val, 0);
  const float ex = lane < a.K ? expf(val - l0) : 0.f;
  const float ssum = warp_sum(ex);
  const bool poisoned = cs.poison != 0;
  if (lane < a.K) {
    const int idx = out_idx < (uint32_t)a.E ? (int)out_idx : 0;  // (always in range)
    const float w = poisoned ? quiet_nan() : ex / ssum;
    cs.idx[lane] = idx;
    cs.w[lane] = w;
    cs.blob[lane] = a.experts + (long long)idx * a.expert_stride;
    if (g.c == 0) {
      if (a.idx_out) a.idx_out[lane] = poisoned ? -1 : idx;
      if (a.w_out) a.w_out[lane] = w;
    }
  }
  if (lane == 0) {
    cs.sg = poisoned ? quiet_nan() : (has_gate ? sigmoidf_(gate_logit) : 1.0f);
    if (g.c == 0 && a.sg_out) *a.sg_out = cs.sg;
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Down projection of one slot over this CTA's block of output rows
// ---------------------------------------------------------------------------

// Every thread of the CTA calls this for the same slots in the same order.
//   1. my warp's first rows' codes are requested;
//   2. the slot's I activations are polled (two tagged words per thread) and
//      staged for the code width into the slot's buffer (vectors of 32,
//      16 threads each);
//   3. CTA barrier;
//   4. my warp's rows: the partial of my slice of each row goes to ysp.
template <int BD>
__device__ void down_step(const DecodeArgs& a, DecodeShared& cs, const Geo& g, char* smem, int s, unsigned tag) {
  const int I = a.I, nvi = I / 32;
  const int Pd = (nvi + 31) / 32, ngd = kWarps / Pd;
  const int gd = g.warp / Pd, qd = g.warp % Pd;
  const int v = qd * 32 + g.lane;
  const bool dw = gd < ngd, von = dw && v < nvi;
  const char* blob = cs.blob[s];
  const long long* o = s < a.K ? a.off_r : a.off_s;
  const long long cbI = (long long)I * BD / 8, sbI = I / 16;
  // 1. codes of my first rows
  uint4 dc[kDownChunk];
  uint32_t ds[kDownChunk];
#pragma unroll
  for (int i = 0; i < kDownChunk; ++i) {
    const int rho = gd + ngd * i;
    dc[i] = make_uint4(0u, 0u, 0u, 0u);
    ds[i] = 0u;
    if (von && rho < g.nrow) {
      const long long r = g.r0 + rho;
      load_vec<BD>(blob + o[4] + r * cbI, blob + o[5] + r * sbI, v, dc[i], ds[i]);
    }
  }
  // 2. activations of slot s, staged
  float* ab = reinterpret_cast<float*>(smem + a.sm_abuf + (s & 1) * a.sm_abuf_stride);
  float2* sfa = reinterpret_cast<float2*>(ab + I);
  const unsigned long long* src = a.tact + (long long)s * I;
  for (int base = 0; base < I; base += 2 * kThreads) {
    const int k = base + 2 * g.tid;  // even element index
    float a0 = 0.f, a1 = 0.f;
    if (k < I) {
      // (once this CTA is poisoned its results are NaN anyway: no more waiting)
      bool done = false, timed_out = cs.poison != 0;
      uint64_t t0 = 0;
      while (!timed_out) {
        unsigned long long w0, w1;
        ld_relaxed_gpu_v2u64(src + k, w0, w1);
        if (tag != 0u && (unsigned)(w0 >> 32) == tag && (unsigned)(w1 >> 32) == tag) {
          a0 = __uint_as_float((unsigned)w0);
          a1 = __uint_as_float((unsigned)w1);
          done = true;
        }
        if (done) break;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > a.timeout_ns) {
          timed_out = true;
          break;
        }
      }
      if (timed_out) {
        if (!cs.poison) set_status(kStatusGridBarrierTimeout);
        cs.poison = 1;
        a0 = a1 = quiet_nan();
      }
    }
    // vector k / 32 is held by 16 consecutive threads (a half warp)
    float mx = fmaxf(fabsf(a0), fabsf(a1)), sm = a0 + a1;
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      sm += __shfl_xor_sync(0xffffffffu, sm, off);
    }
    if (k < I) {
      int S = 109;
      if (mx > 0.f) {
        S = 125 - exp_above(mx);
        S = S < 22 ? 22 : (S > 249 ? 249 : S);
      }
      const int kk = k & 31, vv = k >> 5;
      float t[2] = {a0, a1};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int e = S - code_bitpos_t<BD>((kk + h) % (32 / BD));
        if (e > 126) {
          t[h] *= pow2f(126);
          e -= 126;
        }
        t[h] *= pow2f(e);
      }
      // element kk of vector vv lives in float4 (kk / 4) * nvi + vv
      *reinterpret_cast<float2*>(ab + (((kk >> 2) * nvi + vv) << 2) + (kk & 3)) = make_float2(t[0], t[1]);
      if (kk == 0) sfa[vv] = make_float2(sm, pow2f(149 - S));
    }
  }
  __syncthreads();
  if (!dw) return;
  // 3. my slice of the slot's activations, from the staged buffer
  LaneX X;
  if (von) {
    const float4* a4 = reinterpret_cast<const float4*>(ab);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(a4 + j * nvi + v);
      X.xp[2 * j] = t.x;
      X.xp[2 * j + 1] = t.y;
    }
    const float2 sf = sfa[v];
    X.sum = sf.x;
    X.f = sf.y;
  } else {
#pragma unroll
    for (int m = 0; m < 16; ++m) X.xp[m] = 0ull;
    X.sum = 0.f;
    X.f = 0.f;
  }
  // 4. my rows
  float* ysp = reinterpret_cast<float*>(smem + a.sm_ysp);
  for (int c0 = 0; gd + ngd * c0 < g.nrow; c0 += kDownChunk) {
    if (c0 > 0) {
#pragma unroll
      for (int i = 0; i < kDownChunk; ++i) {
        const int rho = gd + ngd * (c0 + i);
        dc[i] = make_uint4(0u, 0u, 0u, 0u);
        ds[i] = 0u;
        if (von && rho < g.nrow) {
          const long long r = g.r0 + rho;
          load_vec<BD>(blob + o[4] + r * cbI, blob + o[5] + r * sbI, v, dc[i], ds[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kDownChunk; ++i) {
      const int rho = gd + ngd * (c0 + i);
      if (rho < g.nrow) {
        const float y = warp_sum(von ? vec_row<BD>(dc[i], ds[i], X) : 0.f);
        if (g.lane == 0) ysp[((long long)s * a.max_drows + rho) * Pd + qd] = y;
      }
    }
  }
}

// Down steps of the slots finished so far, in the fixed schedule: after the
// routing decision the shared slot; then each routed slot in order.
template <int BR, int BS>
__device__ __forceinline__ void down_slot(const DecodeArgs& a, DecodeShared& cs, const Geo& g, char* smem, int s,
                                          unsigned tag) {
  if (s < a.K) down_step<BR>(a, cs, g, smem, s, tag);
  else down_step<BS>(a, cs, g, smem, s, tag);
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// BR, BS: code width of the routed experts and of the shared (or single)
// expert; each combination is its own instantiation.
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(16) char smem[];
  __shared__ DecodeShared cs;
  const Geo g = make_geo(a);
  const int tid = g.tid, lane = g.lane;
  FMOE_TRACE_WARP(0);
  // The next decode on the stream may be scheduled now: its CTAs take the
  // SMs this grid's CTAs leave and do their weight-only set-up meanwhile.
  grid_dep_launch_dependents();

  // ---- Set-up: weights only until the previous grid on the stream is done ---
  if (tid == 0) {
    mbar_init(&cs.x_bar, 1);
    mbar_init(&cs.route_bar, 1);
    cs.route_claim = 0;
    cs.poison = 0;
    cs.last = 0;
    cs.sg = 1.0f;
    for (int k = 0; k < kMaxTopK; ++k) cs.blob[k] = a.experts;
    cs.blob[a.K] = a.shared;
    if (a.fixed_route) {
      for (int k = 0; k < a.K; ++k) {
        cs.idx[k] = k;
        cs.w[k] = a.fixed_w[k];
        cs.blob[k] = a.fixed_blob[k];
      }
      cs.sg = a.fixed_sg;
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&cs.x_bar, a.H * 4 + (a.norm_w ? a.H * 2 : 0));
    if (a.norm_w) bulk_g2s(smem + a.sm_norm, a.norm_w, a.H * 2, &cs.x_bar);
    if (a.fixed_route) mbar_arrive(&cs.route_bar);
  }
  for (int i = tid; i < a.max_units; i += kThreads) reinterpret_cast<int*>(smem + a.sm_ucnt)[i] = 0;
  for (int i = tid; i < a.max_rrows; i += kThreads) reinterpret_cast<int*>(smem + a.sm_rcnt)[i] = 0;
  // my first router row and my first shared units, into registers
  uint4 rw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) rw[i] = make_uint4(0u, 0u, 0u, 0u);
  if (g.gon && g.grp < g.n_rr_c) load_router(a, g, g.c + g.G * g.grp, rw);  // my group's first row
  const int n_sh_w = my_shared_units(g);
  UnitRegs R[kRing];
  {
    const char* sh = a.shared;
#pragma unroll
    for (int d = 0; d < kRing; ++d) {
      R[d].cg = R[d].cu = make_uint4(0u, 0u, 0u, 0u);
      R[d].sg = R[d].su = 0u;
      if (d < n_sh_w) {
        UnitRef u;
        u.j = g.grp + g.n_grp * d;
        u.row = g.sh_first + g.G * u.j;
        u.slot = a.K;
        u.blob = sh;
        load_unit<BS>(a, u, a.off_s, g, R[d]);
      }
    }
  }
  // L2: the rest of my shared units (slice-0 warps, one lane per row part),
  // and this CTA's block of shared down rows (the last warp)
  if (a.shared != nullptr) {
    if (g.gon && g.q == 0) {
      const long long cb = (long long)a.H * BS / 8, sbr = a.H / 16;
      for (int t = lane + 4 * kRing; t < 4 * n_sh_w; t += 32) {  // (the first kRing are loaded above)
        const int i = t >> 2, part = t & 3;
        const int row = g.sh_first + g.G * (g.grp + g.n_grp * i);
        const long long sec = a.off_s[part], len = (part & 1) ? sbr : cb;
        const long long sec_len = (long long)a.I * len;
        prefetch_l2_in(a.shared + sec + row * len, len, a.shared + sec, a.shared + sec + sec_len);
      }
    }
    if (g.warp == kWarps - 1 && lane < 2 && g.nrow > 0) {
      const long long cbI = (long long)a.I * BS / 8, sbI = a.I / 16;
      const long long len = lane == 0 ? cbI : sbI, sec = a.off_s[4 + lane];
      prefetch_l2_in(a.shared + sec + g.r0 * len, g.nrow * len, a.shared + sec, a.shared + sec + (long long)a.H * len);
    }
  }
  __syncthreads();
  FMOE_TRACE_WARP(1);
  // x, the residual, the workspace and the outputs may be the previous grid's:
  // no access to them before it has completed.
  grid_dep_wait();
  FMOE_TRACE_WARP(2);
  const unsigned epoch = ld_relaxed_gpu(&a.bar[0]);
  const unsigned tag = epoch < kEpochLimit ? epoch + 1u : 0u;  // 0: a workspace that was never zeroed
  if (tid == 0) bulk_g2s(smem, a.x, a.H * 4, &cs.x_bar);
  if (!mbar_wait_bounded(&cs.x_bar, 0, a.timeout_ns) && lane == 0) {
    set_status(kStatusCopyTimeout);
    cs.poison = 1;
  }
  float* xs_raw = reinterpret_cast<float*>(smem);
  if (a.norm_w) {
    // Input RMS norm, in place: x <- x / sqrt(mean(x^2) + eps) * w.  Every
    // thread sums the per-warp partials in the same order.
    const uint16_t* wn = reinterpret_cast<const uint16_t*>(smem + a.sm_norm);
    float ss = 0.f;
    for (int i = tid; i < a.H; i += kThreads) ss = fmaf(xs_raw[i], xs_raw[i], ss);
    ss = warp_sum(ss);
    if (lane == 0) cs.red[g.warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += cs.red[w];
    const float r = 1.0f / sqrtf(tot / (float)a.H + a.norm_eps);
    for (int i = tid; i < a.H; i += kThreads) xs_raw[i] = xs_raw[i] * r * __uint_as_float((uint32_t)wn[i] << 16);
    __syncthreads();
  }
  FMOE_TRACE_WARP(3);
  // ---- Router rows and the shared expert's gate/up --------------------------
  LaneX X;
  {
    float xr[32];
    if (g.xon) {
      const float4* p = reinterpret_cast<const float4*>(xs_raw + g.vx * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 t = p[j];
        xr[4 * j] = t.x;
        xr[4 * j + 1] = t.y;
        xr[4 * j + 2] = t.z;
        xr[4 * j + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) xr[k] = 0.f;
    }
    router_rows(a, cs, g, smem, rw, xr, tag);
    FMOE_TRACE_WARP(4);
    stage_lane<BS>(xr, X);
  }
  unit_loop<BS, false>(a, cs, g, smem, n_sh_w, R, X, tag);
  FMOE_TRACE_WARP(5);

  // ---- Routing ---------------------------------------------------------------
  if (a.K > 0) {
    if (!a.fixed_route) {
      int claim = 0;
      if (lane == 0) claim = atomicAdd(&cs.route_claim, 1) == 0;
      if (__shfl_sync(0xffffffffu, claim, 0)) {
        if (a.E <= 512) route_warp<16>(a, cs, g, tag);
        else route_warp<kMaxExperts / 32>(a, cs, g, tag);
        if (lane == 0) mbar_arrive(&cs.route_bar);
      }
    }
    if (!mbar_wait_bounded(&cs.route_bar, 0, a.timeout_ns) && lane == 0) {
      set_status(kStatusCtaWaitTimeout);
      cs.poison = 1;
    }
    FMOE_TRACE_WARP(6);
    // L2: my routed units (slice-0 warps, one lane per row part) and this
    // CTA's blocks of routed down rows (the last warp, one lane per part)
    const int n_ro_w = my_routed_units(g);
    {
      const long long cb = (long long)a.H * BR / 8, sbr = a.H / 16;
      if (g.gon && g.q == 0) {
        for (int t = lane; t < 4 * n_ro_w; t += 32) {
          const UnitRef u = routed_unit(a, cs, g, t >> 2);
          const int part = t & 3;
          const long long sec = a.off_r[part], len = (part & 1) ? sbr : cb;
          prefetch_l2_in(u.blob + sec + u.row * len, len, u.blob + sec, u.blob + sec + (long long)a.I * len);
        }
      }
      if (g.warp == kWarps - 1 && g.nrow > 0) {
        const long long cbI = (long long)a.I * BR / 8, sbI = a.I / 16;
        for (int t = lane; t < 2 * a.K; t += 32) {
          const char* b = cs.blob[t >> 1];
          const long long len = (t & 1) ? sbI : cbI, sec = a.off_r[4 + (t & 1)];
          prefetch_l2_in(b + sec + g.r0 * len, g.nrow * len, b + sec, b + sec + (long long)a.H * len);
        }
      }
    }
    // While the routed rows stream: the shared expert's down rows.
    if (a.has_shared) down_slot<BR, BS>(a, cs, g, smem, a.K, tag);
    FMOE_TRACE_WARP(7);
    // ---- Routed gate/up ------------------------------------------------------
    {
      float xr[32];
      if (g.xon) {
        const float4* p = reinterpret_cast<const float4*>(xs_raw + g.vx * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 t = p[j];
          xr[4 * j] = t.x;
          xr[4 * j + 1] = t.y;
          xr[4 * j + 2] = t.z;
          xr[4 * j + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) xr[k] = 0.f;
      }
#pragma unroll
      for (int d = 0; d < kRing; ++d) {
        if (d < n_ro_w) load_unit<BR>(a, routed_unit(a, cs, g, d), a.off_r, g, R[d]);
      }
      stage_lane<BR>(xr, X);
    }
    unit_loop<BR, true>(a, cs, g, smem, n_ro_w, R, X, tag);
    FMOE_TRACE_WARP(8);
    for (int s = 0; s < a.K; ++s) down_slot<BR, BS>(a, cs, g, smem, s, tag);
  } else if (a.has_shared) {
    down_slot<BR, BS>(a, cs, g, smem, a.K, tag);
  }
  FMOE_TRACE_WARP(9);

  // ---- Combine: out = residual + sum_k w_k y_k + sg * y_shared, fixed order ---
  __syncthreads();
  {
    const int nvi = a.I / 32, Pd = (nvi + 31) / 32;
    const int n_slots = a.K + (a.has_shared ? 1 : 0);
    const float* ysp = reinterpret_cast<const float*>(smem + a.sm_ysp);
    const bool poisoned = cs.poison != 0;
    for (int t = tid; t < g.nrow; t += kThreads) {
      const int r = g.r0 + t;
      float v = a.residual ? __ldg(a.residual + r) : 0.f;
      for (int s = 0; s < n_slots; ++s) {
        float y = 0.f;
        for (int q = 0; q < Pd; ++q) y += ysp[((long long)s * a.max_drows + t) * Pd + q];
        v = fmaf(s < a.K ? cs.w[s] : cs.sg, y, v);
      }
      a.out[r] = poisoned ? quiet_nan() : v;
    }
  }
  FMOE_TRACE_WARP(10);

  // ---- Done: the last CTA advances the epoch and resets the ticket ----------
  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&a.bar[2], 1u);
    if (t + 1 == (unsigned)g.G) {
      __threadfence();
      cs.last = 1;
    }
  }
  __syncthreads();
  if (cs.last) {
    // Every CTA is past its last use of this launch's tag.  Tags run
    // 1 .. kEpochLimit; before the epoch would reach kEpochLimit (or when it
    // was not a valid epoch) every tagged word is cleared (tag 0 never
    // matches) and the epoch restarts at 0, so no word left by an earlier
    // launch ever carries a later launch's tag.
    unsigned ep = epoch + 1u;
    if (epoch >= kEpochLimit - 1u) {
      for (int e = tid; e < kTagWords; e += kThreads) st_relaxed_gpu_u64(a.tlog + e, 0ull);
      for (int e = tid; e < kMaxActWords; e += kThreads) st_relaxed_gpu_u64(a.tact + e, 0ull);
      ep = 0u;
    }
    __syncthreads();
    if (tid == 0) {
      atomicExch(&a.bar[0], ep);
      atomicExch(&a.bar[2], 0u);
      __threadfence();
    }
  }
}

}  // namespace fmoe
