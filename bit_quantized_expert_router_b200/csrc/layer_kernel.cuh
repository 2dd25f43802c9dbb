// The single-token MoE layer as one persistent, cooperative kernel.
//
// What it computes (the Flash-MoE pages): a router GEMV over the experts, then
// softmax, top-K and renormalised weights ("Flash-MoE: Ausführen eines
// 397B-Parameter-Qwen-Modells ...", section "Pipeline-Leistung"); the selected
// experts plus one shared expert as dequantised GEMVs, gate and up, fused
// SwiGLU, then down (section "Metal-Compute-Shader"); and a fused end step,
// out = residual + sum_k w_k y_k + sigmoid(w_sg . x) * y_shared (same section,
// "MoE-Kombination + Rest + Sigmoid-Gate").
//
// How it runs on B200.  One CTA per SM, every CTA co-resident (cooperative
// launch).  Work is three phases of independent units, dealt round-robin over
// all warps of the grid:
//   A  router rows (direct 16-byte loads) and the shared expert's gate/up rows;
//   B  the routed experts' gate/up rows (need the routing decision);
//   C  blocks of kRC output rows of the down projections of every expert,
//      combined with the routing weights, the shared gate and the residual.
// Two grid-wide hand-offs separate them: "all router logits written" (before
// any warp picks experts) and "all SwiGLU activations written" (before down).
// Both are split-phase: a CTA arrives as soon as its own part is done and
// waits only when it needs the result, and every wait is time-limited (it sets
// a status bit instead of hanging).  Each warp streams its units through a
// private ring of shared-memory stages filled by cp.async.bulk copies completed
// on an mbarrier, so weight bytes keep flowing while the warp computes, and a
// warp prefetches its down-projection rows while it waits for the second
// hand-off.  No float atomics: every output is reduced by one warp in a fixed
// order, so results are bitwise reproducible.
#pragma once
#include "dequant.cuh"

namespace fmoe {

constexpr int kWarps = 16;        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRC = 4;            // down rows per phase-C unit
constexpr int kMaxTopK = 8;
constexpr int kMaxSlots = kMaxTopK + 1;
constexpr int kMaxExperts = 1024; // top-K is one warp with 32 logits per lane

struct LayerArgs {
  const uint16_t* w_router;  // [E][H] bf16 bits, or null (single-expert mode)
  const uint16_t* w_sgate;   // [H] bf16 bits, or null (ungated shared expert)
  const char* experts;       // E routed blobs, blob e at experts + e * expert_stride
  long long expert_stride;
  const char* shared;        // shared expert blob (or the single expert), or null
  const float* x;            // [H]
  const float* residual;     // [H] or null
  float* out;                // [H]
  float* logits;             // workspace [E + 1]
  float* act;                // workspace [n_slots][I]
  unsigned* bar;             // workspace [4]: logits ready, activations ready, done
  int* idx_out;              // optional [K]
  float* w_out;              // optional [K]
  float* sg_out;             // optional [1]
  int H, I, E, K, bits_r, bits_s;
  int n_router;              // router rows: E (+1 with w_sgate), 0 in single-expert mode
  int n_slots;               // K routed slots then the shared slot
  int nst;                   // ring stages per warp
  int stage_bytes;
  int xs4_off, xs2_off, xu_off;  // float offsets inside the vector region (-1 = absent)
  int vec_floats, sf_floats;
  unsigned long long timeout_ns;
};

struct Smem {
  char* ring;
  float* vec;
  float2* sf;
  uint64_t* bars;
};

__device__ __forceinline__ Smem carve_smem(const LayerArgs& a, char* base) {
  Smem s;
  s.ring = base;
  size_t off = (size_t)kWarps * a.nst * a.stage_bytes;
  s.vec = reinterpret_cast<float*>(base + off);
  off += (size_t)a.vec_floats * 4;
  s.sf = reinterpret_cast<float2*>(base + off);
  off += (size_t)a.sf_floats * 8;
  s.bars = reinterpret_cast<uint64_t*>(base + off);
  return s;
}

// ---------------------------------------------------------------------------
// Unit bookkeeping: unit u of a phase whose numbering starts at slot offset
// `off` goes to grid-warp slot (u + off) mod GW; slot s is warp s / G of CTA
// s mod G, so consecutive units land on consecutive CTAs.
// ---------------------------------------------------------------------------
struct PhaseList {
  int first, count;
};
__device__ __forceinline__ PhaseList phase_list(int n_units, int off, int gslot, int GW) {
  PhaseList p;
  int f = (gslot - off) % GW;
  if (f < 0) f += GW;
  p.first = f;
  p.count = (n_units > f) ? (n_units - f - 1) / GW + 1 : 0;
  return p;
}

struct WarpPlan {
  PhaseList router, a, b, c;
  int n_loads;  // ring loads: a.count + b.count + c.count * n_slots
};

__device__ __forceinline__ WarpPlan make_plan(const LayerArgs& a, int cta, int warp, int G) {
  const int GW = G * kWarps;
  const int gslot = warp * G + cta;
  const int n_static = (a.shared != nullptr) ? a.I : 0;
  const int n_routed = a.K * a.I;
  const int n_c = a.H / kRC;
  WarpPlan p;
  int off = 0;
  p.router = phase_list(a.n_router, off, gslot, GW);
  off = (off + a.n_router) % GW;
  p.a = phase_list(n_static, off, gslot, GW);
  off = (off + n_static) % GW;
  p.b = phase_list(n_routed, off, gslot, GW);
  off = (off + n_routed) % GW;
  p.c = phase_list(n_c, off, gslot, GW);
  p.n_loads = p.a.count + p.b.count + p.c.count * a.n_slots;
  return p;
}

// Per-CTA shared state (static shared memory).
struct CtaShared {
  int route_state;     // 0 = not started, 1 = being computed, 2 = ready
  int idx[kMaxTopK];
  float w[kMaxTopK];
  float sg;
  unsigned router_done;
  unsigned router_target;
};

struct SlotInfo {
  const char* blob;
  int bits;
};

__device__ __forceinline__ SlotInfo slot_info(const LayerArgs& a, const CtaShared& cs, int slot) {
  SlotInfo si;
  if (slot < a.K) {
    si.blob = a.experts + (long long)cs.idx[slot] * a.expert_stride;
    si.bits = a.bits_r;
  } else {
    si.blob = a.shared;
    si.bits = a.bits_s;
  }
  return si;
}

// Bytes of the stage sections.
__device__ __forceinline__ int codes_row_bytes(int n_in, int bits) { return n_in * bits / 8; }
__device__ __forceinline__ int sb_row_bytes(int n_in) { return n_in / 16; }
__device__ __forceinline__ int sb_superset_cap(int n_in) { return ((n_in / 16 + 15) & ~15) + 16; }

// Issue the bulk copies of ring load `i` (lane 0 only).  Returns false if the
// load needs the routing decision and it is not known yet.
__device__ __forceinline__ void issue_load(const LayerArgs& a, const WarpPlan& p, const CtaShared& cs,
                                           int i, char* stage, uint64_t* bar, int GW) {
  if (i < p.a.count + p.b.count) {
    int slot, row;
    if (i < p.a.count) {
      slot = a.K;
      row = p.a.first + i * GW;
    } else {
      const int u = p.b.first + (i - p.a.count) * GW;
      slot = u / a.I;
      row = u % a.I;
    }
    const SlotInfo si = slot_info(a, cs, slot);
    const BlobOff o = blob_offsets(a.H, a.I, si.bits);
    const int cb = codes_row_bytes(a.H, si.bits);
    const int sbr = sb_row_bytes(a.H);
    const int cap = sb_superset_cap(a.H);
    const char* g_codes = si.blob + o.gc + (long long)row * cb;
    const char* u_codes = si.blob + o.uc + (long long)row * cb;
    const long long gs0 = o.gsb + (long long)row * sbr, us0 = o.usb + (long long)row * sbr;
    const long long ga = gs0 & ~15LL, ua = us0 & ~15LL;
    const int glen = (int)(((gs0 + sbr + 15) & ~15LL) - ga);
    const int ulen = (int)(((us0 + sbr + 15) & ~15LL) - ua);
    mbar_arrive_expect_tx(bar, 2 * cb + glen + ulen);
    bulk_g2s(stage, g_codes, cb, bar);
    bulk_g2s(stage + cb, u_codes, cb, bar);
    bulk_g2s(stage + 2 * cb, si.blob + ga, glen, bar);
    bulk_g2s(stage + 2 * cb + cap, si.blob + ua, ulen, bar);
  } else {
    const int j = i - p.a.count - p.b.count;
    const int unit = p.c.first + (j / a.n_slots) * GW;
    const int slot = j % a.n_slots;
    const int r0 = unit * kRC;
    const SlotInfo si = slot_info(a, cs, slot);
    const BlobOff o = blob_offsets(a.H, a.I, si.bits);
    const int cb = codes_row_bytes(a.I, si.bits);
    const int sbr = sb_row_bytes(a.I);
    mbar_arrive_expect_tx(bar, kRC * (cb + sbr));
    bulk_g2s(stage, si.blob + o.dc + (long long)r0 * cb, kRC * cb, bar);
    bulk_g2s(stage + kRC * cb, si.blob + o.dsb + (long long)r0 * sbr, kRC * sbr, bar);
  }
}

// ---------------------------------------------------------------------------
// Compute pieces
// ---------------------------------------------------------------------------

// One router row (bf16) against the unscaled input x (shared memory).
__device__ __forceinline__ float router_dot(const uint16_t* row, const float* xu, int H, int lane) {
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  const int nv = H / 8;
  float acc = 0.f;
  for (int base = 0; base < nv; base += 32 * 16) {
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int v = base + lane + 32 * i;
      if (v < nv) w[i] = ld_stream_u4(rv + v);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int v = base + lane + 32 * i;
      if (v < nv) {
        const float4 xa = reinterpret_cast<const float4*>(xu)[2 * v];
        const float4 xb = reinterpret_cast<const float4*>(xu)[2 * v + 1];
        acc = fmaf(bf16_lo(w[i].x), xa.x, acc);
        acc = fmaf(bf16_hi(w[i].x), xa.y, acc);
        acc = fmaf(bf16_lo(w[i].y), xa.z, acc);
        acc = fmaf(bf16_hi(w[i].y), xa.w, acc);
        acc = fmaf(bf16_lo(w[i].z), xb.x, acc);
        acc = fmaf(bf16_hi(w[i].z), xb.y, acc);
        acc = fmaf(bf16_lo(w[i].w), xb.z, acc);
        acc = fmaf(bf16_hi(w[i].w), xb.w, acc);
      }
    }
  }
  return warp_sum(acc);
}

// Gate and up rows of one expert (stage layout: gate codes | up codes | gate sb
// superset | up sb superset) against the staged input.
template <int BITS>
__device__ __forceinline__ void pair_dot(const char* st, int H, int sbo_g, int sbo_u, const float4* xs,
                                         const float2* sf, int lane, float& g_out, float& u_out) {
  constexpr int CPV = 128 / BITS;
  const int NV = H / CPV;
  const int cb = H * BITS / 8;
  const int cap = sb_superset_cap(H);
  const uint4* cg = reinterpret_cast<const uint4*>(st);
  const uint4* cu = reinterpret_cast<const uint4*>(st + cb);
  const uint32_t* sbg = reinterpret_cast<const uint32_t*>(st + 2 * cb + sbo_g);
  const uint32_t* sbu = reinterpret_cast<const uint32_t*>(st + 2 * cb + cap + sbo_u);
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(xs);
  float g = 0.f, u = 0.f;
  for (int v = lane; v < NV; v += 32) {
    const uint4 wg = cg[v], wu = cu[v];
    const int grp = (BITS == 4) ? (v >> 1) : v;
    const uint32_t sbgw = sbg[grp], sbuw = sbu[grp];
    const float2 f = sf[v];
    uint64_t ag = 0, au = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t a_ = (&wg.x)[t], b_ = (&wu.x)[t];
      if (BITS == 4) {
        const ulonglong2 xa = xv[(2 * t) * NV + v], xb = xv[(2 * t + 1) * NV + v];
        dot_word4(ag, a_, xa, xb);
        dot_word4(au, b_, xa, xb);
      } else {
        const ulonglong2 x0 = xv[(4 * t) * NV + v], x1 = xv[(4 * t + 1) * NV + v];
        const ulonglong2 x2 = xv[(4 * t + 2) * NV + v], x3 = xv[(4 * t + 3) * NV + v];
        dot_word2(ag, a_, x0, x1, x2, x3);
        dot_word2(au, b_, x0, x1, x2, x3);
      }
    }
    const float2 dg = unpk_f32(ag), du = unpk_f32(au);
    g = fmaf(bf16_lo(sbgw) * f.y, dg.x + dg.y, g);
    g = fmaf(bf16_hi(sbgw), f.x, g);
    u = fmaf(bf16_lo(sbuw) * f.y, du.x + du.y, u);
    u = fmaf(bf16_hi(sbuw), f.x, u);
  }
  g_out = warp_sum(g);
  u_out = warp_sum(u);
}

// kRC down rows of one expert (stage layout: kRC code rows | kRC sb rows)
// against that expert's staged activation; adds coef * row dot to acc[r].
template <int BITS>
__device__ __forceinline__ void down_rows(const char* st, int I, const float4* as, const float2* sfa,
                                          int lane, float coef, float (&acc)[kRC]) {
  constexpr int CPV = 128 / BITS;
  const int NV = I / CPV;
  const int cb = I * BITS / 8;
  const int ng = I / 64;
  const uint32_t* sb = reinterpret_cast<const uint32_t*>(st + kRC * cb);
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(as);
  float y[kRC];
#pragma unroll
  for (int r = 0; r < kRC; ++r) y[r] = 0.f;
  for (int v = lane; v < NV; v += 32) {
    uint4 w[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) w[r] = reinterpret_cast<const uint4*>(st + r * cb)[v];
    const float2 f = sfa[v];
    const int grp = (BITS == 4) ? (v >> 1) : v;
    uint64_t ac[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) ac[r] = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (BITS == 4) {
        const ulonglong2 xa = xv[(2 * t) * NV + v], xb = xv[(2 * t + 1) * NV + v];
#pragma unroll
        for (int r = 0; r < kRC; ++r) dot_word4(ac[r], (&w[r].x)[t], xa, xb);
      } else {
        const ulonglong2 x0 = xv[(4 * t) * NV + v], x1 = xv[(4 * t + 1) * NV + v];
        const ulonglong2 x2 = xv[(4 * t + 2) * NV + v], x3 = xv[(4 * t + 3) * NV + v];
#pragma unroll
        for (int r = 0; r < kRC; ++r) dot_word2(ac[r], (&w[r].x)[t], x0, x1, x2, x3);
      }
    }
#pragma unroll
    for (int r = 0; r < kRC; ++r) {
      const uint32_t sbw = sb[r * ng + grp];
      const float2 d = unpk_f32(ac[r]);
      y[r] = fmaf(bf16_lo(sbw) * f.y, d.x + d.y, y[r]);
      y[r] = fmaf(bf16_hi(sbw), f.x, y[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < kRC; ++r) acc[r] = fmaf(coef, y[r], acc[r]);
}

// Top-K over n logits by one warp: descending logit, lower index first on
// exact ties; renormalised softmax weights over the selected logits.
__device__ __forceinline__ void warp_topk(const float* logits, int n, int k, int lane, int* idx_out,
                                          float* w_out) {
  float v[kMaxExperts / 32];
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i) {
    const int e = i * 32 + lane;
    v[i] = (e < n) ? __ldcg(logits + e) : -INFINITY;
  }
  float top[kMaxTopK];
  int topi[kMaxTopK];
  for (int kk = 0; kk < k; ++kk) {
    float best = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = i * 32 + lane;
      if (e < n && (v[i] > best || (v[i] == best && e < bi))) {
        best = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    top[kk] = best;
    topi[kk] = bi;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i)
      if (i * 32 + lane == bi) v[i] = -INFINITY;
  }
  // w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0): softmax restricted to the
  // selected experts, equal to softmax-then-renormalise.
  float e[kMaxTopK];
  float s = 0.f;
  for (int kk = 0; kk < k; ++kk) {
    e[kk] = expf(top[kk] - top[0]);
    s += e[kk];
  }
  if (lane == 0) {
    for (int kk = 0; kk < k; ++kk) {
      idx_out[kk] = topi[kk];
      w_out[kk] = e[kk] / s;
    }
  }
}

// Wait until *ctr >= target (one thread), for at most limit_ns.
__device__ __forceinline__ bool grid_wait(const unsigned* ctr, unsigned target, uint64_t limit_ns) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(ctr) < target) {
    __nanosleep(64);
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Make the routing decision available in this CTA's shared state.  The first
// warp to ask waits for all router logits and runs the top-K; the others wait
// for it.  Called by whole warps.
__device__ __noinline__ void ensure_routing(const LayerArgs& a, CtaShared& cs, int lane) {
  if (*((volatile int*)&cs.route_state) == 2) return;
  int old = 0;
  if (lane == 0) old = atomicCAS(&cs.route_state, 0, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old == 0) {
    bool ok = true;
    if (lane == 0) ok = grid_wait(&a.bar[0], gridDim.x, a.timeout_ns);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok && lane == 0) set_status(kStatusGridBarrierTimeout);
    warp_topk(a.logits, a.E, a.K, lane, cs.idx, cs.w);
    if (lane == 0) {
      // Guard the expert index even on a timed-out (garbage) path.
      for (int k = 0; k < a.K; ++k)
        if (cs.idx[k] < 0 || cs.idx[k] >= a.E) cs.idx[k] = 0;
      cs.sg = a.w_sgate ? sigmoidf_(__ldcg(a.logits + a.E)) : 1.0f;
      if (blockIdx.x == 0) {
        for (int k = 0; k < a.K; ++k) {
          if (a.idx_out) a.idx_out[k] = cs.idx[k];
          if (a.w_out) a.w_out[k] = cs.w[k];
        }
        if (a.sg_out) *a.sg_out = cs.sg;
      }
      __threadfence_block();
      atomicExch(&cs.route_state, 2);
    }
    __syncwarp();
  } else {
    bool ok = true;
    if (lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (*((volatile int*)&cs.route_state) != 2) {
        __nanosleep(32);
        if (globaltimer_ns() - t0 > a.timeout_ns) {
          ok = false;
          break;
        }
      }
      if (!ok) set_status(kStatusCtaWaitTimeout);
      __threadfence_block();
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kThreads, 1) layer_kernel(const __grid_constant__ LayerArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ CtaShared cs;
  const Smem sm = carve_smem(a, smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, GW = G * kWarps;
  const WarpPlan plan = make_plan(a, blockIdx.x, warp, G);
  char* my_ring = sm.ring + (size_t)warp * a.nst * a.stage_bytes;
  uint64_t* my_bars = sm.bars + warp * a.nst;
  const bool layer_mode = a.n_router > 0;

  if (tid == 0) {
    cs.route_state = layer_mode ? 0 : 2;
    cs.sg = 1.0f;
    cs.router_done = 0;
    // router rows owned by this CTA
    unsigned tgt = 0;
    for (int w = 0; w < kWarps; ++w) tgt += phase_list(a.n_router, 0, w * G + blockIdx.x, GW).count;
    cs.router_target = tgt;
  }
  if (lane == 0) {
    for (int s = 0; s < a.nst; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (tid == 0 && layer_mode && cs.router_target == 0) red_release_gpu_add(&a.bar[0], 1);

  // Prologue: start the first ring loads that need no routing decision.
  int issued = 0;
  if (lane == 0) {
    while (issued < plan.n_loads && issued < a.nst && issued < plan.a.count) {
      issue_load(a, plan, cs, issued, my_ring + (size_t)issued * a.stage_bytes, &my_bars[issued], GW);
      ++issued;
    }
  }
  issued = __shfl_sync(0xffffffffu, issued, 0);

  // Stage x: unscaled copy for the router, decode layouts for the experts.
  if (layer_mode) {
    float4* xu4 = reinterpret_cast<float4*>(sm.vec + a.xu_off);
    const float4* x4 = reinterpret_cast<const float4*>(a.x);
    for (int i = tid; i < a.H / 4; i += kThreads) xu4[i] = __ldcg(x4 + i);
  }
  if (a.xs4_off >= 0)
    stage_vector(a.x, a.H, 4, reinterpret_cast<float4*>(sm.vec + a.xs4_off), sm.sf, tid, kThreads);
  if (a.xs2_off >= 0)
    stage_vector(a.x, a.H, 2, reinterpret_cast<float4*>(sm.vec + a.xs2_off),
                 sm.sf + (a.xs4_off >= 0 ? a.H / 32 : 0), tid, kThreads);
  __syncthreads();

  // ---- Phase A: router rows --------------------------------------------------
  for (int j = 0; j < plan.router.count; ++j) {
    const int e = plan.router.first + j * GW;
    const uint16_t* row = (e < a.E) ? a.w_router + (long long)e * a.H : a.w_sgate;
    const float l = router_dot(row, sm.vec + a.xu_off, a.H, lane);
    if (lane == 0) {
      a.logits[e] = l;
      __threadfence();
      const unsigned d = atomicAdd(&cs.router_done, 1u);
      if (d + 1 == cs.router_target) red_release_gpu_add(&a.bar[0], 1);
    }
  }

  // ---- Ring loop over phases A (static gate/up) and B (routed gate/up) ------
  const int n_gu = plan.a.count + plan.b.count;
  const float4* xs4 = reinterpret_cast<const float4*>(sm.vec + (a.xs4_off >= 0 ? a.xs4_off : 0));
  const float4* xs2 = reinterpret_cast<const float4*>(sm.vec + (a.xs2_off >= 0 ? a.xs2_off : 0));
  const float2* sf4 = sm.sf;
  const float2* sf2 = sm.sf + (a.xs4_off >= 0 ? a.H / 32 : 0);
  bool have_routing = !layer_mode;

  for (int i = 0; i < n_gu; ++i) {
    // Loads from index plan.a.count on need the routing decision: block for it
    // when the warp is about to consume such a load, otherwise take it only if
    // it is already there.
    if (!have_routing) {
      int ready = 0;
      if (lane == 0) ready = *((volatile int*)&cs.route_state) == 2;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      const bool could = issued >= plan.a.count && issued < i + a.nst && issued < plan.n_loads;
      if (i >= plan.a.count || (could && ready)) {
        ensure_routing(a, cs, lane);
        have_routing = true;
      }
    }
    if (lane == 0) {
      while (issued < plan.n_loads && issued < i + a.nst && (have_routing || issued < plan.a.count)) {
        fence_proxy_async_smem();
        issue_load(a, plan, cs, issued, my_ring + (size_t)(issued % a.nst) * a.stage_bytes,
                   &my_bars[issued % a.nst], GW);
        ++issued;
      }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
    const int st_i = i % a.nst;
    const char* stage = my_ring + (size_t)st_i * a.stage_bytes;
    if (!mbar_wait_bounded(&my_bars[st_i], (i / a.nst) & 1, a.timeout_ns) && lane == 0)
      set_status(kStatusCopyTimeout);
    int slot, row;
    if (i < plan.a.count) {
      slot = a.K;
      row = plan.a.first + i * GW;
    } else {
      const int u = plan.b.first + (i - plan.a.count) * GW;
      slot = u / a.I;
      row = u % a.I;
    }
    const SlotInfo si = slot_info(a, cs, slot);
    const BlobOff o = blob_offsets(a.H, a.I, si.bits);
    const int sbr = sb_row_bytes(a.H);
    const int sbo_g = (int)((o.gsb + (long long)row * sbr) & 15);
    const int sbo_u = (int)((o.usb + (long long)row * sbr) & 15);
    float g, u;
    if (si.bits == 4)
      pair_dot<4>(stage, a.H, sbo_g, sbo_u, xs4, sf4, lane, g, u);
    else
      pair_dot<2>(stage, a.H, sbo_g, sbo_u, xs2, sf2, lane, g, u);
    if (lane == 0) a.act[(long long)slot * a.I + row] = g * sigmoidf_(g) * u;
    __syncwarp();
  }

  // Gate/up work of this warp is done: put its first down-projection loads in
  // flight before joining the hand-off, so they stream during the wait.
  if (plan.n_loads > n_gu) {
    if (!have_routing) {
      ensure_routing(a, cs, lane);
      have_routing = true;
    }
    if (lane == 0) {
      while (issued < plan.n_loads && issued < n_gu + a.nst) {
        fence_proxy_async_smem();
        issue_load(a, plan, cs, issued, my_ring + (size_t)(issued % a.nst) * a.stage_bytes,
                   &my_bars[issued % a.nst], GW);
        ++issued;
      }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
  }

  // ---- Hand-off: every activation of the grid is written --------------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    red_release_gpu_add(&a.bar[1], 1);
    if (!grid_wait(&a.bar[1], G, a.timeout_ns)) set_status(kStatusGridBarrierTimeout);
  }
  __syncthreads();
  if (warp == 0 && layer_mode && *((volatile int*)&cs.route_state) != 2) ensure_routing(a, cs, lane);
  __syncthreads();

  // Stage every slot's activation in its decode layout.
  {
    int vec_off = 0, sf_off = 0;
    for (int s = 0; s < a.n_slots; ++s) {
      const int bits = (s < a.K) ? a.bits_r : a.bits_s;
      stage_vector(a.act + (long long)s * a.I, a.I, bits, reinterpret_cast<float4*>(sm.vec + vec_off),
                   sm.sf + sf_off, tid, kThreads);
      vec_off += a.I;
      sf_off += a.I / 32;
    }
  }
  __syncthreads();

  // ---- Phase C: down projections + combine ----------------------------------
  float accr[kRC];
  for (int r = 0; r < kRC; ++r) accr[r] = 0.f;
  for (int i = n_gu; i < plan.n_loads; ++i) {
    if (lane == 0) {
      while (issued < plan.n_loads && issued < i + a.nst) {
        fence_proxy_async_smem();
        issue_load(a, plan, cs, issued, my_ring + (size_t)(issued % a.nst) * a.stage_bytes,
                   &my_bars[issued % a.nst], GW);
        ++issued;
      }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
    const int st_i = i % a.nst;
    const char* stage = my_ring + (size_t)st_i * a.stage_bytes;
    if (!mbar_wait_bounded(&my_bars[st_i], (i / a.nst) & 1, a.timeout_ns) && lane == 0)
      set_status(kStatusCopyTimeout);
    const int j = i - n_gu;
    const int slot = j % a.n_slots;
    const int bits = (slot < a.K) ? a.bits_r : a.bits_s;
    const float coef = (slot < a.K) ? cs.w[slot] : cs.sg;
    const float4* as = reinterpret_cast<const float4*>(sm.vec + slot * a.I);
    const float2* sfa = sm.sf + slot * (a.I / 32);
    if (bits == 4)
      down_rows<4>(stage, a.I, as, sfa, lane, coef, accr);
    else
      down_rows<2>(stage, a.I, as, sfa, lane, coef, accr);
    __syncwarp();
    if (slot == a.n_slots - 1) {
      const int unit = plan.c.first + (j / a.n_slots) * GW;
      const int r0 = unit * kRC;
      float tot[kRC];
#pragma unroll
      for (int r = 0; r < kRC; ++r) {
        tot[r] = warp_sum(accr[r]);
        accr[r] = 0.f;
      }
      if (lane == 0) {
        float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.residual) res = __ldg(reinterpret_cast<const float4*>(a.residual + r0));
        *reinterpret_cast<float4*>(a.out + r0) =
            make_float4(res.x + tot[0], res.y + tot[1], res.z + tot[2], res.w + tot[3]);
      }
    }
  }

  // ---- Done: the last CTA resets the hand-off counters for the next launch --
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&a.bar[2], 1u);
    if (t + 1 == (unsigned)G) {
      atomicExch(&a.bar[0], 0u);
      atomicExch(&a.bar[1], 0u);
      atomicExch(&a.bar[2], 0u);
      __threadfence();
    }
  }
}

}  // namespace fmoe
