// The single-token MoE layer as one persistent kernel.
//
// What it computes (the Flash-MoE pages): a router GEMV over the experts, then
// softmax, top-K and renormalised weights ("Flash-MoE: Ausführen eines
// 397B-Parameter-Qwen-Modells ...", section "Pipeline-Leistung"); the selected
// experts plus one shared expert as dequantised GEMVs, gate and up, fused
// SwiGLU, then down (section "Metal-Compute-Shader"); and a fused end step,
// out = residual + sum_k w_k y_k + sigmoid(w_sg . x) * y_shared (same section,
// "MoE-Kombination + Rest + Sigmoid-Gate").
//
// How it runs on B200.  One CTA per SM, every CTA co-resident (one CTA fits
// per SM and the grid is the SM count; a programmatic dependent launch by
// default, so that its weight-only set-up overlaps the previous kernel's end,
// or a cooperative launch).  Three phases:
//   A  router rows (each split over several warps of its CTA) and the shared
//      expert's gate/up rows (need nothing);
//   B  the routed experts' gate/up rows (need the routing decision);
//   C  the down projections of every expert over each CTA's own contiguous
//      block of output rows, then the combine (need all SwiGLU activations).
// Units of phases A and B are dealt round-robin over all warps of the grid.
//
// Hand-offs.  Each router warp publishes its logit, and each gate/up warp its
// SwiGLU activation, as one 64-bit word tagged with this launch's number (the
// workspace's epoch + 1); a reader polls a word until it carries the tag, so
// no grid-wide barrier is needed.  Every CTA takes the routing decision with
// all of its warps: each lane polls the words of its warp's slice of the
// logits, each warp selects the top K of its slice, and the candidates are
// ranked (CTA barriers between the steps).  For the down projections every
// CTA polls and stages all activations in one pass.  Every wait is
// time-limited: on expiry
// the kernel sets a status bit and carries on instead of hanging, and the CTA
// that waited in vain writes and hands on NaN from then on (its activations,
// its output rows, the routing outputs), so no result built on a missing value
// looks plausible.
//
// Data movement.  Each warp streams its gate/up units through a private ring
// of shared-memory stages filled by cp.async.bulk copies that complete on an
// mbarrier.  When its gate/up work is done, the warp re-carves its ring into
// smaller stages and issues all of its down-projection items at once, so they
// stream during the second hand-off; L2 is asked to prefetch the shared
// expert's down rows at kernel start and the routed experts' down rows as soon
// as the routing is known.  No float atomics: every output is reduced in a
// fixed order, so results are bitwise reproducible.
#pragma once
#include "dequant.cuh"

namespace fmoe {

constexpr int kWarps = 16;        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRC = 4;            // down rows per phase-C item (the split row reduction assumes 4)
constexpr int kMaxTopK = 8;
constexpr int kMaxSlots = kMaxTopK + 1;
constexpr int kMaxExperts = 1024; // top-K is one warp with 32 logits per lane
constexpr int kTagWords = kMaxExperts + 1;  // tagged-logit words of a workspace (routers and the gate)
constexpr int kActWords = 10240;            // tagged-activation words of a workspace ((K + 1) * I at most)
// Launch epochs run 0 .. kEpochWrap; a launch's tag is its epoch + 1, so tags
// run 1 .. kEpochWrap + 1 and 0 never matches.  An epoch with the top bit set
// is a workspace that was not zeroed (or was overwritten): its launch tags
// nothing (tag 0), so every tagged wait runs out instead of accepting words.
constexpr unsigned kEpochWrap = 0x7FFFFFFEu;
constexpr int kMaxNstC = 8;       // most down-item stages a warp keeps in flight
constexpr int kRouteWarps = 8;    // warps of a CTA that take the routing decision (the others stage x meanwhile)

// Optional phase trace (compile with -DFMOE_TRACE_BUILD): the SM cycle counter
// at fixed points of the kernel, per CTA in shared memory (points marked per
// warp keep the latest warp), copied to g_fmoe_trace[blockIdx] at the end, with
// %globaltimer at the dependency wait and at the end to place and scale them.
#ifdef FMOE_TRACE_BUILD
constexpr int kTracePoints = 25;
constexpr int kTraceCols = kTracePoints + 3;  // + globaltimer at point 24 and at the end, cycles at the end
__device__ unsigned long long g_fmoe_trace[1024][kTraceCols];
#define FMOE_TRACE(i) \
  do { if (threadIdx.x == 0) cs.trace[i] = clock64(); } while (0)
#define FMOE_TRACE_WARP(i) \
  do { if ((threadIdx.x & 31) == 0) atomicMax(&cs.trace[i], (unsigned long long)clock64()); } while (0)
#else
#define FMOE_TRACE(i) do { } while (0)
#define FMOE_TRACE_WARP(i) do { } while (0)
#endif

struct LayerArgs {
  const uint16_t* w_router;  // [E][H] bf16 bits, or null (single-expert mode)
  const uint16_t* w_sgate;   // [H] bf16 bits, or null (ungated shared expert)
  const char* experts;       // E routed blobs, blob e at experts + e * expert_stride
  long long expert_stride;
  const char* shared;        // shared expert blob (or the single expert), or null
  const float* x;            // [H]
  const float* residual;     // [H] or null
  float* out;                // [H]
  // workspace [n_router] tagged logits: word e = (tag << 32) | bits of logit e,
  // tag = this launch's epoch + 1 (written by the router warps only)
  unsigned long long* tlog;
  // workspace [n_slots][I] tagged activations, same word format as tlog
  unsigned long long* tact;
  unsigned* bar;             // workspace: [0] launch epoch, [1] unused (zero), [2] done ticket
  int* idx_out;              // optional [K]
  float* w_out;              // optional [K]
  float* sg_out;             // optional [1]
  int H, I, E, K, bits_r, bits_s;
  int n_router;              // router rows: E (+1 with w_sgate), 0 in single-expert mode
  int n_slots;               // K routed slots then the shared slot
  int off_a, off_b;          // round-robin slot offsets of phases A and B (in [0, G*kWarps))
  int nst;                   // ring stages per warp (gate/up phases)
  int stage_bytes;
  int nst_c;                 // ring stages per warp once re-carved for down items
  int c_stage_bytes;
  int xs4_off, xs2_off, xu_off;  // float offsets inside the vector region (-1 = absent)
  int vec_floats, sf_floats;
  int ys_stride;             // rows per CTA (max) in the phase-C result array
  long long off_r[6], off_s[6];  // blob section offsets for the routed / shared code width
  unsigned long long timeout_ns;
  int router_smem;           // 1: each router warp's row is bulk-copied into its ring at entry
  const uint16_t* norm_w;    // [H] bf16 RMS-norm weight of the input, or null
  float norm_eps;
  // Given routing (no router rows): the blob and combine weight of each
  // routed slot, and the shared expert's gate.
  int fixed_route;
  const char* fixed_blob[kMaxTopK];
  float fixed_w[kMaxTopK];
  float fixed_sg;
};

struct Smem {
  char* ring;
  float* vec;
  float2* sf;
  float* ys;   // [n_slots][ys_stride] per-expert down-projection rows of this CTA
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
  s.ys = reinterpret_cast<float*>(base + off);
  off += (size_t)a.n_slots * a.ys_stride * 4;
  off = (off + 15) & ~(size_t)15;
  s.bars = reinterpret_cast<uint64_t*>(base + off);  // [kWarps][nst + kMaxNstC]
  return s;
}

// ---------------------------------------------------------------------------
// Work assignment.  Router rows: CTA c takes rows c, c + G, c + 2G, ...,
// each split into segments over several of its warps (RouterPart).  Gate/up
// units of phases A and B: unit u of a phase whose numbering starts at offset
// `off` goes to grid-warp slot (u + off) mod GW; slot s is warp s / G of CTA
// s mod G, so consecutive units land on consecutive CTAs.  Phase C: CTA c owns
// output-row quads [c*nq/G, (c+1)*nq/G) and its warps take the items (slot,
// quad) of that block round-robin.
// ---------------------------------------------------------------------------
struct PhaseList {
  int first, count;
};
__device__ __forceinline__ PhaseList phase_list(int n_units, int off, int gslot, int GW) {
  PhaseList p;
  int f = gslot - off;
  if (f < 0) f += GW;
  p.first = f;
  p.count = (n_units > f) ? (n_units - f - 1) / GW + 1 : 0;
  return p;
}

struct WarpPlan {
  PhaseList a, b;
  int q0, nq;      // this CTA's quad block
  int c_count;     // phase-C items of this warp
  int n_loads;     // ring loads: a.count + b.count + c_count
};

// This warp's router segment: the CTA's nr rows are each split into wpr
// segments of H / wpr inputs (wpr the largest power of two with nr * wpr <=
// kWarps and H / wpr a multiple of 8); warp w < nr * wpr takes segment w % wpr
// of row cta + (w / wpr) * G.
struct RouterPart {
  int nr, wpr;   // rows of this CTA, warps per row
  bool on;       // this warp has a segment
  int row;       // its router row (E: the shared gate's row)
  int seg0, n;   // its first input and length
};

__device__ __forceinline__ RouterPart router_part(int n_router, int H, int cta, int warp, int G) {
  RouterPart r;
  r.nr = n_router > cta ? (n_router - cta + G - 1) / G : 0;
  r.wpr = 1;
  while (r.nr > 0 && 2 * r.wpr * r.nr <= kWarps && (H / (2 * r.wpr)) % 8 == 0) r.wpr *= 2;
  r.on = warp < r.nr * r.wpr;
  r.row = cta + (warp / r.wpr) * G;
  r.n = H / r.wpr;
  r.seg0 = (warp % r.wpr) * r.n;
  return r;
}

__device__ __forceinline__ WarpPlan make_plan(const LayerArgs& a, int cta, int warp, int G) {
  const int GW = G * kWarps;
  const int gslot = warp * G + cta;
  WarpPlan p;
  p.a = phase_list(a.shared != nullptr ? a.I : 0, a.off_a, gslot, GW);
  p.b = phase_list(a.K * a.I, a.off_b, gslot, GW);
  const int nq_all = a.H / kRC;  // <= 2048, so cta * nq_all fits in 32 bits
  p.q0 = cta * nq_all / G;
  p.nq = (cta + 1) * nq_all / G - p.q0;
  const int n_items = a.n_slots * p.nq;
  p.c_count = (n_items > warp) ? (n_items - warp - 1) / kWarps + 1 : 0;
  p.n_loads = p.a.count + p.b.count + p.c_count;
  return p;
}

// Per-CTA shared state (static shared memory).
struct CtaShared {
#ifdef FMOE_TRACE_BUILD
  unsigned long long trace[kTraceCols];
#endif
  int poison;           // a wait of this CTA ran out: what it hands on or writes is NaN
  float rpart[kWarps];  // router segment dot products, by warp
  uint64_t x_bar;       // completes once x is in shared memory
  uint64_t rbar[kWarps];  // router warp w's row is in its ring (router_smem)
  unsigned long long param_touch;  // see the kernel's set-up
  float red[kWarps];               // per-warp partial sums (input norm)
  int c_prefetch;          // warps past their gate/up work (the first prefetches down rows)
  int last;                // this CTA took the last done ticket
  float w[kMaxTopK];
  float sg;
  const char* blob[kMaxSlots];  // blob of each slot (routed ones once the routing is known)
  uint32_t cand_key[kWarps * kMaxTopK];  // per-warp top-K candidates (order-preserving keys)
  uint32_t cand_idx[kWarps * kMaxTopK];  // and their expert indices
};


struct SlotInfo {
  const char* blob;
  int bits;
};

__device__ __forceinline__ SlotInfo slot_info(const LayerArgs& a, const CtaShared& cs, int slot) {
  SlotInfo si;
  si.blob = cs.blob[slot];
  si.bits = slot < a.K ? a.bits_r : a.bits_s;
  return si;
}

// Bytes of the stage sections.
__device__ __forceinline__ int codes_row_bytes(int n_in, int bits) { return n_in * bits / 8; }
__device__ __forceinline__ int sb_row_bytes(int n_in) { return n_in / 16; }
__device__ __forceinline__ int sb_superset_cap(int n_in) { return ((n_in / 16 + 15) & ~15) + 16; }

// (slot, row) of gate/up load i < a.count + b.count.
__device__ __forceinline__ void gu_unit(const LayerArgs& a, const WarpPlan& p, int i, int GW, int& slot,
                                        int& row) {
  if (i < p.a.count) {
    slot = a.K;
    row = p.a.first + i * GW;
  } else {
    const int u = p.b.first + (i - p.a.count) * GW;
    slot = u / a.I;
    row = u - slot * a.I;
  }
}

// (slot, first row) of phase-C load i >= a.count + b.count.
__device__ __forceinline__ void c_item(const WarpPlan& p, int i, int warp, int& slot, int& r0) {
  const int j = warp + (i - p.a.count - p.b.count) * kWarps;
  slot = j / p.nq;
  r0 = (p.q0 + (j - slot * p.nq)) * kRC;
}

// Issue the bulk copies of ring load `i` (lane 0 only).
//   gate/up stage: gate codes | up codes | gate sb superset | up sb superset
//   down stage:    kRC code rows | kRC sb rows
__device__ __forceinline__ void issue_load(const LayerArgs& a, const WarpPlan& p, const CtaShared& cs, int i,
                                           int warp, char* stage, uint64_t* bar, int GW) {
  if (i < p.a.count + p.b.count) {
    int slot, row;
    gu_unit(a, p, i, GW, slot, row);
    const char* blob = cs.blob[slot];
    const long long* o = slot < a.K ? a.off_r : a.off_s;
    const int cb = codes_row_bytes(a.H, slot < a.K ? a.bits_r : a.bits_s);
    const int sbr = sb_row_bytes(a.H);
    const int cap = sb_superset_cap(a.H);
    const long long gs0 = o[1] + (long long)row * sbr, us0 = o[3] + (long long)row * sbr;
    const long long ga = gs0 & ~15LL, ua = us0 & ~15LL;
    const int glen = (int)(((gs0 + sbr + 15) & ~15LL) - ga);
    const int ulen = (int)(((us0 + sbr + 15) & ~15LL) - ua);
    mbar_arrive_expect_tx(bar, 2 * cb + glen + ulen);
    bulk_g2s(stage, blob + o[0] + (long long)row * cb, cb, bar);
    bulk_g2s(stage + cb, blob + o[2] + (long long)row * cb, cb, bar);
    bulk_g2s(stage + 2 * cb, blob + ga, glen, bar);
    bulk_g2s(stage + 2 * cb + cap, blob + ua, ulen, bar);
  } else {
    int slot, r0;
    c_item(p, i, warp, slot, r0);
    const char* blob = cs.blob[slot];
    const long long* o = slot < a.K ? a.off_r : a.off_s;
    const int cb = codes_row_bytes(a.I, slot < a.K ? a.bits_r : a.bits_s);
    const int sbr = sb_row_bytes(a.I);
    mbar_arrive_expect_tx(bar, kRC * (cb + sbr));
    bulk_g2s(stage, blob + o[4] + (long long)r0 * cb, kRC * cb, bar);
    bulk_g2s(stage + kRC * cb, blob + o[5] + (long long)r0 * sbr, kRC * sbr, bar);
  }
}

// ---------------------------------------------------------------------------
// Compute pieces
// ---------------------------------------------------------------------------

// One router row (bf16) against the unscaled input x (shared memory), in
// chunks of 8 16-byte vectors per lane (all loads of a chunk in flight).
constexpr int kRouterChunk = 8;
__device__ __forceinline__ float router_dot(const uint16_t* row, const float* xu, int H, int lane) {
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  const int nv = H / 8;
  float acc = 0.f;
  for (int base = 0; base < nv; base += 32 * kRouterChunk) {
    uint4 w[kRouterChunk];
#pragma unroll
    for (int i = 0; i < kRouterChunk; ++i) {
      const int v = base + lane + 32 * i;
      if (v < nv) w[i] = ld_stream_u4(rv + v);
    }
#pragma unroll
    for (int i = 0; i < kRouterChunk; ++i) {
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

// The same dot product with the row in shared memory: four 16-byte vectors
// per lane in flight (their loads issued together), four accumulators.
__device__ __forceinline__ float router_dot_smem(const uint16_t* row, const float* xu, int H, int lane) {
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  const float4* xv = reinterpret_cast<const float4*>(xu);
  const int nv = H / 8;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int v = lane;
  for (; v + 96 < nv; v += 128) {
    uint4 w[4];
    float4 xa[4], xb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[j] = rv[v + 32 * j];
      xa[j] = xv[2 * (v + 32 * j)];
      xb[j] = xv[2 * (v + 32 * j) + 1];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[j] = fmaf(bf16_lo(w[j].x), xa[j].x, acc[j]);
      acc[j] = fmaf(bf16_hi(w[j].x), xa[j].y, acc[j]);
      acc[j] = fmaf(bf16_lo(w[j].y), xa[j].z, acc[j]);
      acc[j] = fmaf(bf16_hi(w[j].y), xa[j].w, acc[j]);
      acc[j] = fmaf(bf16_lo(w[j].z), xb[j].x, acc[j]);
      acc[j] = fmaf(bf16_hi(w[j].z), xb[j].y, acc[j]);
      acc[j] = fmaf(bf16_lo(w[j].w), xb[j].z, acc[j]);
      acc[j] = fmaf(bf16_hi(w[j].w), xb[j].w, acc[j]);
    }
  }
  for (; v < nv; v += 32) {
    const uint4 w = rv[v];
    const float4 xa = xv[2 * v], xb = xv[2 * v + 1];
    acc[0] = fmaf(bf16_lo(w.x), xa.x, acc[0]);
    acc[1] = fmaf(bf16_hi(w.x), xa.y, acc[1]);
    acc[2] = fmaf(bf16_lo(w.y), xa.z, acc[2]);
    acc[3] = fmaf(bf16_hi(w.y), xa.w, acc[3]);
    acc[0] = fmaf(bf16_lo(w.z), xb.x, acc[0]);
    acc[1] = fmaf(bf16_hi(w.z), xb.y, acc[1]);
    acc[2] = fmaf(bf16_lo(w.w), xb.z, acc[2]);
    acc[3] = fmaf(bf16_hi(w.w), xb.w, acc[3]);
  }
  return warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3]));
}

// Gate and up rows of one expert (stage layout: gate codes | up codes | gate sb
// superset | up sb superset) against the staged input.
template <int BITS, bool kG>
__device__ __forceinline__ void pair_dot_src(const char* st, int H, int sbo_g, int sbo_u, const float4* xs,
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
    const float2 f = ld_in<kG>(sf + v);
    uint64_t ag = 0, au = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t a_ = (&wg.x)[t], b_ = (&wu.x)[t];
      if (BITS == 4) {
        const ulonglong2 xa = ld_in<kG>(xv + (2 * t) * NV + v), xb = ld_in<kG>(xv + (2 * t + 1) * NV + v);
        dot_word4(ag, a_, xa, xb);
        dot_word4(au, b_, xa, xb);
      } else {
        const ulonglong2 x0 = ld_in<kG>(xv + (4 * t) * NV + v), x1 = ld_in<kG>(xv + (4 * t + 1) * NV + v);
        const ulonglong2 x2 = ld_in<kG>(xv + (4 * t + 2) * NV + v), x3 = ld_in<kG>(xv + (4 * t + 3) * NV + v);
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
  // g on lanes 0..15 (lane 0 is the one that uses it), u broadcast
  const float v = warp_sum2_split(g, u, lane);
  g_out = v;
  u_out = __shfl_sync(0xffffffffu, v, 16);
}

template <int BITS>
__device__ __forceinline__ void pair_dot(const char* st, int H, int sbo_g, int sbo_u, const float4* xs,
                                         const float2* sf, int lane, float& g_out, float& u_out) {
  pair_dot_src<BITS, false>(st, H, sbo_g, sbo_u, xs, sf, lane, g_out, u_out);
}


// kRC down rows of one expert (stage layout: kRC code rows | kRC sb rows)
// against that expert's staged activation, which is column block
// [col0, col0 + I/CPV) of a staged [F4][NVS] array (several same-width experts
// staged together); sfa points at column col0.  Returns the full row dots.
template <int BITS, bool kG>
__device__ __forceinline__ void down_rows_src(const char* st, int I, const float4* as, int NVS, int col0,
                                          const float2* sfa, int lane, float (&y)[kRC]) {
  constexpr int CPV = 128 / BITS;
  const int NV = I / CPV;
  const int cb = I * BITS / 8;
  const int ng = I / 64;
  const uint32_t* sb = reinterpret_cast<const uint32_t*>(st + kRC * cb);
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(as + col0);
#pragma unroll
  for (int r = 0; r < kRC; ++r) y[r] = 0.f;
  for (int v = lane; v < NV; v += 32) {
    uint4 w[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) w[r] = reinterpret_cast<const uint4*>(st + r * cb)[v];
    const float2 f = ld_in<kG>(sfa + v);
    const int grp = (BITS == 4) ? (v >> 1) : v;
    uint64_t ac[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) ac[r] = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (BITS == 4) {
        const ulonglong2 xa = ld_in<kG>(xv + (2 * t) * NVS + v), xb = ld_in<kG>(xv + (2 * t + 1) * NVS + v);
#pragma unroll
        for (int r = 0; r < kRC; ++r) dot_word4(ac[r], (&w[r].x)[t], xa, xb);
      } else {
        const ulonglong2 x0 = ld_in<kG>(xv + (4 * t) * NVS + v), x1 = ld_in<kG>(xv + (4 * t + 1) * NVS + v);
        const ulonglong2 x2 = ld_in<kG>(xv + (4 * t + 2) * NVS + v), x3 = ld_in<kG>(xv + (4 * t + 3) * NVS + v);
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
  // row (lane >> 3) & 3 on each lane: lanes 0, 8, 16, 24 hold rows 0..3
  y[0] = warp_sum4_split(y, lane);
}

template <int BITS>
__device__ __forceinline__ void down_rows(const char* st, int I, const float4* as, int NVS, int col0,
                                          const float2* sfa, int lane, float (&y)[kRC]) {
  down_rows_src<BITS, false>(st, I, as, NVS, col0, sfa, lane, y);
}


// Top-K by one warp: descending logit, lower index first on exact ties; then
// renormalised softmax weights over the selected logits.  Logits become
// 32-bit keys whose unsigned order is the float order; each lane holds its
// keys in registers with the position of its largest; a round is one
// warp-wide hardware max of the lanes' largest keys, one hardware min of the
// expert indices that hold it (the tie rule), and a rescan by the winner lane.
__device__ __forceinline__ uint32_t order_bits(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_bits(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// NK keys per lane (16 covers 512 experts, 32 covers 1024).  kShared: the
// logits are in this CTA's shared memory, else in global memory.
template <bool kShared, int NK>
__device__ __noinline__ void warp_topk_n(const float* lg, int n, int k, int lane, int* idx_out, float* w_out) {
  // Keys: order-preserving 32-bit images of the logits (0 = empty).  Each
  // lane keeps the position of its largest key (lowest position on ties);
  // per round the warp takes the largest key, and among equal keys the lowest
  // expert index, and only the winner lane rescans its keys.
  uint32_t key[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const int e = i * 32 + lane;
    key[i] = e < n ? order_bits(kShared ? lg[e] : __ldcg(lg + e)) : 0u;
  }
  uint32_t mine = key[0];
  int mi = 0;
#pragma unroll
  for (int i = 1; i < NK; ++i)
    if (key[i] > mine) { mine = key[i]; mi = i; }
  float my_val = 0.f;
  int my_idx = 0;
#pragma unroll 1
  for (int kk = 0; kk < k; ++kk) {
    const uint32_t h = __reduce_max_sync(0xffffffffu, mine);
    const uint32_t e = __reduce_min_sync(0xffffffffu, mine == h ? (uint32_t)(mi * 32 + lane) : 0xffffffffu);
    if ((int)(e & 31u) == lane) {  // the winner lane drops the key and rescans
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (i == mi) key[i] = 0u;
      mine = key[0];
      mi = 0;
#pragma unroll
      for (int i = 1; i < NK; ++i)
        if (key[i] > mine) { mine = key[i]; mi = i; }
    }
    if (lane == kk) {
      my_val = from_order_bits(h);
      my_idx = (int)e;
    }
  }
  // w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0): softmax restricted to the
  // selected experts, equal to softmax-then-renormalise.
  const float l0 = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = (lane < k) ? expf(my_val - l0) : 0.f;
  const float s = warp_sum(ex);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = ex / s;
  }
}
template <bool kShared>
__device__ __forceinline__ void warp_topk(const float* lg, int n, int k, int lane, int* idx_out, float* w_out) {
  if (n <= 512)
    warp_topk_n<kShared, 16>(lg, n, k, lane, idx_out, w_out);
  else
    warp_topk_n<kShared, kMaxExperts / 32>(lg, n, k, lane, idx_out, w_out);
}

__device__ __forceinline__ float quiet_nan() { return __uint_as_float(0x7FC00000u); }

// A wait of this CTA ran out: report it and poison the CTA.
__device__ __forceinline__ void wait_failed(CtaShared& cs, unsigned status_bit) {
  set_status(status_bit);
  cs.poison = 1;
}

// The tag of this launch: the workspace's epoch + 1, or 0 (never matched) for
// an epoch that no launch leaves (a workspace that was not zeroed).
__device__ __forceinline__ unsigned launch_tag(const unsigned* epoch) {
  const unsigned e = ld_relaxed_gpu(epoch);
  return e <= kEpochWrap ? e + 1u : 0u;
}

// Top-K rounds over keys held by a warp, NK per lane, each with its expert
// index (empty slots: key 0): per round the largest key wins and, among equal
// keys, the lowest expert index; only the winner lane rescans.  A winner's key
// and index are both dropped, so a slice with fewer than k nonzero keys (a
// logit that never arrived) still yields distinct entries.  Lane kk < k ends
// with the kk-th winner's key and index.
template <int NK>
__device__ __forceinline__ void warp_select(uint32_t (&key)[NK], uint32_t (&eix)[NK], int k, int lane,
                                            uint32_t& out_key, uint32_t& out_idx) {
  uint32_t mk = key[0], mx = eix[0];
  int mp = 0;
#pragma unroll
  for (int i = 1; i < NK; ++i)
    if (key[i] > mk || (key[i] == mk && eix[i] < mx)) { mk = key[i]; mx = eix[i]; mp = i; }
  out_key = 0u;
  out_idx = 0u;
#pragma unroll 1
  for (int kk = 0; kk < k; ++kk) {
    const uint32_t h = __reduce_max_sync(0xffffffffu, mk);
    const uint32_t e = __reduce_min_sync(0xffffffffu, mk == h ? mx : 0xffffffffu);
    if (mk == h && mx == e) {  // the winner drops its entry and rescans
#pragma unroll
      for (int i = 0; i < NK; ++i)
        if (i == mp) {
          key[i] = 0u;
          eix[i] = 0xffffffffu;
        }
      mk = key[0];
      mx = eix[0];
      mp = 0;
#pragma unroll
      for (int i = 1; i < NK; ++i)
        if (key[i] > mk || (key[i] == mk && eix[i] < mx)) { mk = key[i]; mx = eix[i]; mp = i; }
    }
    if (lane == kk) {
      out_key = h;
      out_idx = e;
    }
  }
}

// Stage 1 of the CTA's top-K (routing warps).  Each lane holds NKW logits of
// its warp's slice (NKW * 32 consecutive experts from w * NKW * 32) as
// order-preserving keys,
// read from the tagged words as soon as they carry this launch's tag (warp 0's
// lane 0 also reads the shared gate's logit, which it returns); the warp then
// selects the top k of its slice into the candidates.  The tag check replaces
// a grid barrier: a word is this launch's logit or it is not read.
template <int NKW>
__device__ __forceinline__ float slice_topk(const unsigned long long* tlog, int E, int K, bool gated,
                                            uint64_t timeout_ns, unsigned tag, int warp, int lane, CtaShared& cs) {
  uint32_t key[NKW], eix[NKW];
  unsigned pend = 0;
#pragma unroll
  for (int i = 0; i < NKW; ++i) {
    const int e = (warp * NKW + i) * 32 + lane;
    key[i] = 0u;
    eix[i] = e < E ? (uint32_t)e : 0xffffffffu;
    if (e < E) pend |= 1u << i;
  }
  if (warp == 0 && lane == 0 && gated) pend |= 1u << NKW;
  float gate_logit = 0.f;
  uint64_t t0 = 0;
  while (pend) {
    unsigned long long v[NKW + 1];
#pragma unroll
    for (int i = 0; i <= NKW; ++i) {
      const int e = i < NKW ? (warp * NKW + i) * 32 + lane : E;
      v[i] = (pend >> i & 1u) ? ld_relaxed_gpu_u64(tlog + e) : 0ull;
    }
#pragma unroll
    for (int i = 0; i <= NKW; ++i) {
      if ((pend >> i & 1u) && tag != 0u && (unsigned)(v[i] >> 32) == tag) {
        const float l = __uint_as_float((unsigned)v[i]);
        if (i < NKW) key[i] = order_bits(l); else gate_logit = l;
        pend &= ~(1u << i);
      }
    }
    if (!pend) break;
    FMOE_SPIN(2);
    const uint64_t now = globaltimer_ns();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > timeout_ns) {
      wait_failed(cs, kStatusGridBarrierTimeout);
      break;
    }
  }
  FMOE_TRACE_WARP(17);
  uint32_t hk, hi;
  warp_select<NKW>(key, eix, K, lane, hk, hi);
  if (lane < K) {
    cs.cand_key[warp * K + lane] = hk;
    cs.cand_idx[warp * K + lane] = hi;
  }
  return gate_logit;
}

// The routing decision of this CTA, taken by its first kRouteWarps warps
// while the others stage x (layer mode): each routing warp takes the top K of
// its slice of the logits as they are published; after a barrier of the
// routing warps, warp 0 selects the top K of their candidates and computes the
// weights; the CTA barrier that follows (in the kernel) publishes the
// decision to every warp.
// Kept out of line (measured faster than inlined into the kernel).
__device__ __noinline__ void cta_routing(const LayerArgs& a, CtaShared& cs, int warp, int lane, unsigned tag) {
  // Every parameter used here, read once up front: the loads overlap the wait
  // for the logits, and no later store can make the compiler read them again.
  const unsigned long long* const tlog = a.tlog;
  const int E = a.E, K = a.K;
  const bool gated = a.n_router > a.E;
  const uint64_t timeout_ns = a.timeout_ns;
  const char* const experts = a.experts;
  const long long expert_stride = a.expert_stride;
  int* const idx_out = a.idx_out;
  float* const w_out = a.w_out;
  float* const sg_out = a.sg_out;
  float gate_logit;
  if (E <= kRouteWarps * 32 * 2)
    gate_logit = slice_topk<2>(tlog, E, K, gated, timeout_ns, tag, warp, lane, cs);
  else
    gate_logit = slice_topk<kMaxExperts / (kRouteWarps * 32)>(tlog, E, K, gated, timeout_ns, tag, warp, lane, cs);
  FMOE_TRACE_WARP(14);
  // the routing warps' candidates are in shared memory
  asm volatile("bar.sync 1, %0;" ::"r"(kRouteWarps * 32) : "memory");
  FMOE_TRACE_WARP(9);
  if (warp == 0) {
    // Stage 2: warp 0 selects the top K of the kRouteWarps * K candidates
    // (the global top K is among them, ties included) with the same rounds;
    // lane kk < K ends with the kk-th.
    const int nc = kRouteWarps * K;
    constexpr int kC = (kRouteWarps * kMaxTopK + 31) / 32;
    uint32_t ckey[kC], cidx[kC];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      const int c = i * 32 + lane;
      ckey[i] = c < nc ? cs.cand_key[c] : 0u;
      cidx[i] = c < nc ? cs.cand_idx[c] : 0xffffffffu;
    }
    uint32_t hk, hi;
    warp_select<kC>(ckey, cidx, K, lane, hk, hi);
    FMOE_TRACE_WARP(23);
    // w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0): softmax restricted to the
    // selected experts, equal to softmax-then-renormalise.
    const float val = lane < K ? from_order_bits(hk) : 0.f;
    const float l0 = __shfl_sync(0xffffffffu, val, 0);
    const float ex = (lane < K) ? expf(val - l0) : 0.f;
    const float ssum = warp_sum(ex);
    const bool poisoned = cs.poison != 0;  // (a logit never arrived: no plausible routing)
    if (lane < K) {
      const int idx = hi < (uint32_t)E ? (int)hi : 0;  // (always in range)
      const float w = poisoned ? quiet_nan() : ex / ssum;
      cs.w[lane] = w;
      cs.blob[lane] = experts + (long long)idx * expert_stride;
      if (blockIdx.x == 0) {
        if (idx_out) idx_out[lane] = poisoned ? -1 : idx;
        if (w_out) w_out[lane] = w;
      }
    }
    if (lane == 0) {
      const float sg = poisoned ? quiet_nan() : (gated ? sigmoidf_(gate_logit) : 1.0f);
      cs.sg = sg;
      if (blockIdx.x == 0 && sg_out) *sg_out = sg;
    }
    FMOE_TRACE_WARP(10);
  }
}

// Issue phase-C load i (>= a.count + b.count) into the re-carved ring (lane 0).
__device__ __forceinline__ void issue_c(const LayerArgs& a, const WarpPlan& p, const CtaShared& cs, int i,
                                        int warp, char* ring, uint64_t* bars_c, int GW) {
  const int j = i - p.a.count - p.b.count;
  fence_proxy_async_smem();
  issue_load(a, p, cs, i, warp, ring + (size_t)(j % a.nst_c) * a.c_stage_bytes, &bars_c[j % a.nst_c], GW);
}

// BR, BS: code width of the routed experts and of the shared (or single)
// expert; each combination is its own instantiation so a launch carries only
// the dequantisation code it runs.
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) layer_kernel(const __grid_constant__ LayerArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ CtaShared cs;
  const Smem sm = carve_smem(a, smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, GW = G * kWarps;
  const WarpPlan plan = make_plan(a, blockIdx.x, warp, G);
  char* my_ring = sm.ring + (size_t)warp * a.nst * a.stage_bytes;
  uint64_t* my_bars = sm.bars + warp * (a.nst + kMaxNstC);
  uint64_t* my_bars_c = my_bars + a.nst;
  const bool layer_mode = a.n_router > 0;
  const RouterPart rp = router_part(a.n_router, a.H, blockIdx.x, warp, G);
#ifdef FMOE_TRACE_BUILD
  if (tid < kTraceCols) cs.trace[tid] = 0;
#endif
  FMOE_TRACE(0);
  // The next layer decode on the stream may be scheduled now: its CTAs take
  // the SMs this grid's CTAs leave, and do their weight-only set-up while
  // this grid ends.
  grid_dep_launch_dependents();

  // ---- Set-up: weights only until the previous grid on the stream is done ---
  auto router_row_ptr = [&](int e) { return (e < a.E) ? a.w_router + (long long)e * a.H : a.w_sgate; };
  if (tid == 0) {
    mbar_init(&cs.x_bar, 1);
    cs.sg = 1.0f;
    cs.c_prefetch = 0;
    cs.poison = 0;
    // Read every kernel parameter once now, while x is in flight, so that the
    // later first uses (routing, publishing, outputs) hit the constant cache.
    {
      unsigned long long t = (uintptr_t)a.w_router ^ (uintptr_t)a.w_sgate ^ (uintptr_t)a.experts ^
                             (unsigned long long)a.expert_stride ^ (uintptr_t)a.shared ^ (uintptr_t)a.x ^
                             (uintptr_t)a.residual ^ (uintptr_t)a.out ^ (uintptr_t)a.tlog ^ (uintptr_t)a.tact ^
                             (uintptr_t)a.bar ^ (uintptr_t)a.idx_out ^ (uintptr_t)a.w_out ^ (uintptr_t)a.sg_out ^
                             a.timeout_ns;
      t += (unsigned)(a.H ^ a.I ^ a.E ^ a.K ^ a.bits_r ^ a.bits_s ^ a.n_router ^ a.n_slots ^ a.off_a ^ a.off_b ^
                      a.nst ^ a.stage_bytes ^ a.nst_c ^ a.c_stage_bytes ^ a.xs4_off ^ a.xs2_off ^ a.xu_off ^
                      a.vec_floats ^ a.sf_floats ^ a.ys_stride ^ a.router_smem);
      for (int i = 0; i < 6; ++i) t += (unsigned long long)(a.off_r[i] ^ a.off_s[i]);
      t ^= (uintptr_t)a.norm_w ^ (unsigned long long)__float_as_uint(a.norm_eps);
      *(volatile unsigned long long*)&cs.param_touch = t;
    }
    // The shared (or single) expert; the routed slots point at expert 0 until
    // the routing decision replaces them (never read before that).
    for (int k = 0; k < a.K; ++k) cs.blob[k] = a.experts;
    cs.blob[a.K] = a.shared;
    if (a.fixed_route) {  // the routing is given: no router rows, no decision to take
      for (int k = 0; k < a.K; ++k) {
        cs.blob[k] = a.fixed_blob[k];
        cs.w[k] = a.fixed_w[k];
      }
      cs.sg = a.fixed_sg;
    }
    fence_proxy_async_smem();
    // x (issued below, after the dependency wait), and the input-norm weight
    // (into the staging area, free until the staging that follows the norm)
    mbar_arrive_expect_tx(&cs.x_bar, a.H * 4 + (a.norm_w ? a.H * 2 : 0));
    if (a.norm_w) bulk_g2s(sm.vec + (a.xs4_off >= 0 ? a.xs4_off : a.xs2_off), a.norm_w, a.H * 2, &cs.x_bar);
  }
  if (lane == 0) {
    if (rp.on && a.router_smem) {
      // The router segment is the first thing this warp needs after x: bring
      // it into the warp's (still unused) ring now, alongside x.
      mbar_init(&cs.rbar[warp], 1);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&cs.rbar[warp], rp.n * 2);
      bulk_g2s(my_ring, router_row_ptr(rp.row) + rp.seg0, rp.n * 2, &cs.rbar[warp]);
    } else if (rp.on) {
      bulk_prefetch_l2(router_row_ptr(rp.row) + rp.seg0, rp.n * 2);
    }
    for (int s = 0; s < a.nst + kMaxNstC; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  __syncthreads();
  FMOE_TRACE(11);
  // x, the residual, the workspace and the outputs may be the previous grid's:
  // no access to them before it has completed.
  grid_dep_wait();
  FMOE_TRACE(24);
#ifdef FMOE_TRACE_BUILD
  if (tid == 0) cs.trace[kTracePoints] = globaltimer_ns();
#endif
  if (tid == 0) bulk_g2s(sm.vec + a.xu_off, a.x, a.H * 4, &cs.x_bar);
  // The tag of this launch's published words (the epoch the previous launch
  // on this workspace left, plus one).
  const unsigned tag = launch_tag(&a.bar[0]);

  // x and the router rows are the critical path to the routing decision; the
  // shared expert's gate/up rows are requested once the router segments are
  // done with the rings, then every warp stages x.
  int issued = 0;
  if (!mbar_wait_bounded(&cs.x_bar, 0, a.timeout_ns) && lane == 0) wait_failed(cs, kStatusCopyTimeout);
  FMOE_TRACE_WARP(16);
  if (a.norm_w) {
    // Input RMS norm, in place: x <- x / sqrt(mean(x^2) + eps) * w.  Every
    // thread sums the per-warp partials in the same order, so all use the
    // same factor.
    float* xw = sm.vec + a.xu_off;
    const uint16_t* wn = reinterpret_cast<const uint16_t*>(sm.vec + (a.xs4_off >= 0 ? a.xs4_off : a.xs2_off));
    float ss = 0.f;
    for (int i = tid; i < a.H; i += kThreads) ss = fmaf(xw[i], xw[i], ss);
    ss = warp_sum(ss);
    if (lane == 0) cs.red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += cs.red[w];
    const float r = 1.0f / sqrtf(tot / (float)a.H + a.norm_eps);
    for (int i = tid; i < a.H; i += kThreads) xw[i] = xw[i] * r * __uint_as_float((uint32_t)wn[i] << 16);
    __syncthreads();
  }
  const float* xu = sm.vec + a.xu_off;
  if (rp.nr > 0) {  // (uniform over the CTA)
    // ---- Phase A, router rows: segment dot products, then each row's sum
    // (fixed order) published as one tagged word ---------------------------------
    if (rp.on) {
      float l;
      if (a.router_smem) {
        if (!mbar_wait_bounded(&cs.rbar[warp], 0, a.timeout_ns) && lane == 0) wait_failed(cs, kStatusCopyTimeout);
        FMOE_TRACE_WARP(20);
        l = router_dot_smem(reinterpret_cast<const uint16_t*>(my_ring), xu + rp.seg0, rp.n, lane);
      } else {
        l = router_dot(router_row_ptr(rp.row) + rp.seg0, xu + rp.seg0, rp.n, lane);
      }
      FMOE_TRACE_WARP(21);
      if (lane == 0) cs.rpart[warp] = l;
    }
    __syncthreads();
    if (rp.on && warp % rp.wpr == 0 && lane == 0) {
      float l = cs.rpart[warp];
      for (int q = 1; q < rp.wpr; ++q) l += cs.rpart[warp + q];
      st_relaxed_gpu_u64(a.tlog + rp.row, ((unsigned long long)tag << 32) | __float_as_uint(cs.poison ? quiet_nan() : l));
      FMOE_TRACE_WARP(22);
    }
    FMOE_TRACE_WARP(2);
  }
  // The shared expert's gate/up loads (no routing decision needed).  A router
  // warp's ring held its segment: its reads come before the copies.
  if (lane == 0) {
    if (rp.on && a.router_smem) fence_proxy_async_smem();
    while (issued < plan.a.count && issued < a.nst) {
      issue_load(a, plan, cs, issued, warp, my_ring + (size_t)issued * a.stage_bytes, &my_bars[issued], GW);
      ++issued;
    }
  }
  issued = __shfl_sync(0xffffffffu, issued, 0);
  if (layer_mode && warp < kRouteWarps) {
    // ---- Routing decision (the first kRouteWarps warps) ------------------------
    cta_routing(a, cs, warp, lane, tag);
  } else {
    // ---- Stage x into the decode layouts (the other warps, meanwhile) ---------
    // (each width the launch uses: a given-routing launch without routed
    // experts has no routed width, whatever its instantiation)
    const int w0 = layer_mode ? kRouteWarps * 32 : 0;
    const int t0 = tid - w0, nt = kThreads - w0;
    if ((BR == 4 || BS == 4) && a.xs4_off >= 0)
      stage_inputs<4, false>(xu, a.H, reinterpret_cast<float4*>(sm.vec + a.xs4_off), sm.sf, t0, nt);
    if ((BR == 2 || BS == 2) && a.xs2_off >= 0)
      stage_inputs<2, false>(xu, a.H, reinterpret_cast<float4*>(sm.vec + a.xs2_off),
                             sm.sf + (a.xs4_off >= 0 ? a.H / 32 : 0), t0, nt);
    __syncwarp();
    FMOE_TRACE_WARP(18);
    if (warp == kWarps - 1 && lane == 0 && a.shared && plan.nq > 0) {
      // the shared expert's down rows of this CTA are known from the start
      const BlobOff o = blob_offsets(a.H, a.I, BS);
      const int cb = codes_row_bytes(a.I, BS), sbr = sb_row_bytes(a.I);
      const long long r0 = (long long)plan.q0 * kRC, nr = (long long)plan.nq * kRC;
      bulk_prefetch_l2(a.shared + o.dc + r0 * cb, (uint32_t)(nr * cb));
      bulk_prefetch_l2(a.shared + o.dsb + r0 * sbr, (uint32_t)(nr * sbr));
    }
  }
  // the routing decision and the staged x reach every warp
  __syncthreads();
  FMOE_TRACE(1);
  FMOE_TRACE_WARP(3);

  // ---- Ring loop over phases A (static gate/up) and B (routed gate/up) ------
  const int n_gu = plan.a.count + plan.b.count;
  const float4* xs4 = reinterpret_cast<const float4*>(sm.vec + (a.xs4_off >= 0 ? a.xs4_off : 0));
  const float4* xs2 = reinterpret_cast<const float4*>(sm.vec + (a.xs2_off >= 0 ? a.xs2_off : 0));
  const float2* sf4 = sm.sf;
  const float2* sf2 = sm.sf + (a.xs4_off >= 0 ? a.H / 32 : 0);

  // The routing decision is known from here on: issue freely.
  for (int i = 0; i < n_gu; ++i) {
    if (lane == 0) {
      while (issued < n_gu && issued < i + a.nst) {
        fence_proxy_async_smem();
        issue_load(a, plan, cs, issued, warp, my_ring + (size_t)(issued % a.nst) * a.stage_bytes,
                   &my_bars[issued % a.nst], GW);
        ++issued;
      }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);
    const int st_i = i % a.nst;
    const char* stage = my_ring + (size_t)st_i * a.stage_bytes;
    if (!mbar_wait_bounded(&my_bars[st_i], (i / a.nst) & 1, a.timeout_ns) && lane == 0)
      wait_failed(cs, kStatusCopyTimeout);
    if (i == n_gu - 1) FMOE_TRACE_WARP(13);
    if (i == 0 && plan.a.count > 0) FMOE_TRACE_WARP(19);
    int slot, row;
    gu_unit(a, plan, i, GW, slot, row);
    const bool routed = slot < a.K;
    const long long* o = routed ? a.off_r : a.off_s;
    const int sbr = sb_row_bytes(a.H);
    const int sbo_g = (int)((o[1] + (long long)row * sbr) & 15);
    const int sbo_u = (int)((o[3] + (long long)row * sbr) & 15);
    float g, u;
    if (BR == BS || routed)
      pair_dot<BR>(stage, a.H, sbo_g, sbo_u, BR == 4 ? xs4 : xs2, BR == 4 ? sf4 : sf2, lane, g, u);
    else
      pair_dot<BS>(stage, a.H, sbo_g, sbo_u, BS == 4 ? xs4 : xs2, BS == 4 ? sf4 : sf2, lane, g, u);
    if (lane == 0) {
      const float act = cs.poison ? quiet_nan() : g * sigmoidf_(g) * u;
      st_relaxed_gpu_u64(a.tact + (long long)slot * a.I + row, ((unsigned long long)tag << 32) | __float_as_uint(act));
    }
    __syncwarp();
  }

  // Gate/up work of this warp is done (its ring is free): re-carve the ring
  // into down-item stages and put this warp's down items in flight before
  // joining the hand-off, so they stream during the wait.
  // The CTA's first warp through its gate/up work asks L2 for the routed
  // experts' down rows of this CTA (one lane per routed slot): late enough not
  // to compete with the gate/up stream, early enough to land before phase C.
  if (a.K > 0 && plan.nq > 0) {
    int first = 0;
    if (lane == 0) first = atomicAdd(&cs.c_prefetch, 1) == 0;
    if (__shfl_sync(0xffffffffu, first, 0) && lane < a.K) {
      const SlotInfo si = slot_info(a, cs, lane);
      const BlobOff o = blob_offsets(a.H, a.I, BR);
      const int cb = codes_row_bytes(a.I, BR), sbr = sb_row_bytes(a.I);
      const long long r0 = (long long)plan.q0 * kRC, nr = (long long)plan.nq * kRC;
      bulk_prefetch_l2(si.blob + o.dc + r0 * cb, (uint32_t)(nr * cb));
      bulk_prefetch_l2(si.blob + o.dsb + r0 * sbr, (uint32_t)(nr * sbr));
    }
  }
  int issued_c = n_gu;
  if (lane == 0)
    while (issued_c < plan.n_loads && issued_c < n_gu + a.nst_c) {
      issue_c(a, plan, cs, issued_c, warp, my_ring, my_bars_c, GW);
      ++issued_c;
    }
  issued_c = __shfl_sync(0xffffffffu, issued_c, 0);

  // ---- Hand-off: poll and stage every activation of the grid ----------------
  // (the staged activations overwrite the staged x: every warp of the CTA is
  // past its gate/up work first).  With one code width every slot (back to
  // back in the workspace) is staged in one pass, as one [F4][n_slots*I/CPV]
  // array; otherwise the K routed experts in one pass and the shared expert in
  // a second, its own [F4][I/CPV] array at sm.vec + K * I.  Slot s's scale
  // pairs start at sm.sf + s * I / CPV either way.
  FMOE_TRACE_WARP(4);
  __syncthreads();
  FMOE_TRACE(5);
  if (plan.nq > 0) {
    bool ok = true;
    if (BR == BS) {
      ok = stage_tagged<BR>(a.tact, a.n_slots * a.I, reinterpret_cast<float4*>(sm.vec), sm.sf, tid, kThreads, tag,
                            a.timeout_ns);
    } else {
      if (a.K > 0)
        ok = stage_tagged<BR>(a.tact, a.K * a.I, reinterpret_cast<float4*>(sm.vec), sm.sf, tid, kThreads, tag,
                              a.timeout_ns);
      if (a.n_slots > a.K)
        ok &= stage_tagged<BS>(a.tact + (long long)a.K * a.I, a.I, reinterpret_cast<float4*>(sm.vec + a.K * a.I),
                               sm.sf + a.K * a.I * BR / 128, tid, kThreads, tag, a.timeout_ns);
    }
    if (!ok) wait_failed(cs, kStatusGridBarrierTimeout);
  }
  FMOE_TRACE(6);
  __syncthreads();

  // ---- Phase C: down projections of this CTA's rows, one (slot, kRC rows)
  // item per re-carved stage; the row dots go to shared memory -----------------
  for (int i = n_gu; i < plan.n_loads; ++i) {
    const int j = i - n_gu;
    if (lane == 0)
      while (issued_c < plan.n_loads && issued_c < i + a.nst_c) {
        issue_c(a, plan, cs, issued_c, warp, my_ring, my_bars_c, GW);
        ++issued_c;
      }
    issued_c = __shfl_sync(0xffffffffu, issued_c, 0);
    const char* stage = my_ring + (size_t)(j % a.nst_c) * a.c_stage_bytes;
    if (!mbar_wait_bounded(&my_bars_c[j % a.nst_c], (j / a.nst_c) & 1, a.timeout_ns) && lane == 0)
      wait_failed(cs, kStatusCopyTimeout);
    if (j == 0) FMOE_TRACE_WARP(15);
    int slot, r0;
    c_item(plan, i, warp, slot, r0);
    const bool routed = slot < a.K;
    const int cpv = 128 / (routed ? BR : BS);
    // One code width: every slot is column block slot of one staged array.
    // Otherwise the routed slots share one [F4][K*I/CPV] array and the shared
    // slot has its own [F4][I/CPV] array after it.
    const bool one = BR == BS || routed;
    const float4* as = reinterpret_cast<const float4*>(sm.vec + (one ? 0 : a.K * a.I));
    const int nvs = (BR == BS ? a.n_slots : routed ? a.K : 1) * (a.I / cpv);
    const int col0 = one ? slot * (a.I / cpv) : 0;
    const float2* sfa = sm.sf + (one ? 0 : a.K * a.I * BR / 128) + col0;
    float y[kRC];
    if (BR == BS || routed)
      down_rows<BR>(stage, a.I, as, nvs, col0, sfa, lane, y);
    else
      down_rows<BS>(stage, a.I, as, nvs, col0, sfa, lane, y);
    if (j == 0) FMOE_TRACE_WARP(12);
    if ((lane & 7) == 0) sm.ys[slot * a.ys_stride + (r0 - plan.q0 * kRC) + (lane >> 3)] = y[0];
    __syncwarp();
  }
  FMOE_TRACE_WARP(7);
  __syncthreads();

  // ---- Combine: out = residual + sum_k w_k y_k + sg * y_shared, fixed order ---
  for (int t = tid; t < plan.nq * kRC; t += kThreads) {
    const int r = plan.q0 * kRC + t;
    float v = a.residual ? __ldg(a.residual + r) : 0.f;
    for (int s = 0; s < a.n_slots; ++s) v = fmaf(s < a.K ? cs.w[s] : cs.sg, sm.ys[s * a.ys_stride + t], v);
    a.out[r] = cs.poison ? quiet_nan() : v;
  }

  // ---- Done: the last CTA advances the epoch and resets the counters -------
  __syncthreads();
  FMOE_TRACE(8);
  if (tid == 0) cs.last = atomicAdd(&a.bar[2], 1u) + 1u == (unsigned)G;
  __syncthreads();
  if (cs.last) {
    // Every CTA is past its last use of the epoch.  Before the epoch would
    // pass kEpochWrap (or when it is not a valid epoch) every tagged word is
    // cleared (tag 0 never matches) and it restarts at 0, so no word left by
    // an earlier launch ever carries a later launch's tag.
    const unsigned ep = ld_relaxed_gpu(&a.bar[0]);
    const bool wrap = ep >= kEpochWrap;
    if (wrap) {
      if (a.tlog)
        for (int e = tid; e < kTagWords; e += kThreads) st_relaxed_gpu_u64(a.tlog + e, 0ull);
      for (int e = tid; e < kActWords; e += kThreads) st_relaxed_gpu_u64(a.tact + e, 0ull);
    }
    __syncthreads();
    if (tid == 0) {
      atomicExch(&a.bar[0], wrap ? 0u : ep + 1u);
      atomicExch(&a.bar[1], 0u);
      atomicExch(&a.bar[2], 0u);
      __threadfence();
    }
  }
#ifdef FMOE_TRACE_BUILD
  if (tid == 0 && blockIdx.x < 1024) {
    cs.trace[kTracePoints + 2] = clock64();
    cs.trace[kTracePoints + 1] = globaltimer_ns();
    for (int i = 0; i < kTraceCols; ++i) g_fmoe_trace[blockIdx.x][i] = cs.trace[i];
  }
#endif
}

}  // namespace fmoe
