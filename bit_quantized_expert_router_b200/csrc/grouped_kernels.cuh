// Grouped decode: T tokens (2 <= T <= 16) through one MoE layer at once.
//
// What it computes is the single-token layer of the Flash-MoE pages ("Flash-MoE:
// Ausführen eines 397B-Parameter-Qwen-Modells ...", sections "Pipeline-Leistung"
// and "Metal-Compute-Shader") for every token independently: router, softmax,
// top-K with renormalised weights, the selected experts plus the shared one as
// dequantised gate/up, SwiGLU, down, and the gated combine with the residual.
// The pages decode one token at a time; with several tokens the weights of an
// expert chosen by n tokens are read once and applied to all n.
//
// Steps (one launch each, all on the caller's stream):
//   router   logits[t][e] for every token; each CTA owns a few router rows and
//            reads every token's input once;
//   prep     CTA 0: top-K per token (one warp each), then the grouping: the
//            (token, k) pairs sorted by (expert, token), one slot per distinct
//            expert in ascending expert order, the shared expert last with all
//            T tokens; CTAs 1..T: each token's input staged in the decode
//            layouts (stage_inputs) into the workspace;
//   gate/up  units (slot, input chunk, row); every unit reads its gate and up
//            row chunk once and applies it to each token of the slot, giving
//            partial dot products per chunk;
//   stage    per pair: the chunk partials summed in order, silu(g) * u, and the
//            activation staged for the down projection;
//   down     units (slot, input chunk, 4 output rows), as gate/up;
//   combine  per token and output row: residual + sum_k w_k y_k + sg * y_shared
//            with each y summed over its chunks in order.
// Scheduling of gate/up and down: the units are ordered (slot, chunk, row)
// and cut into one contiguous range per CTA of equal estimated cost (bytes
// plus per-token work); inside a CTA consecutive units go to consecutive
// warps, so the warps of a CTA work on the same slot and chunk at the same
// time and share its staged inputs through L1.  A slot with many tokens has
// its inputs split into chunks so that one chunk of all its tokens' inputs
// stays within a fixed budget.  No float atomics: every sum has a fixed
// order, so results are bitwise reproducible.
#pragma once
#include "route_quant_kernels.cuh"

namespace fmoe {

constexpr int kMaxTokens = 16;
constexpr int kMaxPairs = kMaxTokens * kMaxTopK + kMaxTokens;
constexpr int kMaxChunks = 8;              // input chunks per slot, at most
constexpr int kChunkBudget = 32 << 10;     // bytes of staged inputs of one (slot, chunk)
constexpr int kUnitCostBase = 2;           // unit cost = chunk length * (kUnitCostBase + tokens)
constexpr int kRouterRows = 4;             // router rows per CTA
constexpr int kMaxSchedCtas = 1024;        // CTAs of the gate/up and down grids, at most
// Unit schedule of one grid (gate/up or down), ints: every slot's input
// chunks and inputs per chunk, every slot's first unit (and the total), every
// CTA's first unit (and the total).
constexpr int kSchedNk = 0, kSchedCl = kMaxPairs + 1, kSchedUbase = 2 * (kMaxPairs + 1);
constexpr int kSchedRange = kSchedUbase + kMaxPairs + 2;
constexpr int kSchedInts = kSchedRange + kMaxSchedCtas + 1;

// Chunks the n_in inputs of a slot with n_tok tokens are split into: the
// fewest (a divisor of n_in / 64, at most kMaxChunks) that keep n_tok chunks of
// staged fp32 inputs within kChunkBudget, else the most allowed.
__host__ __device__ inline int input_chunks(int n_tok, int n_in) {
  const int ng = n_in / 64;
  int best = 1;
  for (int d = 1; d <= kMaxChunks && d <= ng; ++d) {
    if (ng % d) continue;
    best = d;
    if ((long long)n_tok * (n_in / d) * 4 <= kChunkBudget) return d;
  }
  return best;
}

// Grouping tables (workspace).
struct GroupTables {
  int* meta;         // [0] slots, [1] pairs (routed pairs, then one shared pair per token)
  int* slot_expert;  // [slots] expert id, -1 = the shared expert
  int* slot_pair0;   // [slots + 1] first pair of each slot
  int* pair_token;   // [pairs]
  int* pair_slot;    // [pairs]
  int* pair_nk;      // [pairs] input chunks of the pair's slot: gate/up (bits 0-7), down (bits 8-15)
  int* tok_pair;     // [T][K + 1] pair of (t, k); column K: the shared pair (-1 if none)
  float* tok_w;      // [T][K]
  float* tok_sg;     // [T]
  int* sched;        // [2][kSchedInts] unit schedules of the gate/up (0) and down (1) grids
};

struct GroupArgs {
  const char* experts;
  long long expert_stride;
  const char* shared;     // or null
  const float* x;         // [T][H]
  const float* residual;  // [T][H] or null
  float* out;             // [T][H]
  const float* logits;    // [T][E + 1]
  GroupTables tb;
  float4* xs_r;     // [T][H/4] staged inputs for the routed code width
  float2* sf_r;     // [T][H*BR/128]
  float4* xs_s;     // same for the shared expert's width (aliases xs_r when equal)
  float2* sf_s;
  float2* gu_part;  // [pairs][kMaxChunks][I] {gate, up} partial dot products
  float4* as;       // [pairs][I/4] staged activations
  float2* sfa;      // [pairs][I/32]
  float* y_part;    // [pairs][kMaxChunks][H] partial down projections
  int* idx_out;     // optional [T][K]
  float* w_out;     // optional [T][K]
  const uint16_t* w_router;  // [E][H] bf16
  const uint16_t* w_sgate;   // [H] bf16 or null
  float* sh_gu;     // tensor-core shared expert: [2][H/512][16][I] gate/up partials
  float* sh_y;      // [I/512][16][H] down partials
  int H, I, E, K, T, bits_r, bits_s;
  int grid;         // CTAs of the gate/up and down grids
  int has_sgate;
  int shared_tc;    // the shared expert runs on the tensor cores (not as a slot)
  int nst, stage_bytes;      // gate/up ring
  int nst_c, c_stage_bytes;  // down ring
  long long off_r[6], off_s[6];
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------------------
// router: logits[t][r] = W_r[r] . x[t] (row E: the shared gate vector)
// ---------------------------------------------------------------------------
// Router rows r0 .. r0 + kRouterRows - 1 for all T tokens; all threads of the
// CTA call it.  Each thread takes 16-byte weight vectors of the rows and the
// matching inputs of every token; per-warp sums are combined in fixed order.
__device__ __noinline__ void router_rows_tokens(const uint16_t* __restrict__ w_router,
                                                const uint16_t* __restrict__ w_sgate, const float* __restrict__ x,
                                                int T, int H, int E, int r0, float* __restrict__ logits) {
  __shared__ float part[kWarps][kRouterRows * kMaxTokens];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rows = E + (w_sgate ? 1 : 0);
  float acc[kRouterRows][kMaxTokens];
#pragma unroll
  for (int r = 0; r < kRouterRows; ++r)
#pragma unroll
    for (int t = 0; t < kMaxTokens; ++t) acc[r][t] = 0.f;
  const int nv = H / 8;  // 16-byte vectors of 8 bf16 weights
  for (int v = tid; v < nv; v += kThreads) {
    uint4 w[kRouterRows];
#pragma unroll
    for (int r = 0; r < kRouterRows; ++r) {
      const int row = r0 + r;
      w[r] = make_uint4(0u, 0u, 0u, 0u);
      if (row < rows) w[r] = ld_stream_u4((row < E ? w_router + (long long)row * H : w_sgate) + 8 * v);
    }
#pragma unroll
    for (int t = 0; t < kMaxTokens; ++t) {
      if (t < T) {
        const float4* xt = reinterpret_cast<const float4*>(x + (long long)t * H) + 2 * v;
        const float4 xa = __ldg(xt), xb = __ldg(xt + 1);
#pragma unroll
        for (int r = 0; r < kRouterRows; ++r) {
          float s = acc[r][t];
          s = fmaf(bf16_lo(w[r].x), xa.x, s);
          s = fmaf(bf16_hi(w[r].x), xa.y, s);
          s = fmaf(bf16_lo(w[r].y), xa.z, s);
          s = fmaf(bf16_hi(w[r].y), xa.w, s);
          s = fmaf(bf16_lo(w[r].z), xb.x, s);
          s = fmaf(bf16_hi(w[r].z), xb.y, s);
          s = fmaf(bf16_lo(w[r].w), xb.z, s);
          s = fmaf(bf16_hi(w[r].w), xb.w, s);
          acc[r][t] = s;
        }
      }
    }
  }
  // Transposed warp reduction of the 64 sums: each of 5 halving steps keeps
  // the half of the values selected by one lane bit and adds the partner's
  // copy of it (62 shuffles in all); lane l ends with sums 2l and 2l + 1
  // (index r * 16 + t).
  {
    float* v = &acc[0][0];
#pragma unroll
    for (int o = 16, n = kRouterRows * kMaxTokens; o >= 1; o >>= 1, n >>= 1) {
      const bool hi = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < n / 2; ++j) {
        const float keep = hi ? v[j + n / 2] : v[j];
        const float send = hi ? v[j] : v[j + n / 2];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    part[warp][2 * lane] = v[0];
    part[warp][2 * lane + 1] = v[1];
  }
  static_assert(kRouterRows * kMaxTokens == 64, "the transposed reduction assumes 64 sums per lane");
  __syncthreads();
  if (tid < kRouterRows * T) {
    const int r = tid / T, t = tid - r * T, row = r0 + r;
    float s = 0.f;
    for (int w = 0; w < kWarps; ++w) s += part[w][r * kMaxTokens + t];
    if (row < rows) logits[(long long)t * (E + 1) + row] = s;
  }
  __syncthreads();  // `part` is reused by the next call
}

__global__ void __launch_bounds__(kThreads) router_tokens_kernel(const uint16_t* __restrict__ w_router,
                                                                 const uint16_t* __restrict__ w_sgate,
                                                                 const float* __restrict__ x, int T, int H, int E,
                                                                 float* __restrict__ logits) {
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  router_rows_tokens(w_router, w_sgate, x, T, H, E, blockIdx.x * kRouterRows, logits);
}

// ---------------------------------------------------------------------------
// input RMS norm: xn[t] = x[t] / sqrt(mean(x[t]^2) + eps) * w (one CTA per token)
// ---------------------------------------------------------------------------
constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads) rms_norm_tokens_kernel(const float* __restrict__ x,
                                                                       const uint16_t* __restrict__ w, float eps,
                                                                       int H, float* __restrict__ xn) {
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  __shared__ float red[kNormThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* xt = x + (long long)blockIdx.x * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += kNormThreads) ss = fmaf(xt[i], xt[i], ss);
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
  const float r = 1.0f / sqrtf(tot / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += kNormThreads)
    xn[(long long)blockIdx.x * H + i] = xt[i] * r * __uint_as_float((uint32_t)__ldg(w + i) << 16);
}

// ---------------------------------------------------------------------------
// Unit schedules of the gate/up (q = 0: kin = H inputs, ru = I row units per
// chunk) and down (q = 1: kin = I, ru = H / kRC) grids.  The units of slot s
// are its input chunks x ru row units, chunk-major; slot after slot in slot
// order.  A unit costs (kin / chunks) * (kUnitCostBase + tokens of the slot)
// (bytes read plus per-token work); CTA b of G takes the units whose cost
// intervals start in [total * b / G, total * (b + 1) / G).  Computed once by
// all threads of the grouping CTA: per-slot values in parallel, prefix sums by
// one thread per slot, each CTA's first unit by one thread per CTA.
// ---------------------------------------------------------------------------
__device__ __noinline__ void schedule_units(const GroupArgs& a) {
  __shared__ long long s_cost[2][kMaxPairs + 2];  // cost of slot s, then cost before slot s
  __shared__ int s_units[2][kMaxPairs + 2];       // units of slot s, then units before slot s
  __shared__ int s_n[kMaxPairs + 1];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int ns = a.tb.meta[0], G = a.grid;
  for (int i = tid; i < 2 * ns; i += nt) {
    const int q = i / ns, s = i - q * ns;
    const int kin = q ? a.I : a.H, ru = q ? a.H / kRC : a.I;
    const int n = a.tb.slot_pair0[s + 1] - a.tb.slot_pair0[s];
    const int nk = input_chunks(n, kin);
    if (q == 0) s_n[s] = n;
    a.tb.sched[q * kSchedInts + kSchedNk + s] = nk;
    a.tb.sched[q * kSchedInts + kSchedCl + s] = kin / nk;
    s_units[q][s] = nk * ru;
    s_cost[q][s] = (long long)ru * kin * (kUnitCostBase + n);
  }
  __syncthreads();
  long long cb = 0;
  int ub = 0;
  const int q0 = tid / (ns + 1), s0 = tid - q0 * (ns + 1);
  if (tid < 2 * (ns + 1)) {  // sums over the slots before s0
    for (int j = 0; j < s0; ++j) {
      cb += s_cost[q0][j];
      ub += s_units[q0][j];
    }
    a.tb.sched[q0 * kSchedInts + kSchedUbase + s0] = ub;
  }
  __syncthreads();
  if (tid < 2 * (ns + 1)) {
    s_cost[q0][s0] = cb;
    s_units[q0][s0] = ub;
  }
  __syncthreads();
  for (int i = tid; i < 2 * (G + 1); i += nt) {
    const int q = i / (G + 1), b = i - q * (G + 1);
    const long long target = s_cost[q][ns] * b / G;
    int u = s_units[q][ns];  // first unit whose cost interval starts at or after target
    for (int s = 0; s < ns; ++s) {
      if (target < s_cost[q][s + 1]) {
        const long long uc = (long long)a.tb.sched[q * kSchedInts + kSchedCl + s] * (kUnitCostBase + s_n[s]);
        u = s_units[q][s] + (int)((target - s_cost[q][s] + uc - 1) / uc);
        break;
      }
    }
    a.tb.sched[q * kSchedInts + kSchedRange + b] = u;
  }
}

// ---------------------------------------------------------------------------
// prep: top-K per token, grouping, input staging
// ---------------------------------------------------------------------------
// CTA `b` of the prep step (0 <= b <= T): b = 0 routes and groups, b > 0
// stages token b - 1's input.
template <int BR, int BS>
__device__ __noinline__ void prep_cta(const GroupArgs& a, int b) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool shared_slot = a.shared != nullptr && !a.shared_tc;  // the shared expert runs as a slot
  if (b > 0) {
    const int t = b - 1;
    const float* x = a.x + (long long)t * a.H;
    stage_inputs<BR, true>(x, a.H, a.xs_r + (long long)t * (a.H / 4), a.sf_r + (long long)t * (a.H * BR / 128), tid,
                           kThreads);
    if (shared_slot && a.xs_s != a.xs_r)
      stage_inputs<BS, true>(x, a.H, a.xs_s + (long long)t * (a.H / 4), a.sf_s + (long long)t * (a.H * BS / 128),
                             tid, kThreads);
    return;
  }
  __shared__ int s_idx[kMaxTokens * kMaxTopK];
  __shared__ float s_w[kMaxTokens * kMaxTopK];
  __shared__ int s_se[kMaxTokens * kMaxTopK];  // expert of sorted pair p
  __shared__ int s_start[kMaxTokens * kMaxTopK];
  __shared__ int s_slot[kMaxTokens * kMaxTopK];
  const int T = a.T, K = a.K, NP = T * K;
  if (warp < T) {
    const float* lt = a.logits + (long long)warp * (a.E + 1);
    warp_topk<false>(lt, a.E, K, lane, s_idx + warp * K, s_w + warp * K);
    if (lane == 0) a.tb.tok_sg[warp] = a.has_sgate ? sigmoidf_(__ldcg(lt + a.E)) : 1.0f;
  }
  __syncthreads();
  if (tid < NP) {
    int e = s_idx[tid];
    if (e < 0 || e >= a.E) e = 0;  // (cannot happen: top-K indices lie in [0, E))
    s_idx[tid] = e;
  }
  __syncthreads();
  // Rank of pair j = t*K + k in (expert, j) order, i.e. (expert, token) order
  // since a token's top-K experts are distinct; ties on j keep the ranks a
  // permutation whatever the indices are.
  if (tid < NP) {
    const int e = s_idx[tid], t = tid / K;
    int rank = 0;
    for (int j = 0; j < NP; ++j) {
      const int e2 = s_idx[j];
      rank += (e2 < e) || (e2 == e && j < tid);
    }
    s_se[rank] = e;
    a.tb.pair_token[rank] = t;
    a.tb.tok_pair[t * (K + 1) + tid % K] = rank;
    if (a.idx_out) a.idx_out[tid] = e;
    if (a.w_out) a.w_out[tid] = s_w[tid];
    a.tb.tok_w[tid] = s_w[tid];
  }
  __syncthreads();
  if (tid < NP) s_start[tid] = (tid == 0) || s_se[tid] != s_se[tid - 1];
  __syncthreads();
  if (tid < NP) {
    int slot = -1;
    for (int j = 0; j <= tid; ++j) slot += s_start[j];
    s_slot[tid] = slot;
    a.tb.pair_slot[tid] = slot;
    if (s_start[tid]) {
      a.tb.slot_expert[slot] = s_se[tid];
      a.tb.slot_pair0[slot] = tid;
    }
  }
  __syncthreads();
  if (tid < NP) {  // tokens of this pair's slot -> its chunk counts
    int n = 0;
    for (int j = 0; j < NP; ++j) n += s_slot[j] == s_slot[tid];
    a.tb.pair_nk[tid] = input_chunks(n, a.H) | (input_chunks(n, a.I) << 8);
  }
  const int nr = NP > 0 ? s_slot[NP - 1] + 1 : 0;
  if (tid < T) {
    a.tb.tok_pair[tid * (K + 1) + K] = shared_slot ? NP + tid : -1;
    if (shared_slot) {
      a.tb.pair_token[NP + tid] = tid;
      a.tb.pair_slot[NP + tid] = nr;
      a.tb.pair_nk[NP + tid] = input_chunks(T, a.H) | (input_chunks(T, a.I) << 8);
    }
  }
  if (tid == 0) {
    int ns = nr, np = NP;
    if (shared_slot) {
      a.tb.slot_expert[nr] = -1;
      a.tb.slot_pair0[nr] = NP;
      ns = nr + 1;
      np = NP + T;
    }
    a.tb.slot_pair0[ns] = np;
    a.tb.meta[0] = ns;
    a.tb.meta[1] = np;
  }
  __syncthreads();  // (the tables above are read back by this CTA's threads)
  schedule_units(a);
}

template <int BR, int BS>
__global__ void __launch_bounds__(kThreads) grouped_prep_kernel(const __grid_constant__ GroupArgs a) {
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  prep_cta<BR, BS>(a, blockIdx.x);
}

// ---------------------------------------------------------------------------
// Unit scheduling shared by gate/up and down
// ---------------------------------------------------------------------------
// Units of slot s: input_chunks(n_s, kin) chunks x ru row units, chunk-major.
struct CtaSched {
  int ns;
  int* pair0;   // [ns + 1]
  int* expert;  // [ns]
  int* nk;      // [ns] input chunks
  int* cl;      // [ns] inputs per chunk
  int* ubase;   // [ns + 1] units before slot s
  int* ptok;    // [pairs] token of each pair
  int u0, u1;   // this CTA's units
};

// Shared-memory copies of the slot tables, declared by each grid's kernel.
struct SchedSmem {
  int pair0[kMaxPairs + 2], expert[kMaxPairs + 1], nk[kMaxPairs + 1], cl[kMaxPairs + 1], ubase[kMaxPairs + 2];
  int ptok[kMaxPairs];
  int range[2];
};

// Load the slot tables and this CTA's unit range of grid q (0 gate/up, 1
// down) from the schedule the grouping step computed; all threads call it.
__device__ inline void cta_sched(const GroupArgs& a, int q, CtaSched& cs, SchedSmem& sm) {
  const int tid = threadIdx.x;
  const int ns = a.tb.meta[0], np = a.tb.meta[1];
  const int* t = a.tb.sched + q * kSchedInts;
  for (int s = tid; s <= ns; s += blockDim.x) {
    sm.pair0[s] = a.tb.slot_pair0[s];
    sm.ubase[s] = t[kSchedUbase + s];
    if (s < ns) {
      sm.expert[s] = a.tb.slot_expert[s];
      sm.nk[s] = t[kSchedNk + s];
      sm.cl[s] = t[kSchedCl + s];
    }
  }
  for (int p = tid; p < np; p += blockDim.x) sm.ptok[p] = a.tb.pair_token[p];
  if (tid < 2) sm.range[tid] = t[kSchedRange + blockIdx.x + tid];
  __syncthreads();
  cs.ns = ns;
  cs.pair0 = sm.pair0;
  cs.expert = sm.expert;
  cs.nk = sm.nk;
  cs.cl = sm.cl;
  cs.ubase = sm.ubase;
  cs.ptok = sm.ptok;
  cs.u0 = sm.range[0];
  cs.u1 = sm.range[1];
}

// (slot, chunk, row unit) of unit u; `s` is a cursor that only moves forward.
__device__ __forceinline__ void locate(const CtaSched& cs, int ru, int u, int& s, int& c, int& r) {
  while (cs.ubase[s + 1] <= u) ++s;
  const int w = u - cs.ubase[s];
  c = w / ru;
  r = w - c * ru;
}

// A warp's units are u0 + warp + i * kWarps: one division to find the first,
// then each step moves kWarps units on, which crosses at most one chunk and
// one slot boundary because every chunk has ru >= kWarps units.
struct UnitCursor {
  int s, c, r;
};
__device__ __forceinline__ UnitCursor cursor_at(const CtaSched& cs, int ru, int u) {
  UnitCursor k;
  k.s = 0;
  locate(cs, ru, u, k.s, k.c, k.r);
  return k;
}
__device__ __forceinline__ void cursor_step(const CtaSched& cs, int ru, UnitCursor& k) {
  k.r += kWarps;
  if (k.r >= ru) {
    k.r -= ru;
    if (++k.c >= cs.nk[k.s]) {
      k.c = 0;
      ++k.s;
    }
  }
}

// ---------------------------------------------------------------------------
// Dot products over one input chunk
// ---------------------------------------------------------------------------
// Gate and up row chunks (nvc vectors each) against one token's staged input:
// vectors v0 .. v0+nvc-1 of a [F4][NV] staged array.
template <int BITS>
__device__ __forceinline__ void gu_dot_chunk(const char* st, int nvc, int cb, int cap, int sbo_g, int sbo_u,
                                             const float4* xs, int NV, int v0, const float2* sf, int lane,
                                             float& g_out, float& u_out) {
  const uint4* cg = reinterpret_cast<const uint4*>(st);
  const uint4* cu = reinterpret_cast<const uint4*>(st + cb);
  const uint32_t* sbg = reinterpret_cast<const uint32_t*>(st + 2 * cb + sbo_g);
  const uint32_t* sbu = reinterpret_cast<const uint32_t*>(st + 2 * cb + cap + sbo_u);
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(xs) + v0;
  float g = 0.f, u = 0.f;
  for (int v = lane; v < nvc; v += 32) {
    const uint4 wg = cg[v], wu = cu[v];
    const int grp = (BITS == 4) ? (v >> 1) : v;
    const uint32_t sbgw = sbg[grp], sbuw = sbu[grp];
    const float2 f = __ldg(sf + v0 + v);
    uint64_t ag = 0, au = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t a_ = (&wg.x)[t], b_ = (&wu.x)[t];
      if (BITS == 4) {
        const ulonglong2 xa = __ldg(xv + (2 * t) * NV + v), xb = __ldg(xv + (2 * t + 1) * NV + v);
        dot_word4(ag, a_, xa, xb);
        dot_word4(au, b_, xa, xb);
      } else {
        const ulonglong2 x0 = __ldg(xv + (4 * t) * NV + v), x1 = __ldg(xv + (4 * t + 1) * NV + v);
        const ulonglong2 x2 = __ldg(xv + (4 * t + 2) * NV + v), x3 = __ldg(xv + (4 * t + 3) * NV + v);
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

// kRC down-row chunks (nvc vectors each, rows cb bytes apart in the stage;
// scale/bias words of row j at sbw + j * sb_stride) against one staged
// activation (vectors v0 .. v0+nvc-1 of a [F4][NV] array).
template <int BITS>
__device__ __forceinline__ void down_dot_chunk(const char* st, int nvc, int cb, const uint32_t* sbw, int sb_stride,
                                               const float4* as, int NV, int v0, const float2* sfa, int lane,
                                               float (&y)[kRC]) {
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(as) + v0;
#pragma unroll
  for (int r = 0; r < kRC; ++r) y[r] = 0.f;
  for (int v = lane; v < nvc; v += 32) {
    uint4 w[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) w[r] = reinterpret_cast<const uint4*>(st + r * cb)[v];
    const float2 f = __ldg(sfa + v0 + v);
    const int grp = (BITS == 4) ? (v >> 1) : v;
    uint64_t ac[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) ac[r] = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (BITS == 4) {
        const ulonglong2 xa = __ldg(xv + (2 * t) * NV + v), xb = __ldg(xv + (2 * t + 1) * NV + v);
#pragma unroll
        for (int r = 0; r < kRC; ++r) dot_word4(ac[r], (&w[r].x)[t], xa, xb);
      } else {
        const ulonglong2 x0 = __ldg(xv + (4 * t) * NV + v), x1 = __ldg(xv + (4 * t + 1) * NV + v);
        const ulonglong2 x2 = __ldg(xv + (4 * t + 2) * NV + v), x3 = __ldg(xv + (4 * t + 3) * NV + v);
#pragma unroll
        for (int r = 0; r < kRC; ++r) dot_word2(ac[r], (&w[r].x)[t], x0, x1, x2, x3);
      }
    }
#pragma unroll
    for (int r = 0; r < kRC; ++r) {
      const uint32_t sbv = sbw[r * sb_stride + grp];
      const float2 d = unpk_f32(ac[r]);
      y[r] = fmaf(bf16_lo(sbv) * f.y, d.x + d.y, y[r]);
      y[r] = fmaf(bf16_hi(sbv), f.x, y[r]);
    }
  }
  // row (lane >> 3) & 3 on each lane: lanes 0, 8, 16, 24 hold rows 0..3
  y[0] = warp_sum4_split(y, lane);
}

// Two gate/up units (stages stA, stB: rows of the same slot and input chunk)
// against one token's staged input, each input load serving four rows.
// Results: unit A's g, u on lane 0, unit B's g, u on lane 16.
template <int BITS>
__device__ __forceinline__ void gu_dot_chunk2(const char* stA, const char* stB, int nvc, int cb, int cap, int sbo_gA,
                                              int sbo_uA, int sbo_gB, int sbo_uB, const float4* xs, int NV, int v0,
                                              const float2* sf, int lane, float& g_out, float& u_out) {
  const uint4* cgA = reinterpret_cast<const uint4*>(stA);
  const uint4* cuA = reinterpret_cast<const uint4*>(stA + cb);
  const uint4* cgB = reinterpret_cast<const uint4*>(stB);
  const uint4* cuB = reinterpret_cast<const uint4*>(stB + cb);
  const uint32_t* sgA = reinterpret_cast<const uint32_t*>(stA + 2 * cb + sbo_gA);
  const uint32_t* suA = reinterpret_cast<const uint32_t*>(stA + 2 * cb + cap + sbo_uA);
  const uint32_t* sgB = reinterpret_cast<const uint32_t*>(stB + 2 * cb + sbo_gB);
  const uint32_t* suB = reinterpret_cast<const uint32_t*>(stB + 2 * cb + cap + sbo_uB);
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(xs) + v0;
  float y[4] = {0.f, 0.f, 0.f, 0.f};  // gA, uA, gB, uB
  for (int v = lane; v < nvc; v += 32) {
    const uint4 w0 = cgA[v], w1 = cuA[v], w2 = cgB[v], w3 = cuB[v];
    const int grp = (BITS == 4) ? (v >> 1) : v;
    const uint32_t sb[4] = {sgA[grp], suA[grp], sgB[grp], suB[grp]};
    const float2 f = __ldg(sf + v0 + v);
    uint64_t ac[4] = {0, 0, 0, 0};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t c0 = (&w0.x)[t], c1 = (&w1.x)[t], c2 = (&w2.x)[t], c3 = (&w3.x)[t];
      if (BITS == 4) {
        const ulonglong2 xa = __ldg(xv + (2 * t) * NV + v), xb = __ldg(xv + (2 * t + 1) * NV + v);
        dot_word4(ac[0], c0, xa, xb);
        dot_word4(ac[1], c1, xa, xb);
        dot_word4(ac[2], c2, xa, xb);
        dot_word4(ac[3], c3, xa, xb);
      } else {
        const ulonglong2 x0 = __ldg(xv + (4 * t) * NV + v), x1 = __ldg(xv + (4 * t + 1) * NV + v);
        const ulonglong2 x2 = __ldg(xv + (4 * t + 2) * NV + v), x3 = __ldg(xv + (4 * t + 3) * NV + v);
        dot_word2(ac[0], c0, x0, x1, x2, x3);
        dot_word2(ac[1], c1, x0, x1, x2, x3);
        dot_word2(ac[2], c2, x0, x1, x2, x3);
        dot_word2(ac[3], c3, x0, x1, x2, x3);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float2 d = unpk_f32(ac[r]);
      y[r] = fmaf(bf16_lo(sb[r]) * f.y, d.x + d.y, y[r]);
      y[r] = fmaf(bf16_hi(sb[r]), f.x, y[r]);
    }
  }
  const float v = warp_sum4_split(y, lane);  // lanes 0, 8, 16, 24: gA, uA, gB, uB
  g_out = v;
  u_out = __shfl_down_sync(0xffffffffu, v, 8);
}

// Two down units (stA, stB: kRC rows each, same slot and input chunk) against
// one staged activation, each activation load serving 2 * kRC rows.  Results:
// lane 8r holds row r of A in yA and row r of B in yB.
template <int BITS>
__device__ __forceinline__ void down_dot_chunk2(const char* stA, const char* stB, int nvc, int cb,
                                                const uint32_t* sbwA, const uint32_t* sbwB, int sb_stride,
                                                const float4* as, int NV, int v0, const float2* sfa, int lane,
                                                float& yA, float& yB) {
  const ulonglong2* xv = reinterpret_cast<const ulonglong2*>(as) + v0;
  float ya[kRC], yb[kRC];
#pragma unroll
  for (int r = 0; r < kRC; ++r) ya[r] = yb[r] = 0.f;
  for (int v = lane; v < nvc; v += 32) {
    uint4 wa[kRC], wb[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) {
      wa[r] = reinterpret_cast<const uint4*>(stA + r * cb)[v];
      wb[r] = reinterpret_cast<const uint4*>(stB + r * cb)[v];
    }
    const float2 f = __ldg(sfa + v0 + v);
    const int grp = (BITS == 4) ? (v >> 1) : v;
    uint64_t aa[kRC], ab[kRC];
#pragma unroll
    for (int r = 0; r < kRC; ++r) aa[r] = ab[r] = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (BITS == 4) {
        const ulonglong2 xa = __ldg(xv + (2 * t) * NV + v), xb = __ldg(xv + (2 * t + 1) * NV + v);
#pragma unroll
        for (int r = 0; r < kRC; ++r) {
          dot_word4(aa[r], (&wa[r].x)[t], xa, xb);
          dot_word4(ab[r], (&wb[r].x)[t], xa, xb);
        }
      } else {
        const ulonglong2 x0 = __ldg(xv + (4 * t) * NV + v), x1 = __ldg(xv + (4 * t + 1) * NV + v);
        const ulonglong2 x2 = __ldg(xv + (4 * t + 2) * NV + v), x3 = __ldg(xv + (4 * t + 3) * NV + v);
#pragma unroll
        for (int r = 0; r < kRC; ++r) {
          dot_word2(aa[r], (&wa[r].x)[t], x0, x1, x2, x3);
          dot_word2(ab[r], (&wb[r].x)[t], x0, x1, x2, x3);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRC; ++r) {
      const uint32_t sa = sbwA[r * sb_stride + grp], sbv = sbwB[r * sb_stride + grp];
      const float2 da = unpk_f32(aa[r]), db = unpk_f32(ab[r]);
      ya[r] = fmaf(bf16_lo(sa) * f.y, da.x + da.y, ya[r]);
      ya[r] = fmaf(bf16_hi(sa), f.x, ya[r]);
      yb[r] = fmaf(bf16_lo(sbv) * f.y, db.x + db.y, yb[r]);
      yb[r] = fmaf(bf16_hi(sbv), f.x, yb[r]);
    }
  }
  yA = warp_sum4_split(ya, lane);
  yB = warp_sum4_split(yb, lane);
}

// ---------------------------------------------------------------------------
// gate/up
// ---------------------------------------------------------------------------
// Ring position of a warp's unit: stage index and the phase parity its
// mbarrier completes with; advanced one unit at a time (no divisions).
struct RingPos {
  int idx;
  uint32_t ph;
};
__device__ __forceinline__ void ring_next(RingPos& r, int n) {
  if (++r.idx == n) {
    r.idx = 0;
    r.ph ^= 1u;
  }
}

template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) grouped_gateup_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ SchedSmem ss;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nst = a.nst, stage_bytes = a.stage_bytes;
  char* my_ring = smem_raw + (size_t)warp * nst * stage_bytes;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem_raw + (size_t)kWarps * nst * stage_bytes) + warp * nst;
  if (lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  CtaSched cs;
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  cta_sched(a, 0, cs, ss);  // includes __syncthreads
  // this warp's units: cs.u0 + warp + i * kWarps
  const int n = cs.u1 - cs.u0 > warp ? (cs.u1 - cs.u0 - warp - 1) / kWarps + 1 : 0;
  const int H = a.H, I = a.I;
  const int sbr = sb_row_bytes(H), cap = sb_superset_cap(H);
  // Section offsets of both code widths; the up section's scale/bias words lie
  // a multiple of 16 bytes after the gate section's (code and scale/bias
  // sections are whole multiples of 16 bytes), so a row chunk's gate and up
  // scale/bias copies share their alignment and length.
  const long long gc_r = a.off_r[0], gsb_r = a.off_r[1], uc_r = a.off_r[2], usb_r = a.off_r[3];
  const long long gc_s = a.off_s[0], gsb_s = a.off_s[1], uc_s = a.off_s[2], usb_s = a.off_s[3];

  UnitCursor ki = cursor_at(cs, I, cs.u0 + warp);  // next unit to issue
  int ri = 0;                                       // its ring stage
  auto issue = [&]() {  // lane 0; units are issued in order
    const int s = ki.s, c = ki.c, row = ki.r;
    cursor_step(cs, I, ki);
    const int e = cs.expert[s];
    const bool routed = e >= 0;
    const char* blob = routed ? a.experts + (long long)e * a.expert_stride : a.shared;
    const int cl = cs.cl[s];
    const int cb = routed ? cl * BR / 8 : cl * BS / 8;
    const int rowb = routed ? H * BR / 8 : H * BS / 8;
    const long long code0 = (long long)row * rowb + c * cb;
    const long long gs0 = (routed ? gsb_r : gsb_s) + (long long)row * sbr + ((c * cl) >> 4);
    const long long ga = gs0 & ~15LL;
    const int len = (((int)gs0 & 15) + (cl >> 4) + 15) & ~15;
    char* stage = my_ring + ri * stage_bytes;
    uint64_t* bar = &my_bars[ri];
    if (++ri == nst) ri = 0;
    mbar_arrive_expect_tx(bar, 2 * cb + 2 * len);
    bulk_g2s(stage, blob + (routed ? gc_r : gc_s) + code0, cb, bar);
    bulk_g2s(stage + cb, blob + (routed ? uc_r : uc_s) + code0, cb, bar);
    bulk_g2s(stage + 2 * cb, blob + ga, len, bar);
    bulk_g2s(stage + 2 * cb + cap, blob + ga + (routed ? usb_r - gsb_r : usb_s - gsb_s), len, bar);
  };
  if (lane == 0)
    for (int i = 0; i < n && i < nst; ++i) issue();

  UnitCursor kc = cursor_at(cs, I, cs.u0 + warp);  // unit being computed
  RingPos rc{0, 0u};                                // its ring stage
  for (int i = 0; i < n;) {
    // Two consecutive units of the same slot and input chunk are computed in
    // one pass (each input load then serves four rows).
    UnitCursor kn = kc;
    cursor_step(cs, I, kn);
    const bool two = nst >= 2 && i + 1 < n && kn.s == kc.s && kn.c == kc.c;
    RingPos r2 = rc;
    ring_next(r2, nst);
    const char* stage = my_ring + rc.idx * stage_bytes;
    const char* stage2 = my_ring + r2.idx * stage_bytes;
    // A copy that did not arrive in time makes its unit's results NaN (the
    // decision is the whole warp's), which reaches every token using them.
    const bool ok1 = __all_sync(0xffffffffu, mbar_wait_bounded(&my_bars[rc.idx], rc.ph, a.timeout_ns));
    const bool ok2 = !two || __all_sync(0xffffffffu, mbar_wait_bounded(&my_bars[r2.idx], r2.ph, a.timeout_ns));
    if (!(ok1 && ok2) && lane == 0) set_status(kStatusCopyTimeout);
    const int s = kc.s, c = kc.c, row = kc.r, row2 = kn.r;
    const bool routed = cs.expert[s] >= 0;
    const int cl = cs.cl[s];
    const int sb_c = (int)(routed ? gsb_r : gsb_s) + ((c * cl) >> 4);
    const int sbo = (sb_c + row * sbr) & 15, sbo2 = (sb_c + row2 * sbr) & 15;
    for (int p = cs.pair0[s]; p < cs.pair0[s + 1]; ++p) {
      const int t = cs.ptok[p];
      float g, up;
      float2* dst = a.gu_part + ((long long)p * kMaxChunks + c) * I;
      if (routed || BR == BS) {
        constexpr int CPV = 128 / BR;
        const float4* xs = a.xs_r + (long long)t * (H / 4);
        const float2* sf = a.sf_r + (long long)t * (H / CPV);
        if (two)
          gu_dot_chunk2<BR>(stage, stage2, cl / CPV, cl * BR / 8, cap, sbo, sbo, sbo2, sbo2, xs, H / CPV,
                            c * (cl / CPV), sf, lane, g, up);
        else
          gu_dot_chunk<BR>(stage, cl / CPV, cl * BR / 8, cap, sbo, sbo, xs, H / CPV, c * (cl / CPV), sf, lane, g, up);
      } else {
        constexpr int CPV = 128 / BS;
        const float4* xs = a.xs_s + (long long)t * (H / 4);
        const float2* sf = a.sf_s + (long long)t * (H / CPV);
        if (two)
          gu_dot_chunk2<BS>(stage, stage2, cl / CPV, cl * BS / 8, cap, sbo, sbo, sbo2, sbo2, xs, H / CPV,
                            c * (cl / CPV), sf, lane, g, up);
        else
          gu_dot_chunk<BS>(stage, cl / CPV, cl * BS / 8, cap, sbo, sbo, xs, H / CPV, c * (cl / CPV), sf, lane, g, up);
      }
      if (lane == 0) dst[row] = ok1 ? make_float2(g, up) : make_float2(quiet_nan(), quiet_nan());
      if (two && lane == 16) dst[row2] = ok2 ? make_float2(g, up) : make_float2(quiet_nan(), quiet_nan());
    }
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      if (i + nst < n) issue();
      if (two && i + 1 + nst < n) issue();
    }
    i += two ? 2 : 1;
    kc = kn;
    rc = r2;
    if (two) {
      cursor_step(cs, I, kc);
      ring_next(rc, nst);
    }
  }
}

// ---------------------------------------------------------------------------
// stage: act = silu(g) * u from the chunk partials, staged for the down
// projection (one CTA per pair)
// ---------------------------------------------------------------------------
constexpr int kStageThreads = 256;

template <int BR, int BS>
__global__ void __launch_bounds__(kStageThreads) grouped_stage_act_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(16) float act[];  // [I]
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  const int p = blockIdx.x;
  if (p >= a.tb.meta[1]) return;
  const int nk = a.tb.pair_nk[p] & 0xFF;
  const bool routed = p < a.T * a.K;  // routed pairs come first
  const float2* part = a.gu_part + (long long)p * kMaxChunks * a.I;
  for (int r = threadIdx.x; r < a.I; r += kStageThreads) {
    float g = 0.f, u = 0.f;
    for (int c = 0; c < nk; ++c) {
      const float2 v = __ldcg(part + (long long)c * a.I + r);
      g += v.x;
      u += v.y;
    }
    act[r] = g * sigmoidf_(g) * u;
  }
  __syncthreads();
  float4* as = a.as + (long long)p * (a.I / 4);
  float2* sf = a.sfa + (long long)p * (a.I / 32);
  if (routed || BR == BS)
    stage_inputs<BR, false>(act, a.I, as, sf, threadIdx.x, kStageThreads);
  else
    stage_inputs<BS, false>(act, a.I, as, sf, threadIdx.x, kStageThreads);
}

// ---------------------------------------------------------------------------
// down
// ---------------------------------------------------------------------------
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) grouped_down_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ SchedSmem ss;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nst = a.nst_c, stage_bytes = a.c_stage_bytes;
  char* my_ring = smem_raw + (size_t)warp * nst * stage_bytes;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem_raw + (size_t)kWarps * nst * stage_bytes) + warp * nst;
  if (lane == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  const int H = a.H, I = a.I, nq = H / kRC;
  CtaSched cs;
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  cta_sched(a, 1, cs, ss);
  const int n = cs.u1 - cs.u0 > warp ? (cs.u1 - cs.u0 - warp - 1) / kWarps + 1 : 0;
  const int sbr = sb_row_bytes(I);  // bytes of one row's scale/bias words
  const long long dc_r = a.off_r[4], dsb_r = a.off_r[5], dc_s = a.off_s[4], dsb_s = a.off_s[5];

  UnitCursor ki = cursor_at(cs, nq, cs.u0 + warp);  // next unit to issue
  int ri = 0;                                        // its ring stage
  auto issue = [&]() {  // lane 0; units are issued in order
    const int s = ki.s, c = ki.c, q = ki.r;
    cursor_step(cs, nq, ki);
    const int e = cs.expert[s];
    const bool routed = e >= 0;
    const char* blob = routed ? a.experts + (long long)e * a.expert_stride : a.shared;
    const int cl = cs.cl[s];
    const int cb = routed ? cl * BR / 8 : cl * BS / 8;
    const int rowb = routed ? I * BR / 8 : I * BS / 8;
    const int r0 = q * kRC;
    char* stage = my_ring + ri * stage_bytes;
    uint64_t* bar = &my_bars[ri];
    if (++ri == nst) ri = 0;
    // kRC code row chunks, then one copy covering the rows' scale/bias chunks
    const long long sb0 = (routed ? dsb_r : dsb_s) + (long long)r0 * sbr + ((c * cl) >> 4);
    const long long sba = sb0 & ~15LL;
    const int sblen = (((int)sb0 & 15) + (kRC - 1) * sbr + (cl >> 4) + 15) & ~15;
    mbar_arrive_expect_tx(bar, kRC * cb + sblen);
    const char* codes = blob + (routed ? dc_r : dc_s) + (long long)r0 * rowb + c * cb;
    if (cb == rowb) {
      bulk_g2s(stage, codes, kRC * cb, bar);
    } else {
#pragma unroll
      for (int j = 0; j < kRC; ++j) bulk_g2s(stage + j * cb, codes + j * rowb, cb, bar);
    }
    bulk_g2s(stage + kRC * cb, blob + sba, sblen, bar);
  };
  if (lane == 0)
    for (int i = 0; i < n && i < nst; ++i) issue();

  UnitCursor kc = cursor_at(cs, nq, cs.u0 + warp);  // unit being computed
  RingPos rc{0, 0u};                                 // its ring stage
  for (int i = 0; i < n;) {
    // Two consecutive units of the same slot and input chunk are computed in
    // one pass (each activation load then serves 2 * kRC rows).
    UnitCursor kn = kc;
    cursor_step(cs, nq, kn);
    const bool two = nst >= 2 && i + 1 < n && kn.s == kc.s && kn.c == kc.c;
    RingPos r2 = rc;
    ring_next(r2, nst);
    const char* stage = my_ring + rc.idx * stage_bytes;
    const char* stage2 = my_ring + r2.idx * stage_bytes;
    // A copy that did not arrive in time makes its unit's results NaN (the
    // decision is the whole warp's), which reaches every token using them.
    const bool ok1 = __all_sync(0xffffffffu, mbar_wait_bounded(&my_bars[rc.idx], rc.ph, a.timeout_ns));
    const bool ok2 = !two || __all_sync(0xffffffffu, mbar_wait_bounded(&my_bars[r2.idx], r2.ph, a.timeout_ns));
    if (!(ok1 && ok2) && lane == 0) set_status(kStatusCopyTimeout);
    const int s = kc.s, c = kc.c, q = kc.r, q2 = kn.r;
    const bool routed = cs.expert[s] >= 0;
    const int cl = cs.cl[s];
    const int sb_c = (int)(routed ? dsb_r : dsb_s) + ((c * cl) >> 4);
    const int cb = routed ? cl * BR / 8 : cl * BS / 8;
    const uint32_t* sbw = reinterpret_cast<const uint32_t*>(stage + kRC * cb + ((sb_c + q * kRC * sbr) & 15));
    const uint32_t* sbw2 = reinterpret_cast<const uint32_t*>(stage2 + kRC * cb + ((sb_c + q2 * kRC * sbr) & 15));
    for (int p = cs.pair0[s]; p < cs.pair0[s + 1]; ++p) {
      float y[kRC], y2 = 0.f;
      const float4* as = a.as + (long long)p * (I / 4);
      const float2* sf = a.sfa + (long long)p * (I / 32);
      if (routed || BR == BS) {
        constexpr int CPV = 128 / BR;
        if (two)
          down_dot_chunk2<BR>(stage, stage2, cl / CPV, cb, sbw, sbw2, sbr / 4, as, I / CPV, c * (cl / CPV), sf, lane,
                              y[0], y2);
        else
          down_dot_chunk<BR>(stage, cl / CPV, cb, sbw, sbr / 4, as, I / CPV, c * (cl / CPV), sf, lane, y);
      } else {
        constexpr int CPV = 128 / BS;
        if (two)
          down_dot_chunk2<BS>(stage, stage2, cl / CPV, cb, sbw, sbw2, sbr / 4, as, I / CPV, c * (cl / CPV), sf, lane,
                              y[0], y2);
        else
          down_dot_chunk<BS>(stage, cl / CPV, cb, sbw, sbr / 4, as, I / CPV, c * (cl / CPV), sf, lane, y);
      }
      float* dst = a.y_part + ((long long)p * kMaxChunks + c) * H + (lane >> 3);
      if ((lane & 7) == 0) {
        dst[q * kRC] = ok1 ? y[0] : quiet_nan();
        if (two) dst[q2 * kRC] = ok2 ? y2 : quiet_nan();
      }
    }
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      if (i + nst < n) issue();
      if (two && i + 1 + nst < n) issue();
    }
    i += two ? 2 : 1;
    kc = kn;
    rc = r2;
    if (two) {
      cursor_step(cs, nq, kc);
      ring_next(rc, nst);
    }
  }
}

// ---------------------------------------------------------------------------
// combine: out[t] = residual[t] + sum_k w[t][k] y[pair(t,k)] + sg[t] y[shared pair of t]
// One CTA per (token, 1024 outputs); each thread takes 4 consecutive outputs.
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) grouped_combine_kernel(const __grid_constant__ GroupArgs a) {
  grid_dep_wait();  // (programmatic dependent launch: the previous kernel's writes are visible from here)
  grid_dep_launch_dependents();
  __shared__ int s_pair[kMaxTopK + 1], s_nk[kMaxTopK + 1];
  __shared__ float s_w[kMaxTopK + 1];
  const int t = blockIdx.y, K = a.K;
  if (threadIdx.x <= K) {
    const int p = a.tb.tok_pair[t * (K + 1) + threadIdx.x];
    s_pair[threadIdx.x] = p;
    s_nk[threadIdx.x] = p >= 0 ? (__ldcg(a.tb.pair_nk + p) >> 8) & 0xFF : 0;
    s_w[threadIdx.x] = threadIdx.x < K ? a.tb.tok_w[t * K + threadIdx.x] : a.tb.tok_sg[t];
  }
  __syncthreads();
  const int h = (blockIdx.x * kCombineThreads + threadIdx.x) * 4;
  if (h >= a.H) return;
  const long long q = (long long)t * a.H + h;
  float4 v = a.residual ? __ldg(reinterpret_cast<const float4*>(a.residual + q)) : make_float4(0.f, 0.f, 0.f, 0.f);
  auto add = [&](float w, float4 y) {
    v.x = fmaf(w, y.x, v.x);
    v.y = fmaf(w, y.y, v.y);
    v.z = fmaf(w, y.z, v.z);
    v.w = fmaf(w, y.w, v.w);
  };
  for (int k = 0; k <= K; ++k) {  // routed pairs in k order, then the shared pair
    const int p = s_pair[k];
    if (p < 0) continue;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < s_nk[k]; ++c) {
      const float4 u = __ldcg(reinterpret_cast<const float4*>(a.y_part + ((long long)p * kMaxChunks + c) * a.H + h));
      y.x += u.x;
      y.y += u.y;
      y.z += u.z;
      y.w += u.w;
    }
    add(s_w[k], y);
  }
  if (a.shared_tc) {
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int ks = 0; ks < a.I / 512; ++ks) {
      const float4 u = __ldcg(reinterpret_cast<const float4*>(a.sh_y + ((long long)ks * kMaxTokens + t) * a.H + h));
      y.x += u.x;
      y.y += u.y;
      y.z += u.z;
      y.w += u.w;
    }
    add(s_w[K], y);
  }
  *reinterpret_cast<float4*>(a.out + q) = v;
}

}  // namespace fmoe
