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
//   router   logits[t][e] for every token, each router row read once
//            (router_logits_kernel);
//   prep     CTA 0: top-K per token (one warp each), then the grouping: the
//            (token, k) pairs sorted by (expert, token), one slot per distinct
//            expert in ascending expert order, the shared expert last with all
//            T tokens; CTAs 1..T: each token's input staged in the decode
//            layouts (stage_inputs) into the workspace;
//   gate/up  every (slot, row) unit reads the gate and up rows once and
//            produces silu(g) * u for each token of the slot;
//   stage    each pair's activation vector staged for the down projection;
//   down     each CTA owns a block of output rows; for every slot it reads the
//            down rows of its block once and applies them to each token of the
//            slot; then the combine, per token in fixed k order.
// No float atomics anywhere: results are bitwise reproducible and equal for a
// token whatever else is in the batch, up to the order of the combine.
#pragma once
#include "route_quant_kernels.cuh"

namespace fmoe {

constexpr int kMaxTokens = 16;
constexpr int kMaxPairs = kMaxTokens * kMaxTopK + kMaxTokens;
constexpr int kUnitCostBase = 2;  // gate/up unit cost = kUnitCostBase + tokens of its slot

// Grouping tables (workspace).
struct GroupTables {
  int* meta;         // [0] slots, [1] pairs (routed pairs, then one shared pair per token)
  int* slot_expert;  // [slots] expert id, -1 = the shared expert
  int* slot_pair0;   // [slots + 1] first pair of each slot
  int* pair_token;   // [pairs]
  int* tok_pair;     // [T][K + 1] pair of (t, k); column K: the shared pair (-1 if none)
  float* tok_w;      // [T][K]
  float* tok_sg;     // [T]
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
  float4* xs_r;  // [T][H/4] staged inputs for the routed code width
  float2* sf_r;  // [T][H*BR/128]
  float4* xs_s;  // same for the shared expert's width (aliases xs_r when equal)
  float2* sf_s;
  float* act;    // [pairs][I] silu(g) * u
  float4* as;    // [pairs][I/4] staged activations
  float2* sfa;   // [pairs][I/32]
  int* idx_out;  // optional [T][K]
  float* w_out;  // optional [T][K]
  int H, I, E, K, T, bits_r, bits_s;
  int has_sgate;
  int nst, stage_bytes;      // gate/up ring
  int nst_c, c_stage_bytes;  // down ring
  int ys_stride;             // rows per CTA (max) of the down results
  long long off_r[6], off_s[6];
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------------------
// prep: top-K per token, grouping, input staging
// ---------------------------------------------------------------------------
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads) grouped_prep_kernel(const __grid_constant__ GroupArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (blockIdx.x > 0) {
    const int t = blockIdx.x - 1;
    const float* x = a.x + (long long)t * a.H;
    stage_inputs<BR, true>(x, a.H, a.xs_r + (long long)t * (a.H / 4), a.sf_r + (long long)t * (a.H * BR / 128), tid,
                           kThreads);
    if (a.shared != nullptr && a.xs_s != a.xs_r)
      stage_inputs<BS, true>(x, a.H, a.xs_s + (long long)t * (a.H / 4), a.sf_s + (long long)t * (a.H * BS / 128),
                             tid, kThreads);
    return;
  }
  __shared__ int s_idx[kMaxTokens * kMaxTopK];
  __shared__ float s_w[kMaxTokens * kMaxTopK];
  __shared__ int s_rank[kMaxTokens * kMaxTopK];
  __shared__ int s_se[kMaxTokens * kMaxTopK];  // expert of sorted pair p
  __shared__ int s_start[kMaxTokens * kMaxTopK];
  const int T = a.T, K = a.K, NP = T * K;
  if (warp < T) {
    const float* lt = a.logits + (long long)warp * (a.E + 1);
    warp_topk<false>(lt, a.E, K, lane, s_idx + warp * K, s_w + warp * K);
    if (lane == 0) a.tb.tok_sg[warp] = a.has_sgate ? sigmoidf_(__ldcg(lt + a.E)) : 1.0f;
  }
  __syncthreads();
  // Rank of pair j = t*K + k in (expert, j) order, i.e. (expert, token) order
  // since a token's top-K experts are distinct; ties on j keep the ranks a
  // permutation whatever the indices are.
  if (tid < NP) {
    int e = s_idx[tid];
    if (e < 0 || e >= a.E) e = 0;  // (cannot happen: top-K indices lie in [0, E))
    s_idx[tid] = e;
  }
  __syncthreads();
  if (tid < NP) {
    const int e = s_idx[tid], t = tid / K;
    int rank = 0;
    for (int j = 0; j < NP; ++j) {
      const int e2 = s_idx[j];
      rank += (e2 < e) || (e2 == e && j < tid);
    }
    s_rank[tid] = rank;
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
  if (tid < NP && s_start[tid]) {
    int slot = -1;
    for (int j = 0; j <= tid; ++j) slot += s_start[j];
    a.tb.slot_expert[slot] = s_se[tid];
    a.tb.slot_pair0[slot] = tid;
  }
  if (tid < T) {
    a.tb.tok_pair[tid * (K + 1) + K] = a.shared != nullptr ? NP + tid : -1;
    if (a.shared != nullptr) a.tb.pair_token[NP + tid] = tid;
  }
  if (tid == 0) {
    int nr = 0;
    for (int j = 0; j < NP; ++j) nr += s_start[j];
    int ns = nr, np = NP;
    if (a.shared != nullptr) {
      a.tb.slot_expert[nr] = -1;
      a.tb.slot_pair0[nr] = NP;
      ns = nr + 1;
      np = NP + T;
    }
    a.tb.slot_pair0[ns] = np;
    a.tb.meta[0] = ns;
    a.tb.meta[1] = np;
  }
}

// ---------------------------------------------------------------------------
// gate/up
// ---------------------------------------------------------------------------

// First unit (flattened slot * I + row) whose cost interval starts at or after
// `target`; slot s's units each cost kUnitCostBase + n_s.
__device__ __forceinline__ int first_unit(long long target, const int* pair0, int ns, int I) {
  long long cc = 0;
  for (int s = 0; s < ns; ++s) {
    const long long c = kUnitCostBase + (pair0[s + 1] - pair0[s]);
    const long long span = c * I;
    if (target < cc + span) return s * I + (int)((target - cc + c - 1) / c);
    cc += span;
  }
  return ns * I;
}

template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) grouped_gateup_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ int s_pair0[kMaxPairs + 2];
  __shared__ int s_expert[kMaxPairs + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = a.tb.meta[0];
  for (int s = tid; s <= ns; s += kThreads) {
    s_pair0[s] = a.tb.slot_pair0[s];
    if (s < ns) s_expert[s] = a.tb.slot_expert[s];
  }
  char* my_ring = smem_raw + (size_t)warp * a.nst * a.stage_bytes;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem_raw + (size_t)kWarps * a.nst * a.stage_bytes) + warp * a.nst;
  if (lane == 0) {
    for (int s = 0; s < a.nst; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  __syncthreads();

  // This warp's units: an equal share of the total cost, contiguous.
  long long total = 0;
  for (int s = 0; s < ns; ++s) total += (long long)(kUnitCostBase + s_pair0[s + 1] - s_pair0[s]) * a.I;
  const long long GW = (long long)gridDim.x * kWarps, gw = (long long)blockIdx.x * kWarps + warp;
  const int u0 = first_unit(total * gw / GW, s_pair0, ns, a.I);
  const int u1 = first_unit(total * (gw + 1) / GW, s_pair0, ns, a.I);
  const int n = u1 - u0;

  const int sbr = sb_row_bytes(a.H), cap = sb_superset_cap(a.H);
  auto issue = [&](int i) {  // lane 0
    const int u = u0 + i, s = u / a.I, row = u - s * a.I;
    const int e = s_expert[s];
    const char* blob = e >= 0 ? a.experts + (long long)e * a.expert_stride : a.shared;
    const long long* o = e >= 0 ? a.off_r : a.off_s;
    const int cb = codes_row_bytes(a.H, e >= 0 ? BR : BS);
    const long long gs0 = o[1] + (long long)row * sbr, us0 = o[3] + (long long)row * sbr;
    const long long ga = gs0 & ~15LL, ua = us0 & ~15LL;
    const int glen = (int)(((gs0 + sbr + 15) & ~15LL) - ga);
    const int ulen = (int)(((us0 + sbr + 15) & ~15LL) - ua);
    char* stage = my_ring + (size_t)(i % a.nst) * a.stage_bytes;
    uint64_t* bar = &my_bars[i % a.nst];
    mbar_arrive_expect_tx(bar, 2 * cb + glen + ulen);
    bulk_g2s(stage, blob + o[0] + (long long)row * cb, cb, bar);
    bulk_g2s(stage + cb, blob + o[2] + (long long)row * cb, cb, bar);
    bulk_g2s(stage + 2 * cb, blob + ga, glen, bar);
    bulk_g2s(stage + 2 * cb + cap, blob + ua, ulen, bar);
  };
  if (lane == 0)
    for (int i = 0; i < n && i < a.nst; ++i) issue(i);

  for (int i = 0; i < n; ++i) {
    const char* stage = my_ring + (size_t)(i % a.nst) * a.stage_bytes;
    if (!mbar_wait_bounded(&my_bars[i % a.nst], (i / a.nst) & 1, a.timeout_ns) && lane == 0)
      set_status(kStatusCopyTimeout);
    const int u = u0 + i, s = u / a.I, row = u - s * a.I;
    const bool routed = s_expert[s] >= 0;
    const BlobOff o = blob_offsets(a.H, a.I, routed ? BR : BS);
    const int sbo_g = (int)((o.gsb + (long long)row * sbr) & 15);
    const int sbo_u = (int)((o.usb + (long long)row * sbr) & 15);
    for (int p = s_pair0[s]; p < s_pair0[s + 1]; ++p) {
      const int t = a.tb.pair_token[p];
      float g, up;
      if (routed || BR == BS)
        pair_dot_src<BR, true>(stage, a.H, sbo_g, sbo_u, a.xs_r + (long long)t * (a.H / 4),
                               a.sf_r + (long long)t * (a.H * BR / 128), lane, g, up);
      else
        pair_dot_src<BS, true>(stage, a.H, sbo_g, sbo_u, a.xs_s + (long long)t * (a.H / 4),
                               a.sf_s + (long long)t * (a.H * BS / 128), lane, g, up);
      if (lane == 0) a.act[(long long)p * a.I + row] = g * sigmoidf_(g) * up;
    }
    __syncwarp();
    if (lane == 0 && i + a.nst < n) {
      fence_proxy_async_smem();
      issue(i + a.nst);
    }
  }
}

// ---------------------------------------------------------------------------
// stage the activations (one CTA per pair)
// ---------------------------------------------------------------------------
template <int BR, int BS>
__global__ void __launch_bounds__(256) grouped_stage_act_kernel(const __grid_constant__ GroupArgs a) {
  const int p = blockIdx.x;
  if (p >= a.tb.meta[1]) return;
  const bool routed = p < a.T * a.K;
  const float* src = a.act + (long long)p * a.I;
  float4* as = a.as + (long long)p * (a.I / 4);
  float2* sf = a.sfa + (long long)p * (a.I / 32);
  if (routed || BR == BS)
    stage_inputs<BR, true>(src, a.I, as, sf, threadIdx.x, blockDim.x);
  else
    stage_inputs<BS, true>(src, a.I, as, sf, threadIdx.x, blockDim.x);
}

// ---------------------------------------------------------------------------
// down + combine
// ---------------------------------------------------------------------------
template <int BR, int BS>
__global__ void __launch_bounds__(kThreads, 1) grouped_down_kernel(const __grid_constant__ GroupArgs a) {
  extern __shared__ __align__(128) char smem_raw[];
  __shared__ int s_pair0[kMaxPairs + 2];
  __shared__ int s_expert[kMaxPairs + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int ns = a.tb.meta[0];
  for (int s = tid; s <= ns; s += kThreads) {
    s_pair0[s] = a.tb.slot_pair0[s];
    if (s < ns) s_expert[s] = a.tb.slot_expert[s];
  }
  char* my_ring = smem_raw + (size_t)warp * a.nst_c * a.c_stage_bytes;
  size_t off = (size_t)kWarps * a.nst_c * a.c_stage_bytes;
  float* ys = reinterpret_cast<float*>(smem_raw + off);  // [pairs][ys_stride]
  off += (size_t)kMaxPairs * a.ys_stride * 4;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem_raw + off) + warp * a.nst_c;
  if (lane == 0) {
    for (int s = 0; s < a.nst_c; ++s) mbar_init(&my_bars[s], 1);
    fence_proxy_async_smem();
  }
  __syncthreads();

  const int nq_all = a.H / kRC;
  const int q0 = (int)((long long)blockIdx.x * nq_all / G);
  const int nq = (int)((long long)(blockIdx.x + 1) * nq_all / G) - q0;
  const int n_items = ns * nq;
  const int n = n_items > warp ? (n_items - warp - 1) / kWarps + 1 : 0;  // items j = warp + i * kWarps
  const int sbr = sb_row_bytes(a.I);

  auto issue = [&](int i) {  // lane 0
    const int j = warp + i * kWarps, s = j / nq, r0 = (q0 + j - s * nq) * kRC;
    const int e = s_expert[s];
    const char* blob = e >= 0 ? a.experts + (long long)e * a.expert_stride : a.shared;
    const long long* o = e >= 0 ? a.off_r : a.off_s;
    const int cb = codes_row_bytes(a.I, e >= 0 ? BR : BS);
    char* stage = my_ring + (size_t)(i % a.nst_c) * a.c_stage_bytes;
    uint64_t* bar = &my_bars[i % a.nst_c];
    mbar_arrive_expect_tx(bar, kRC * (cb + sbr));
    bulk_g2s(stage, blob + o[4] + (long long)r0 * cb, kRC * cb, bar);
    bulk_g2s(stage + kRC * cb, blob + o[5] + (long long)r0 * sbr, kRC * sbr, bar);
  };
  if (lane == 0)
    for (int i = 0; i < n && i < a.nst_c; ++i) issue(i);

  for (int i = 0; i < n; ++i) {
    const char* stage = my_ring + (size_t)(i % a.nst_c) * a.c_stage_bytes;
    if (!mbar_wait_bounded(&my_bars[i % a.nst_c], (i / a.nst_c) & 1, a.timeout_ns) && lane == 0)
      set_status(kStatusCopyTimeout);
    const int j = warp + i * kWarps, s = j / nq, rl = (j - s * nq) * kRC;
    const bool routed = s_expert[s] >= 0;
    for (int p = s_pair0[s]; p < s_pair0[s + 1]; ++p) {
      float y[kRC];
      const float4* as = a.as + (long long)p * (a.I / 4);
      const float2* sf = a.sfa + (long long)p * (a.I / 32);
      if (routed || BR == BS)
        down_rows_src<BR, true>(stage, a.I, as, a.I * BR / 128, 0, sf, lane, y);
      else
        down_rows_src<BS, true>(stage, a.I, as, a.I * BS / 128, 0, sf, lane, y);
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < kRC; ++r) ys[p * a.ys_stride + rl + r] = y[r];
      }
    }
    __syncwarp();
    if (lane == 0 && i + a.nst_c < n) {
      fence_proxy_async_smem();
      issue(i + a.nst_c);
    }
  }
  __syncthreads();

  // out[t] = residual[t] + sum_k w[t][k] y[pair(t,k)] + sg[t] y[shared pair of t], fixed order
  const int rows = nq * kRC, K = a.K;
  for (int q = tid; q < a.T * rows; q += kThreads) {
    const int t = q / rows, rl = q - t * rows, h = q0 * kRC + rl;
    float v = a.residual ? __ldg(a.residual + (long long)t * a.H + h) : 0.f;
    const int* tp = a.tb.tok_pair + t * (K + 1);
    for (int k = 0; k < K; ++k) v = fmaf(a.tb.tok_w[t * K + k], ys[tp[k] * a.ys_stride + rl], v);
    if (tp[K] >= 0) v = fmaf(a.tb.tok_sg[t], ys[tp[K] * a.ys_stride + rl], v);
    a.out[(long long)t * a.H + h] = v;
  }
}

}  // namespace fmoe
