// Constants and helpers shared by the layer decode kernels: the CTA shape,
// the limits of a layer, the byte sizes of a row's sections, and the top-K
// selection of the router logits (descending logit, lower expert index first
// on exact ties; "Flash-MoE: Ausführen eines 397B-Parameter-Qwen-Modells ...",
// section "Pipeline-Leistung": softmax and top-K routing of each token).
#pragma once
#include "dequant.cuh"

namespace fmoe {

constexpr int kWarps = 16;        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRC = 4;            // down rows per grouped down item (the split row reduction assumes 4)
constexpr int kMaxTopK = 8;
constexpr int kMaxSlots = kMaxTopK + 1;
constexpr int kMaxExperts = 1024; // top-K is one warp with 32 logits per lane
constexpr int kTagWords = kMaxExperts + 1;  // tagged-logit words of a workspace (routers and the gate)
constexpr int kMaxActWords = 10240;         // tagged activations of a workspace: (K + 1) * I at most
constexpr int kMaxNstC = 8;       // most down-item stages a warp of the grouped kernels keeps in flight

// Bytes of a row's sections.
__host__ __device__ __forceinline__ int codes_row_bytes(int n_in, int bits) { return n_in * bits / 8; }
__host__ __device__ __forceinline__ int sb_row_bytes(int n_in) { return n_in / 16; }
// Capacity reserved for one row's (s, b) words copied with 16-byte-aligned
// bulk copies (the copy may start up to 12 bytes before the row and end up to
// 12 after it).
__host__ __device__ __forceinline__ int sb_superset_cap(int n_in) { return ((n_in / 16 + 15) & ~15) + 16; }

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

}  // namespace fmoe
