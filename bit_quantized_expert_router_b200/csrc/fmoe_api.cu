// Host side of libfmoe.so: argument validation, shared-memory planning and
// launches.  The C ABI is declared (and documented) in include/fmoe.h.
#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/fmoe.h"
#include "deltanet.cuh"
#include "expert_cache.h"
#include "shared_tc.cuh"

using namespace fmoe;

namespace {

constexpr unsigned long long kTimeoutNs = 2000000000ull;  // default bound on every device-side wait: 2 s
constexpr unsigned long long kMinWaitNs = 1000000ull;      // 1 ms
constexpr unsigned long long kMaxWaitNs = 60000000000ull;  // 60 s
std::atomic<unsigned long long> g_wait_limit_ns{kTimeoutNs};
std::atomic<int> g_dependent_launch{1};
constexpr size_t kCounterBytes = 256;
// Every workspace starts with the counters, then the single-token decode's
// tagged router logits and tagged activations (each sized for the largest
// layer, so that no other use of a workspace, whatever its layer's shape,
// ever writes these bytes).
constexpr size_t kTagBytes = (kTagWords * 8 + 255) / 256 * 256;
constexpr size_t kActTagBytes = (kActWords * 8 + 255) / 256 * 256;
constexpr size_t kHeaderBytes = kCounterBytes + kTagBytes + kActTagBytes;
constexpr int kMaxNst = 4;

struct DevInfo {
  int sms = 0;
  int max_smem = 0;     // opt-in dynamic shared memory available to the layer kernel
  int optin = 0;        // opt-in shared memory per block
  bool layer_attr_set[4] = {false, false, false, false};
  int layer_occupancy[4] = {-1, -1, -1, -1};  // resident CTAs per SM at pl.smem (-1: not asked yet)
  bool grouped_attr_set[4] = {false, false, false, false};
  int grouped_max_smem = 0;  // dynamic shared memory left by the grouped kernels' static arrays
};

using LayerFn = void (*)(LayerArgs);
// The instantiation for (routed bits, shared bits), and its index 0..3.
LayerFn layer_fn(int br, int bs) {
  if (br == 4) return bs == 4 ? layer_kernel<4, 4> : layer_kernel<4, 2>;
  return bs == 4 ? layer_kernel<2, 4> : layer_kernel<2, 2>;
}
int layer_fn_index(int br, int bs) { return (br == 4 ? 0 : 2) + (bs == 4 ? 0 : 1); }
DevInfo g_dev[64];
std::mutex g_mu;
thread_local int g_last_cuda_error = 0;

// Record a failed CUDA call for fmoe_last_cuda_error() and map it to FMOE_ECUDA.
int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return FMOE_ECUDA;
}

int dev_info(int* dev_out, DevInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FMOE_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (d.sms == 0) {
    cudaError_t e;
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    int optin = 0;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return cuda_fail(e);
    int static_smem = 0;
    for (int br : {4, 2})
      for (int bs : {4, 2}) {
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, layer_fn(br, bs))) != cudaSuccess) return cuda_fail(e);
        static_smem = std::max(static_smem, (int)fa.sharedSizeBytes);
      }
    d.max_smem = optin - static_smem;
    d.optin = optin;
    int gstatic = 0;
    for (const void* f : {(const void*)grouped_gateup_kernel<4, 4>, (const void*)grouped_down_kernel<4, 4>}) {
      cudaFuncAttributes fa;
      if ((e = cudaFuncGetAttributes(&fa, f)) != cudaSuccess) return cuda_fail(e);
      gstatic = std::max(gstatic, (int)fa.sharedSizeBytes);
    }
    d.grouped_max_smem = optin - gstatic;
  }
  *dev_out = dev;
  *info = &d;
  return FMOE_OK;
}

// The stream must belong to the current device.  The check is skipped while
// the stream is being captured into a CUDA graph (a device query there would
// invalidate the capture); the capture's own launches are checked on replay.
int check_stream(fmoe_stream_t s, int dev) {
  if (s == nullptr) return FMOE_OK;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(s);
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(cs, &st) != cudaSuccess) return FMOE_EINVAL;
  if (st != cudaStreamCaptureStatusNone) return FMOE_OK;
  int sdev = -1;
  if (cudaStreamGetDevice(cs, &sdev) != cudaSuccess) return FMOE_EINVAL;
  return sdev == dev ? FMOE_OK : FMOE_EINVAL;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool shape_ok(int h, int i) {
  return h > 0 && i > 0 && h % 64 == 0 && i % 64 == 0 && h <= FMOE_MAX_HIDDEN && i <= 8192;
}
bool bits_ok(int b) { return b == 2 || b == 4; }
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory plan of the layer kernel (see carve_smem in layer_kernel.cuh).
struct Plan {
  int nst, stage_bytes, nst_c, c_stage_bytes, xs4_off, xs2_off, xu_off, vec_floats, sf_floats, ys_stride;
  size_t smem;
};

bool plan_layer(int H, int I, int K, bool has_shared, int bits_r, int bits_s, int G, int n_router, int max_smem,
                Plan* p) {
  const int n_slots = K + (has_shared ? 1 : 0);
  bool use4 = false, use2 = false;
  int stage = 0, cstage = 0;
  auto use_bits = [&](int b) {
    if (b == 4) use4 = true; else use2 = true;
    const int cb = H * b / 8;
    const int cap = ((H / 16 + 15) & ~15) + 16;
    stage = std::max(stage, 2 * cb + 2 * cap);
    cstage = std::max(cstage, kRC * (I * b / 8 + I / 16));
  };
  if (K > 0) use_bits(bits_r);
  if (has_shared) use_bits(bits_s);
  cstage = (int)round_up(cstage, 128);
  stage = (int)round_up(std::max(stage, cstage), 128);
  int off = 0;
  p->xu_off = off;  // x, copied in by one bulk copy
  off += H;
  p->xs4_off = -1;
  p->xs2_off = -1;
  if (use4) { p->xs4_off = off; off += H; }
  if (use2) { p->xs2_off = off; off += H; }
  p->vec_floats = (int)round_up((size_t)std::max(off, n_slots * I), 32);
  p->sf_floats = (int)round_up((size_t)std::max((use4 ? H / 32 : 0) + (use2 ? H / 64 : 0), n_slots * I / 32), 16);
  const int nq = H / kRC;
  p->ys_stride = kRC * ((nq + G - 1) / G);
  p->stage_bytes = stage;
  const size_t fixed = (size_t)p->vec_floats * 4 + (size_t)p->sf_floats * 8 +
                       round_up((size_t)n_slots * p->ys_stride * 4, 16);
  p->c_stage_bytes = cstage;
  for (int nst = kMaxNst; nst >= 1; --nst) {
    const size_t total = (size_t)kWarps * nst * stage + fixed + (size_t)kWarps * (nst + kMaxNstC) * 8;
    if (total <= (size_t)max_smem) {
      p->nst = nst;
      p->nst_c = std::min(kMaxNstC, nst * stage / cstage);
      p->smem = total;
      return true;
    }
  }
  return false;
}

// The single-token decode uses the header alone ((K + 1) * I <= kActWords).
size_t layer_ws_bytes() { return kHeaderBytes; }

// Workspace of the grouped (T >= 2) decode, byte offsets (every section 256-B aligned).
struct GroupedLayout {
  size_t logits, meta, slot_expert, slot_pair0, pair_token, pair_slot, pair_nk, tok_pair, tok_w, tok_sg;
  size_t sched, xs_r, sf_r, xs_s, sf_s, gu_part, as, sfa, y_part, sh_gu, sh_y, xn, total;
};

GroupedLayout grouped_layout(int E, int H, int I, int K, int T) {
  GroupedLayout g;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  const size_t P = (size_t)T * K + T;
  g.logits = take((size_t)T * (E + 1) * 4);
  g.meta = take(16);
  g.slot_expert = take((size_t)kMaxPairs * 4);
  g.slot_pair0 = take((size_t)(kMaxPairs + 2) * 4);
  g.pair_token = take((size_t)kMaxPairs * 4);
  g.pair_slot = take((size_t)kMaxPairs * 4);
  g.pair_nk = take((size_t)kMaxPairs * 4);
  g.tok_pair = take((size_t)T * (K + 1) * 4);
  g.tok_w = take((size_t)T * K * 4);
  g.tok_sg = take((size_t)T * 4);
  g.sched = take((size_t)2 * kSchedInts * 4);
  g.xs_r = take((size_t)T * H * 4);
  g.sf_r = take((size_t)T * (H / 32) * 8);
  g.xs_s = take((size_t)T * H * 4);
  g.sf_s = take((size_t)T * (H / 32) * 8);
  g.gu_part = take(P * kMaxChunks * I * 8);
  g.as = take(P * I * 4);
  g.sfa = take(P * (I / 32) * 8);
  g.y_part = take(P * kMaxChunks * H * 4);
  // tensor-core shared expert partials (used when H and I are multiples of 512)
  g.sh_gu = take((size_t)2 * (H / kTcK) * kMaxTokens * I * 4);
  g.sh_y = take((size_t)(I / kTcK) * kMaxTokens * H * 4);
  g.xn = take((size_t)T * H * 4);  // the normalised inputs (input norm)
  g.total = off;
  return g;
}

using GroupedFn = void (*)(GroupArgs);
struct GroupedFns {
  GroupedFn prep, gateup, stage, down;
};
template <int BR, int BS>
GroupedFns grouped_fns_t() {
  return {grouped_prep_kernel<BR, BS>, grouped_gateup_kernel<BR, BS>, grouped_stage_act_kernel<BR, BS>,
          grouped_down_kernel<BR, BS>};
}
// (the combine and the router are independent of the code widths)
GroupedFns grouped_fns(int br, int bs) {
  if (br == 4) return bs == 4 ? grouped_fns_t<4, 4>() : grouped_fns_t<4, 2>();
  return bs == 4 ? grouped_fns_t<2, 4>() : grouped_fns_t<2, 2>();
}

// Launch the grouped decode (router, prep, gate/up, activation staging, down).
int launch_grouped(const fmoe_layer* L, const float* x, const float* residual, float* out, int T, void* ws,
                   int32_t* idx_out, float* w_out, DevInfo* info, cudaStream_t s) {
  const float* x_in = x;
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k, G = info->sms;
  const bool has_shared = L->shared != nullptr;
  const int br = L->bits, bs = has_shared ? L->shared_bits : L->bits;
  const GroupedLayout gl = grouped_layout(E, H, I, K, T);
  if (G > kMaxSchedCtas) return FMOE_EINVAL;  // (more SMs than the unit schedule holds CTAs)
  char* w8 = static_cast<char*>(ws);
  GroupArgs a;
  std::memset(&a, 0, sizeof(a));
  a.experts = static_cast<const char*>(L->experts);
  a.expert_stride = L->expert_stride;
  a.shared = static_cast<const char*>(L->shared);
  // With an input norm every later step reads the normalised inputs.
  float* xn = reinterpret_cast<float*>(w8 + gl.xn);
  if (L->norm_weight) x = xn;
  a.x = x;
  a.residual = residual;
  a.out = out;
  a.logits = reinterpret_cast<float*>(w8 + gl.logits);
  a.tb.meta = reinterpret_cast<int*>(w8 + gl.meta);
  a.tb.slot_expert = reinterpret_cast<int*>(w8 + gl.slot_expert);
  a.tb.slot_pair0 = reinterpret_cast<int*>(w8 + gl.slot_pair0);
  a.tb.pair_token = reinterpret_cast<int*>(w8 + gl.pair_token);
  a.tb.pair_slot = reinterpret_cast<int*>(w8 + gl.pair_slot);
  a.tb.pair_nk = reinterpret_cast<int*>(w8 + gl.pair_nk);
  a.tb.tok_pair = reinterpret_cast<int*>(w8 + gl.tok_pair);
  a.tb.tok_w = reinterpret_cast<float*>(w8 + gl.tok_w);
  a.tb.tok_sg = reinterpret_cast<float*>(w8 + gl.tok_sg);
  a.tb.sched = reinterpret_cast<int*>(w8 + gl.sched);
  a.xs_r = reinterpret_cast<float4*>(w8 + gl.xs_r);
  a.sf_r = reinterpret_cast<float2*>(w8 + gl.sf_r);
  const bool separate = has_shared && bs != br;
  a.xs_s = reinterpret_cast<float4*>(w8 + (separate ? gl.xs_s : gl.xs_r));
  a.sf_s = reinterpret_cast<float2*>(w8 + (separate ? gl.sf_s : gl.sf_r));
  a.gu_part = reinterpret_cast<float2*>(w8 + gl.gu_part);
  a.as = reinterpret_cast<float4*>(w8 + gl.as);
  a.sfa = reinterpret_cast<float2*>(w8 + gl.sfa);
  a.y_part = reinterpret_cast<float*>(w8 + gl.y_part);
  a.sh_gu = reinterpret_cast<float*>(w8 + gl.sh_gu);
  a.sh_y = reinterpret_cast<float*>(w8 + gl.sh_y);
  a.w_router = L->w_router;
  a.w_sgate = L->w_sgate;
  // The shared expert runs on the tensor cores when its matrices tile into
  // 128-row x 512-input tiles; otherwise it is one more slot of the CUDA-core
  // kernels.
  a.shared_tc = has_shared && H % kTcK == 0 && I % kTcK == 0;
  a.idx_out = idx_out;
  a.w_out = w_out;
  a.H = H;
  a.I = I;
  a.E = E;
  a.K = K;
  a.T = T;
  a.grid = G;
  a.bits_r = br;
  a.bits_s = bs;
  a.has_sgate = L->w_sgate != nullptr;
  a.timeout_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  for (int r = 0; r < 2; ++r) {
    const BlobOff o = blob_offsets(H, I, r == 0 ? br : bs);
    long long* d = r == 0 ? a.off_r : a.off_s;
    d[0] = o.gc;
    d[1] = o.gsb;
    d[2] = o.uc;
    d[3] = o.usb;
    d[4] = o.dc;
    d[5] = o.dsb;
  }
  // Shared-memory plans: per-warp rings of gate/up stages (full-row sized:
  // gate and up codes, each row's scale/bias superset) and of down stages
  // (kRC code rows and one scale/bias copy spanning them).
  int stage = 0, cstage = 0;
  for (int b : {br, bs}) {
    const int cap = ((H / 16 + 15) & ~15) + 16;
    stage = std::max(stage, 2 * (H * b / 8) + 2 * cap);
    cstage = std::max(cstage, kRC * (I * b / 8) + (int)round_up((size_t)kRC * (I / 16), 16) + 32);
  }
  a.stage_bytes = (int)round_up(stage, 128);
  a.c_stage_bytes = (int)round_up(cstage, 128);
  const int budget = info->grouped_max_smem;
  a.nst = std::min(kMaxNst, (budget - kWarps * kMaxNst * 8) / (kWarps * a.stage_bytes));
  a.nst_c = std::min(kMaxNstC, (budget - kWarps * kMaxNstC * 8) / (kWarps * a.c_stage_bytes));
  if (a.nst < 1 || a.nst_c < 1) return FMOE_EINVAL;
  const size_t smem_gu = (size_t)kWarps * a.nst * a.stage_bytes + (size_t)kWarps * a.nst * 8;
  const size_t smem_d = (size_t)kWarps * a.nst_c * a.c_stage_bytes + (size_t)kWarps * a.nst_c * 8;
  const GroupedFns fns = grouped_fns(br, bs);
  const int fi = layer_fn_index(br, bs);
  const GroupedFn tc1 = bs == 4 ? router_shared_gu_kernel<4> : router_shared_gu_kernel<2>;
  const GroupedFn tc2 = br == 4 ? (bs == 4 ? prep_shared_down_kernel<4, 4> : prep_shared_down_kernel<4, 2>)
                                : (bs == 4 ? prep_shared_down_kernel<2, 4> : prep_shared_down_kernel<2, 2>);
  if (!info->grouped_attr_set[fi]) {
    for (GroupedFn f : {fns.gateup, fns.down})
      if (cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, budget))
        return cuda_fail(e);
    for (GroupedFn f : {tc1, tc2})
      if (cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes))
        return cuda_fail(e);
    info->grouped_attr_set[fi] = true;
  }
  // Every step is a programmatic dependent launch (when enabled): its CTAs
  // may start while the previous kernel ends and wait for it in the kernel.
  cudaError_t e = cudaSuccess;
  auto launch = [&](auto f, dim3 grid, int threads, size_t smem, auto... args) {
    if (e != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (g_dependent_launch.load(std::memory_order_relaxed)) {
      cfg.attrs = attr;
      cfg.numAttrs = 1;
    }
    e = cudaLaunchKernelEx(&cfg, f, args...);
  };
  if (L->norm_weight) launch(rms_norm_tokens_kernel, dim3(T), kNormThreads, 0, x_in, L->norm_weight, L->norm_eps, H, xn);
  const int rows = E + (L->w_sgate ? 1 : 0);
  const int router_ctas = (rows + kRouterRows - 1) / kRouterRows;
  if (a.shared_tc) {
    const int n_gu = 2 * (I / kTcRows) * (H / kTcK), n_down = (H / kTcRows) * (I / kTcK);
    launch(tc1, dim3(std::max(router_ctas, n_gu)), kThreads, kTcSmemBytes, a);
    launch(tc2, dim3(1 + T + n_down), kThreads, kTcSmemBytes, a);
  } else {
    launch(router_tokens_kernel, dim3(router_ctas), kThreads, 0, L->w_router, L->w_sgate, x, T, H, E,
           const_cast<float*>(a.logits));
    launch(fns.prep, dim3(1 + T), kThreads, 0, a);
  }
  launch(fns.gateup, dim3(G), kThreads, smem_gu, a);
  launch(fns.stage, dim3(T * K + T), kStageThreads, (size_t)I * 4, a);
  launch(fns.down, dim3(G), kThreads, smem_d, a);
  launch(grouped_combine_kernel, dim3((H / 4 + kCombineThreads - 1) / kCombineThreads, T), kCombineThreads, 0, a);
  if (e != cudaSuccess) return cuda_fail(e);
  return FMOE_OK;
}

// Fill the grid-shape-dependent fields and the blob section offsets.
void set_offsets(LayerArgs& a, int G) {
  const int GW = G * kWarps;
  const int n_static = a.shared ? a.I : 0;
  a.off_a = a.n_router % GW;
  a.off_b = (int)(((long long)a.n_router + n_static) % GW);
  for (int r = 0; r < 2; ++r) {
    const BlobOff o = blob_offsets(a.H, a.I, r == 0 ? a.bits_r : a.bits_s);
    long long* d = r == 0 ? a.off_r : a.off_s;
    d[0] = o.gc;
    d[1] = o.gsb;
    d[2] = o.uc;
    d[3] = o.usb;
    d[4] = o.dc;
    d[5] = o.dsb;
  }
}

int launch_layer(const LayerArgs& args, const Plan& pl, DevInfo* info, cudaStream_t s) {
  const LayerFn fn = layer_fn(args.bits_r, args.bits_s);
  const int fi = layer_fn_index(args.bits_r, args.bits_s);
  if (!info->layer_attr_set[fi]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, info->max_smem);
    if (e != cudaSuccess) return cuda_fail(e);
    info->layer_attr_set[fi] = true;
  }
  LayerArgs a = args;
  if (!g_dependent_launch.load(std::memory_order_relaxed)) {
    void* kargs[] = {&a};
    cudaError_t e = cudaLaunchCooperativeKernel((const void*)fn, dim3(info->sms), dim3(kThreads), kargs, pl.smem, s);
    return e == cudaSuccess ? FMOE_OK : cuda_fail(e);
  }
  // Programmatic dependent launch: this grid's CTAs may start while the
  // previous kernel on the stream finishes (the kernel waits for it before
  // its first dependent access).  A plain launch gives no co-residency
  // guarantee, so it is only made when one CTA fits on every SM; the grid
  // is then resident once the previous grid has left (the grid barriers are
  // bounded waits either way).
  if (info->layer_occupancy[fi] < 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, pl.smem);
    if (e != cudaSuccess) return cuda_fail(e);
    info->layer_occupancy[fi] = n;
  }
  if (info->layer_occupancy[fi] < 1) return FMOE_EINVAL;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(info->sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, a);
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e);
}

// Fixed scratch for fmoe_layer_decode_noalloc: callers that cannot allocate
// device memory themselves get the decode's workspace from this file-scope
// array, which every GPU that loads the library keeps until the process exits.
constexpr size_t kNoallocScratchBytes = 128 << 10;
static_assert(kHeaderBytes <= kNoallocScratchBytes, "the scratch holds a single-token workspace");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch per device, looked up once per device
// (host code only sees a stand-in for the symbol, never its device address).
void* g_noalloc_ptr[64];
std::mutex g_noalloc_mu;

int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) return cuda_fail(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FMOE_OK;
}

}  // namespace

extern "C" {

size_t fmoe_expert_bytes(int hidden, int inter, int bits) {
  if (!shape_ok(hidden, inter) || !bits_ok(bits)) return 0;
  return (size_t)blob_offsets(hidden, inter, bits).total;
}

int fmoe_blob_offsets(int hidden, int inter, int bits, int64_t off[6]) {
  if (!off || !shape_ok(hidden, inter) || !bits_ok(bits)) return FMOE_EINVAL;
  const BlobOff o = blob_offsets(hidden, inter, bits);
  off[0] = o.gc;
  off[1] = o.gsb;
  off[2] = o.uc;
  off[3] = o.usb;
  off[4] = o.dc;
  off[5] = o.dsb;
  return FMOE_OK;
}

int fmoe_quantize_expert(const float* w_gate, const float* w_up, const float* w_down, int hidden,
                         int inter, int bits, int group, void* blob_out, size_t blob_bytes,
                         fmoe_stream_t stream) {
  if (!w_gate || !w_up || !w_down || !blob_out || group != FMOE_GROUP || !bits_ok(bits) ||
      !shape_ok(hidden, inter) || !aligned(blob_out, 256))
    return FMOE_EINVAL;
  const BlobOff o = blob_offsets(hidden, inter, bits);
  if (blob_bytes < (size_t)o.total) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = dev_info(&dev, &info)) return rc;
  if (int rc = check_stream(stream, dev)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(blob_out);
  struct M { const float* w; int rows, nin; long long c, sb; } m[3] = {
      {w_gate, inter, hidden, o.gc, o.gsb}, {w_up, inter, hidden, o.uc, o.usb}, {w_down, hidden, inter, o.dc, o.dsb}};
  for (auto& mm : m) {
    const long long n = (long long)mm.rows * (mm.nin / 64);
    quantize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        mm.w, mm.rows, mm.nin, bits, reinterpret_cast<uint32_t*>(b + mm.c), reinterpret_cast<uint32_t*>(b + mm.sb));
    if (cudaError_t e = cudaGetLastError()) return cuda_fail(e);
  }
  return FMOE_OK;
}

size_t fmoe_route_workspace_bytes(int T, int n_experts) {
  if (T < 1 || T > FMOE_MAX_TOKENS || n_experts < 1 || n_experts > FMOE_MAX_EXPERTS) return 0;
  return round_up((size_t)T * (n_experts + 1) * 4, 256);
}

int fmoe_route(const uint16_t* w_router, const uint16_t* w_sgate, const float* x, int T, int hidden,
               int n_experts, int top_k, int32_t* idx, float* w, float* sgate, float* logits_opt,
               void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  if (!w_router || !x || !idx || !w || !ws) return FMOE_EINVAL;
  if (T < 1 || T > FMOE_MAX_TOKENS || hidden <= 0 || hidden % 64 || hidden > FMOE_MAX_HIDDEN ||
      n_experts < 1 || n_experts > FMOE_MAX_EXPERTS || top_k < 1 || top_k > FMOE_MAX_TOPK ||
      top_k > n_experts)
    return FMOE_EINVAL;
  if (!aligned(w_router, 16) || !aligned(x, 16) || (w_sgate && !aligned(w_sgate, 16))) return FMOE_EINVAL;
  if (ws_bytes < fmoe_route_workspace_bytes(T, n_experts)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = dev_info(&dev, &info)) return rc;
  if (int rc = check_stream(stream, dev)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* lg = static_cast<float*>(ws);
  const int rows = n_experts + (w_sgate ? 1 : 0);
  router_logits_kernel<<<(rows + 7) / 8, 256, 0, s>>>(w_router, w_sgate, x, T, hidden, n_experts, lg);
  topk_kernel<<<(T + 3) / 4, 128, 0, s>>>(lg, T, n_experts, top_k, w_sgate != nullptr, idx, w, sgate);
  if (logits_opt) copy_logits_kernel<<<32, 256, 0, s>>>(lg, T, n_experts, logits_opt);
  if (cudaError_t e = cudaGetLastError()) return cuda_fail(e);
  return FMOE_OK;
}

size_t fmoe_expert_workspace_bytes(int hidden, int inter) {
  if (!shape_ok(hidden, inter)) return 0;
  return kHeaderBytes;  // inter <= 8192 < kActWords tagged activations
}

int fmoe_expert_forward(const void* blob, int hidden, int inter, int bits, const float* x, float* y,
                        void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  if (!blob || !x || !y || !ws || !bits_ok(bits) || !shape_ok(hidden, inter)) return FMOE_EINVAL;
  if (!aligned(blob, 256) || !aligned(x, 16) || !aligned(y, 16) || !aligned(ws, 256) || x == y)
    return FMOE_EINVAL;
  if (ws_bytes < fmoe_expert_workspace_bytes(hidden, inter)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = dev_info(&dev, &info)) return rc;
  if (int rc = check_stream(stream, dev)) return rc;
  Plan pl;
  if (!plan_layer(hidden, inter, 0, true, bits, bits, info->sms, 0, info->max_smem, &pl)) return FMOE_EINVAL;
  LayerArgs a;
  std::memset(&a, 0, sizeof(a));
  a.shared = static_cast<const char*>(blob);
  a.x = x;
  a.out = y;
  char* w8 = static_cast<char*>(ws);
  a.bar = reinterpret_cast<unsigned*>(w8);
  a.tact = reinterpret_cast<unsigned long long*>(w8 + kCounterBytes + kTagBytes);
  a.H = hidden;
  a.I = inter;
  a.E = 0;
  a.K = 0;
  a.bits_r = bits;
  a.bits_s = bits;
  a.n_router = 0;
  a.n_slots = 1;
  a.nst = pl.nst;
  a.stage_bytes = pl.stage_bytes;
  a.xs4_off = pl.xs4_off;
  a.xs2_off = pl.xs2_off;
  a.xu_off = pl.xu_off;
  a.vec_floats = pl.vec_floats;
  a.sf_floats = pl.sf_floats;
  a.ys_stride = pl.ys_stride;
  a.nst_c = pl.nst_c;
  a.c_stage_bytes = pl.c_stage_bytes;
  a.timeout_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  set_offsets(a, info->sms);
  return launch_layer(a, pl, info, reinterpret_cast<cudaStream_t>(stream));
}

size_t fmoe_workspace_bytes(const fmoe_layer* L, int T) {
  if (!L || T < 1 || T > FMOE_MAX_TOKENS) return 0;
  const size_t single = layer_ws_bytes();
  if (T == 1) return single;
  return std::max(single, grouped_layout(L->n_experts, L->hidden, L->inter, L->top_k, T).total);
}

int fmoe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  if (!ws) return FMOE_EINVAL;
  if (cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream))) return cuda_fail(e);
  return FMOE_OK;
}

}  // extern "C"

namespace {

// The argument checks of a layer decode call that need no device (shapes,
// pointers, alignment).  With `routed_given` the layer's router and expert
// table are not used (the caller passes the experts).
int check_layer_shape(const fmoe_layer* L, int T, bool routed_given) {
  if (!L) return FMOE_EINVAL;
  if (!routed_given && (!L->w_router || !L->experts)) return FMOE_EINVAL;
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
  if (!shape_ok(H, I) || !bits_ok(L->bits) || (L->shared && !bits_ok(L->shared_bits)) ||
      L->group != FMOE_GROUP || K < 1 || K > FMOE_MAX_TOPK || T < 1 || T > FMOE_MAX_TOKENS || (K + 1) * I > kActWords)
    return FMOE_EINVAL;
  if (!routed_given) {
    if (E < 1 || E > FMOE_MAX_EXPERTS || K > E) return FMOE_EINVAL;
    if (L->expert_stride < (int64_t)fmoe_expert_bytes(H, I, L->bits) || L->expert_stride % 256)
      return FMOE_EINVAL;
    if (!aligned(L->experts, 256) || !aligned(L->w_router, 16) || (L->w_sgate && !aligned(L->w_sgate, 16)))
      return FMOE_EINVAL;
  }
  if (L->shared && !aligned(L->shared, 256)) return FMOE_EINVAL;
  if (L->norm_weight && (!aligned(L->norm_weight, 16) || !(L->norm_eps >= 0.f) || !(L->norm_eps < INFINITY)))
    return FMOE_EINVAL;
  return FMOE_OK;
}

int check_layer_args(const fmoe_layer* L, const float* x, const float* residual, const float* out, int T,
                     bool routed_given) {
  if (!L || !x || !out) return FMOE_EINVAL;
  if (int rc = check_layer_shape(L, T, routed_given)) return rc;
  if (!aligned(x, 16) || !aligned(out, 16) || (residual && !aligned(residual, 16)) || x == out) return FMOE_EINVAL;
  return FMOE_OK;
}

// The current device and its info, and the check that `stream` belongs to it.
int device_for(fmoe_stream_t stream, int* dev_out, DevInfo** info_out) {
  if (int rc = dev_info(dev_out, info_out)) return rc;
  return check_stream(stream, *dev_out);
}


// The single-token kernel's arguments for a checked layer call; with
// `routed_given` there are no router rows (the routing comes from the
// caller).  Returns false if the layer does not fit the kernel's plan.
bool layer_args(const fmoe_layer* L, void* ws, DevInfo* info, bool routed_given, LayerArgs* out_a, Plan* pl) {
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
  const bool has_shared = L->shared != nullptr;
  const int n_router = routed_given ? 0 : E + (L->w_sgate ? 1 : 0);
  if (!plan_layer(H, I, K, has_shared, L->bits, has_shared ? L->shared_bits : L->bits, info->sms, n_router,
                  info->max_smem, pl))
    return false;
  LayerArgs& a = *out_a;
  std::memset(&a, 0, sizeof(a));
  a.w_router = routed_given ? nullptr : L->w_router;
  a.w_sgate = routed_given ? nullptr : L->w_sgate;
  a.experts = static_cast<const char*>(L->experts);
  a.expert_stride = L->expert_stride;
  a.shared = static_cast<const char*>(L->shared);
  char* w8 = static_cast<char*>(ws);
  a.bar = reinterpret_cast<unsigned*>(w8);
  a.tlog = reinterpret_cast<unsigned long long*>(w8 + kCounterBytes);
  a.tact = reinterpret_cast<unsigned long long*>(w8 + kCounterBytes + kTagBytes);
  a.H = H;
  a.I = I;
  a.E = routed_given ? 0 : E;
  a.K = K;
  a.bits_r = L->bits;
  a.bits_s = has_shared ? L->shared_bits : L->bits;
  a.n_router = n_router;
  a.n_slots = K + (has_shared ? 1 : 0);
  a.nst = pl->nst;
  a.stage_bytes = pl->stage_bytes;
  a.xs4_off = pl->xs4_off;
  a.xs2_off = pl->xs2_off;
  a.xu_off = pl->xu_off;
  a.vec_floats = pl->vec_floats;
  a.sf_floats = pl->sf_floats;
  a.ys_stride = pl->ys_stride;
  a.nst_c = pl->nst_c;
  a.c_stage_bytes = pl->c_stage_bytes;
  a.timeout_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  a.norm_w = L->norm_weight;
  a.norm_eps = L->norm_eps;
  // A router warp's row (2H bytes) fits in its ring: copy it there at entry.
  a.router_smem = (long long)pl->nst * pl->stage_bytes >= 2LL * H ? 1 : 0;
  set_offsets(a, info->sms);
  return true;
}

}  // namespace

extern "C" {

int fmoe_layer_decode(const fmoe_layer* L, const float* x, const float* residual, float* out, int T,
                      void* ws, size_t ws_bytes, int32_t* idx_out_opt, float* w_out_opt,
                      fmoe_stream_t stream) {
  if (!ws || !aligned(ws, 256)) return FMOE_EINVAL;
  if (int rc = check_layer_args(L, x, residual, out, T, false)) return rc;
  if (ws_bytes < fmoe_workspace_bytes(L, T)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = device_for(stream, &dev, &info)) return rc;
  if (L->n_experts + 1 > (kWarps / 2) * info->sms) return FMOE_EINVAL;  // router rows must leave staging warps
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T > 1) return launch_grouped(L, x, residual, out, T, ws, idx_out_opt, w_out_opt, info, s);
  LayerArgs a;
  Plan pl;
  if (!layer_args(L, ws, info, false, &a, &pl)) return FMOE_EINVAL;
  a.x = x;
  a.residual = residual;
  a.out = out;
  a.idx_out = idx_out_opt;
  a.w_out = w_out_opt;
  a.sg_out = nullptr;
  return launch_layer(a, pl, info, s);
}

int fmoe_experts_decode(const fmoe_layer* L, const void* const* expert_blobs, const float* expert_weights,
                        float shared_gate, const float* x, const float* residual, float* out, void* ws,
                        size_t ws_bytes, fmoe_stream_t stream) {
  if (!expert_blobs || !expert_weights || !ws || !aligned(ws, 256)) return FMOE_EINVAL;
  if (int rc = check_layer_args(L, x, residual, out, 1, true)) return rc;
  for (int k = 0; k < L->top_k; ++k)
    if (!expert_blobs[k] || !aligned(expert_blobs[k], 256)) return FMOE_EINVAL;
  if (ws_bytes < fmoe_workspace_bytes(L, 1)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = device_for(stream, &dev, &info)) return rc;
  LayerArgs a;
  Plan pl;
  if (!layer_args(L, ws, info, true, &a, &pl)) return FMOE_EINVAL;
  a.fixed_route = 1;
  for (int k = 0; k < L->top_k; ++k) {
    a.fixed_blob[k] = static_cast<const char*>(expert_blobs[k]);
    a.fixed_w[k] = expert_weights[k];
  }
  a.fixed_sg = shared_gate;
  a.x = x;
  a.residual = residual;
  a.out = out;
  return launch_layer(a, pl, info, reinterpret_cast<cudaStream_t>(stream));
}

int fmoe_layer_decode_noalloc(const fmoe_layer* L, const float* x, const float* residual, float* out, int T,
                              int32_t* idx_out_opt, float* w_out_opt, fmoe_stream_t stream) {
  if (!L) return FMOE_EINVAL;
  if (T != 1) return FMOE_EINVAL;  // single-token decodes only (a grouped workspace never fits the scratch)
  const size_t need = fmoe_workspace_bytes(L, T);
  if (need == 0) return FMOE_EINVAL;
  if (need > kNoallocScratchBytes) return FMOE_ENOMEM;  // layer too large for the fixed scratch
  // Every check of the decode itself comes first: a call that is rejected
  // enqueues nothing (not even the clearing of the scratch below).
  if (int rc = check_layer_args(L, x, residual, out, T, false)) return rc;
  int dev = 0;
  DevInfo* info = nullptr;
  if (int rc = device_for(stream, &dev, &info)) return rc;
  if (L->n_experts + 1 > (kWarps / 2) * info->sms) return FMOE_EINVAL;  // router rows must leave staging warps
  void* ws = nullptr;
  if (int rc = noalloc_scratch(dev, &ws)) return rc;
  // The scratch keeps whatever the previous call left: clear the counters and
  // the tagged words (epoch 0, no word tagged), as a fresh workspace has them.
  if (cudaError_t e = cudaMemsetAsync(ws, 0, kHeaderBytes, reinterpret_cast<cudaStream_t>(stream)))
    return cuda_fail(e);
  return fmoe_layer_decode(L, x, residual, out, T, ws, kNoallocScratchBytes, idx_out_opt, w_out_opt, stream);
}

int fmoe_get_status(fmoe_stream_t stream, unsigned* bits_out) {
  if (cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream))) return cuda_fail(e);
  unsigned v = 0, zero = 0;
  if (cudaError_t e = cudaMemcpyFromSymbol(&v, g_fmoe_status, sizeof(v))) return cuda_fail(e);
  if (v) {
    if (cudaError_t e = cudaMemcpyToSymbol(g_fmoe_status, &zero, sizeof(zero))) return cuda_fail(e);
  }
  if (bits_out) *bits_out = v;
  return v ? FMOE_EDEVICE : FMOE_OK;
}

int fmoe_last_cuda_error(void) { return g_last_cuda_error; }

int fmoe_set_wait_limit_ns(unsigned long long limit_ns, unsigned long long* previous_opt) {
  if (limit_ns < kMinWaitNs || limit_ns > kMaxWaitNs) return FMOE_EINVAL;
  const unsigned long long old = g_wait_limit_ns.exchange(limit_ns);
  if (previous_opt) *previous_opt = old;
  return FMOE_OK;
}

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bn && y < x + an;
}

int fmoe_delta_update(float* state, const float* q, const float* k, const float* v, const float* alpha,
                      const float* beta, float* o, int heads, int dk, int dv, int T, fmoe_stream_t stream) {
  if (!state || !q || !k || !v || !alpha || !beta || !o) return FMOE_EINVAL;
  if (heads < 1 || heads > FMOE_DELTA_MAX_DIM || dv < 1 || dv > FMOE_DELTA_MAX_DIM || T < 1 ||
      T > FMOE_DELTA_MAX_DIM || dk < 128 || dk > 512 || dk % 128 != 0)
    return FMOE_EINVAL;
  if (!aligned(state, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 4) || !aligned(alpha, 4) ||
      !aligned(beta, 4) || !aligned(o, 4))
    return FMOE_EINVAL;
  // The state and the readout are written: neither may overlap the other or an input.
  const size_t sb = (size_t)heads * dv * dk * 4, kb = (size_t)T * heads * dk * 4, vb = (size_t)T * heads * dv * 4,
               gb = (size_t)T * heads * 4;
  const void* in[5] = {q, k, v, alpha, beta};
  const size_t inb[5] = {kb, kb, vb, gb, gb};
  if (overlaps(state, sb, o, vb)) return FMOE_EINVAL;
  for (int j = 0; j < 5; ++j)
    if (overlaps(state, sb, in[j], inb[j]) || overlaps(o, vb, in[j], inb[j])) return FMOE_EINVAL;
  int dev;
  DevInfo* info;
  if (int rc = dev_info(&dev, &info)) return rc;
  if (int rc = check_stream(stream, dev)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeltaArgs a;
  a.state = state;
  a.q = q;
  a.k = k;
  a.v = v;
  a.alpha = alpha;
  a.beta = beta;
  a.o = o;
  a.heads = heads;
  a.dk = dk;
  a.dv = dv;
  a.T = T;
  const long long rows = (long long)heads * dv;
  const long long per_cta = (long long)kDeltaWarps * delta_rows_per_warp(dk / 128);
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  switch (dk / 128) {
    case 1: delta_update_kernel<1><<<grid, kDeltaWarps * 32, 0, s>>>(a); break;
    case 2: delta_update_kernel<2><<<grid, kDeltaWarps * 32, 0, s>>>(a); break;
    case 3: delta_update_kernel<3><<<grid, kDeltaWarps * 32, 0, s>>>(a); break;
    default: delta_update_kernel<4><<<grid, kDeltaWarps * 32, 0, s>>>(a); break;
  }
  if (cudaError_t e = cudaGetLastError()) return cuda_fail(e);
  return FMOE_OK;
}

struct fmoe_expert_cache_s {
  fmoe::ExpertCache c;
  explicit fmoe_expert_cache_s(int n) : c(n) {}
};

int fmoe_cache_create(int n_slots, fmoe_expert_cache** cache_out) {
  if (!cache_out || n_slots < 1 || n_slots > FMOE_CACHE_MAX_SLOTS) return FMOE_EINVAL;
  *cache_out = nullptr;
  try {
    *cache_out = new fmoe_expert_cache_s(n_slots);
  } catch (...) {
    return FMOE_ENOMEM;
  }
  return FMOE_OK;
}

int fmoe_cache_destroy(fmoe_expert_cache* cache) {
  delete cache;
  return FMOE_OK;
}

int fmoe_cache_lookup(fmoe_expert_cache* cache, int layer, const int32_t* idx, int K, int32_t* slot_out,
                      int32_t* miss_out, int* n_miss_out) {
  if (!cache || !idx || !slot_out || !miss_out || layer < 0 || K < 1 || K > cache->c.n_slots()) return FMOE_EINVAL;
  for (int k = 0; k < K; ++k)
    if (idx[k] < 0) return FMOE_EINVAL;
  try {
    cache->c.lookup(layer, idx, K, slot_out, miss_out);
  } catch (...) {
    return FMOE_ENOMEM;
  }
  if (n_miss_out) {
    int n = 0;
    for (int k = 0; k < K; ++k) n += miss_out[k];
    *n_miss_out = n;
  }
  return FMOE_OK;
}

int fmoe_cache_stats(const fmoe_expert_cache* cache, uint64_t* hits, uint64_t* misses, uint64_t* evictions) {
  if (!cache) return FMOE_EINVAL;
  cache->c.stats(hits, misses, evictions);
  return FMOE_OK;
}

int fmoe_cache_reset(fmoe_expert_cache* cache) {
  if (!cache) return FMOE_EINVAL;
  cache->c.reset();
  return FMOE_OK;
}

int fmoe_set_dependent_launch(int enable, int* previous_opt) {
  if (enable != 0 && enable != 1) return FMOE_EINVAL;
  const int old = g_dependent_launch.exchange(enable);
  if (previous_opt) *previous_opt = old;
  return FMOE_OK;
}

#ifdef FMOE_TRACE_BUILD
// Trace builds only: copy the phase timestamps of the last layer launch
// ([1024][kTraceCols] u64: SM cycles at the trace points, then globaltimer ns
// at the dependency wait and at the end and the cycles at the end) to host
// memory and clear them.
int fmoe_trace_read(unsigned long long* host) {
  if (cudaError_t e = cudaMemcpyFromSymbol(host, g_fmoe_trace, sizeof(g_fmoe_trace))) return cuda_fail(e);
  static unsigned long long zero[1024][kTraceCols];
  if (cudaError_t e = cudaMemcpyToSymbol(g_fmoe_trace, zero, sizeof(zero))) return cuda_fail(e);
  return FMOE_OK;
}
int fmoe_spins_read(unsigned long long* host4) {
  if (cudaError_t e = cudaMemcpyFromSymbol(host4, g_fmoe_spins, 4 * sizeof(unsigned long long))) return cuda_fail(e);
  static unsigned long long zero[4];
  if (cudaError_t e = cudaMemcpyToSymbol(g_fmoe_spins, zero, sizeof(zero))) return cuda_fail(e);
  return FMOE_OK;
}
#endif

const char* fmoe_strerror(int code) {
  switch (code) {
    case FMOE_OK: return "ok";
    case FMOE_EINVAL: return "invalid argument (null pointer, unsupported size or alignment)";
    case FMOE_ENOMEM: return "caller-provided buffer or workspace too small";
    case FMOE_ECUDA: return "CUDA runtime or launch error";
    case FMOE_EDEVICE: return "a kernel reported an error through the device status word";
    default: return "unknown error code";
  }
}

}  // extern "C"

#include "streamer.cuh"
