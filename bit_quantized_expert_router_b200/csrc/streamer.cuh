// Streaming routed experts from host memory: the B200 counterpart of the
// pages' expert streaming ("Flash-MoE: Ausführen eines 397B-Parameter-Qwen-
// Modells ...", sections "SSD-Experten-Streaming" and "Verzögerte GPU-
// Experten-Berechnung").  In the pages the routed experts stay on the SSD,
// only the K selected ones are read per layer (parallel pread), and the OS
// page cache keeps the recently used ones (an LRU).  Here they stay in pinned
// host memory, the device keeps n_slots of them in slots of one buffer, and
// the LRU directory is the library's fmoe_cache.  Per layer and token:
//   1. router GEMV + top-K on the GPU (fmoe_route's kernels), the decision
//      copied to pinned host memory: the one synchronisation of the step;
//   2. the directory gives each selected expert its slot; every miss is one
//      cudaMemcpyAsync from host to its slot, on the copy stream;
//   3. meanwhile the shared expert and the hits are decoded on the compute
//      stream (out = residual + hits + gated shared), and the misses are added
//      by a second launch once their copies have landed.
// The host returns as soon as the launches are queued (the pages' deferred
// expert command): the next layer's routing is queued behind them.
// Included at the end of fmoe_api.cu (it uses that file's internal helpers).
#pragma once

struct fmoe_streamer_s {
  std::vector<fmoe_layer> layers;
  std::vector<const char*> host;  // per layer: E blobs at expert_stride (pinned host memory)
  char* slots = nullptr;
  int n_slots = 0;
  long long stride = 0;
  size_t blob_bytes = 0;
  fmoe_expert_cache* cache = nullptr;
  int dev = 0;
  // device: [K] idx, [K] w, [1] sg (one block), the router workspace
  void* d_route = nullptr;
  void* d_route_ws = nullptr;
  size_t route_ws_bytes = 0;
  void* h_route = nullptr;  // pinned host copy of the decision block
  cudaEvent_t copied = nullptr;
  uint64_t h2d_bytes = 0, steps = 0;
};

namespace {

constexpr size_t kDecisionBytes = 2 * FMOE_MAX_TOPK * 4 + 16;

// Host-only checks of a streamer's layers (no CUDA call).
int check_streamer_layers(const fmoe_layer* layers, int n_layers, const void* const* host_experts, void* slots,
                          int n_slots) {
  if (!layers || n_layers < 1 || !host_experts || !slots || !aligned(slots, 256)) return FMOE_EINVAL;
  const fmoe_layer& L0 = layers[0];
  for (int l = 0; l < n_layers; ++l) {
    const fmoe_layer& L = layers[l];
    if (!host_experts[l] || !aligned(host_experts[l], 256)) return FMOE_EINVAL;
    if (!L.w_router || L.norm_weight) return FMOE_EINVAL;  // routing reads x as given
    if (L.hidden != L0.hidden || L.inter != L0.inter || L.n_experts != L0.n_experts || L.top_k != L0.top_k ||
        L.bits != L0.bits || L.expert_stride != L0.expert_stride)
      return FMOE_EINVAL;  // the slots are shared by every layer
    if (int rc = check_layer_shape(&L, 1, true)) return rc;
    if (L.n_experts < 1 || L.n_experts > FMOE_MAX_EXPERTS || L.top_k > L.n_experts) return FMOE_EINVAL;
    if (L.expert_stride < (int64_t)fmoe_expert_bytes(L.hidden, L.inter, L.bits) || L.expert_stride % 256)
      return FMOE_EINVAL;
    if (!aligned(L.w_router, 16) || (L.w_sgate && !aligned(L.w_sgate, 16))) return FMOE_EINVAL;
  }
  if (n_slots < L0.top_k || n_slots > FMOE_CACHE_MAX_SLOTS) return FMOE_EINVAL;
  return FMOE_OK;
}

void streamer_free(fmoe_streamer* s) {
  if (!s) return;
  if (s->copied) cudaEventDestroy(s->copied);
  if (s->h_route) cudaFreeHost(s->h_route);
  if (s->d_route) cudaFree(s->d_route);
  if (s->d_route_ws) cudaFree(s->d_route_ws);
  if (s->cache) fmoe_cache_destroy(s->cache);
  delete s;
}

// One given-routing launch of the layer kernel: experts blobs[0..n) with
// weights w, plus the shared expert when `shared` (gate sg).
int streamer_launch(const fmoe_layer& L, int n, const char* const* blobs, const float* w, bool shared, float sg,
                    const float* x, const float* residual, float* out, void* ws, DevInfo* info, cudaStream_t s) {
  fmoe_layer Lc = L;
  Lc.top_k = n;
  if (!shared) Lc.shared = nullptr;
  if (n == 0) Lc.bits = Lc.shared_bits;  // no routed expert: one code width
  LayerArgs a;
  Plan pl;
  if (!layer_args(&Lc, ws, info, true, &a, &pl)) return FMOE_EINVAL;
  a.fixed_route = 1;
  for (int k = 0; k < n; ++k) {
    a.fixed_blob[k] = blobs[k];
    a.fixed_w[k] = w[k];
  }
  a.fixed_sg = sg;
  a.x = x;
  a.residual = residual;
  a.out = out;
  return launch_layer(a, pl, info, s);
}

}  // namespace

extern "C" {

int fmoe_streamer_create(const fmoe_layer* layers, int n_layers, const void* const* host_experts, void* slots,
                         int n_slots, fmoe_streamer** out) {
  if (!out) return FMOE_EINVAL;
  *out = nullptr;
  if (int rc = check_streamer_layers(layers, n_layers, host_experts, slots, n_slots)) return rc;
  int dev;
  DevInfo* info;
  if (int rc = dev_info(&dev, &info)) return rc;
  // the experts must be page-locked host memory, so that each copy is one
  // asynchronous DMA transfer
  for (int l = 0; l < n_layers; ++l) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host_experts[l]) != cudaSuccess || at.type != cudaMemoryTypeHost) {
      cudaGetLastError();
      return FMOE_EINVAL;
    }
  }
  fmoe_streamer* s = new (std::nothrow) fmoe_streamer;
  if (!s) return FMOE_ENOMEM;
  s->layers.assign(layers, layers + n_layers);
  for (int l = 0; l < n_layers; ++l) s->host.push_back(static_cast<const char*>(host_experts[l]));
  s->slots = static_cast<char*>(slots);
  s->n_slots = n_slots;
  s->stride = layers[0].expert_stride;
  s->blob_bytes = fmoe_expert_bytes(layers[0].hidden, layers[0].inter, layers[0].bits);
  s->dev = dev;
  s->route_ws_bytes = fmoe_route_workspace_bytes(1, layers[0].n_experts);
  int rc = fmoe_cache_create(n_slots, &s->cache);
  cudaError_t e = cudaSuccess;
  if (rc == FMOE_OK && (e = cudaMalloc(&s->d_route, kDecisionBytes)) != cudaSuccess) rc = cuda_fail(e);
  if (rc == FMOE_OK && (e = cudaMalloc(&s->d_route_ws, s->route_ws_bytes)) != cudaSuccess) rc = cuda_fail(e);
  if (rc == FMOE_OK && (e = cudaHostAlloc(&s->h_route, kDecisionBytes, cudaHostAllocDefault)) != cudaSuccess)
    rc = cuda_fail(e);
  if (rc == FMOE_OK && (e = cudaEventCreateWithFlags(&s->copied, cudaEventDisableTiming)) != cudaSuccess)
    rc = cuda_fail(e);
  if (rc != FMOE_OK) {
    streamer_free(s);
    return rc;
  }
  *out = s;
  return FMOE_OK;
}

int fmoe_streamer_destroy(fmoe_streamer* s) {
  streamer_free(s);
  return FMOE_OK;
}

int fmoe_streamer_decode(fmoe_streamer* s, int layer, const float* x, const float* residual, float* out, void* ws,
                         size_t ws_bytes, fmoe_stream_t stream, fmoe_stream_t copy_stream, int32_t* idx_out_opt,
                         float* w_out_opt) {
  if (!s || layer < 0 || layer >= (int)s->layers.size() || !ws || !aligned(ws, 256)) return FMOE_EINVAL;
  const fmoe_layer& L = s->layers[layer];
  if (int rc = check_layer_args(&L, x, residual, out, 1, true)) return rc;
  if (ws_bytes < fmoe_workspace_bytes(&L, 1)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = device_for(stream, &dev, &info)) return rc;
  if (dev != s->dev) return FMOE_EINVAL;
  if (int rc = check_stream(copy_stream, dev)) return rc;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t ks = reinterpret_cast<cudaStream_t>(copy_stream);
  const int K = L.top_k;
  // 1. routing on the GPU, the decision to the host
  char* d = static_cast<char*>(s->d_route);
  int32_t* d_idx = reinterpret_cast<int32_t*>(d);
  float* d_w = reinterpret_cast<float*>(d + FMOE_MAX_TOPK * 4);
  float* d_sg = reinterpret_cast<float*>(d + 2 * FMOE_MAX_TOPK * 4);
  if (int rc = fmoe_route(L.w_router, L.w_sgate, x, 1, L.hidden, L.n_experts, K, d_idx, d_w, d_sg, nullptr,
                          s->d_route_ws, s->route_ws_bytes, stream))
    return rc;
  if (cudaError_t e = cudaMemcpyAsync(s->h_route, s->d_route, kDecisionBytes, cudaMemcpyDeviceToHost, cs))
    return cuda_fail(e);
  if (cudaError_t e = cudaStreamSynchronize(cs)) return cuda_fail(e);
  const char* h = static_cast<const char*>(s->h_route);
  const int32_t* idx = reinterpret_cast<const int32_t*>(h);
  const float* w = reinterpret_cast<const float*>(h + FMOE_MAX_TOPK * 4);
  const float sg = *reinterpret_cast<const float*>(h + 2 * FMOE_MAX_TOPK * 4);
  for (int k = 0; k < K; ++k)
    if (idx[k] < 0 || idx[k] >= L.n_experts) return FMOE_EDEVICE;  // (fmoe_route always gives valid indices)
  if (idx_out_opt) std::memcpy(idx_out_opt, idx, K * sizeof(int32_t));
  if (w_out_opt) std::memcpy(w_out_opt, w, K * sizeof(float));
  // 2. slots; the misses' copies on the copy stream (every earlier kernel that
  // read a slot has completed: the stream was synchronised above)
  int32_t slot[FMOE_MAX_TOPK], miss[FMOE_MAX_TOPK];
  int n_miss = 0;
  if (int rc = fmoe_cache_lookup(s->cache, layer, idx, K, slot, miss, &n_miss)) return rc;
  const char* hit_blob[FMOE_MAX_TOPK];
  const char* miss_blob[FMOE_MAX_TOPK];
  float hit_w[FMOE_MAX_TOPK], miss_w[FMOE_MAX_TOPK];
  int n_hit = 0, nm = 0;
  for (int k = 0; k < K; ++k) {
    const char* dst = s->slots + (long long)slot[k] * s->stride;
    if (miss[k]) {
      const char* src = s->host[layer] + (long long)idx[k] * s->stride;
      if (cudaError_t e = cudaMemcpyAsync((void*)dst, src, s->blob_bytes, cudaMemcpyHostToDevice, ks))
        return cuda_fail(e);
      s->h2d_bytes += s->blob_bytes;
      miss_blob[nm] = dst;
      miss_w[nm++] = w[k];
    } else {
      hit_blob[n_hit] = dst;
      hit_w[n_hit++] = w[k];
    }
  }
  if (nm > 0)
    if (cudaError_t e = cudaEventRecord(s->copied, ks)) return cuda_fail(e);
  // 3. the shared expert and the hits while the copies run, then the misses
  const bool first = n_hit > 0 || L.shared != nullptr;
  if (first)
    if (int rc = streamer_launch(L, n_hit, hit_blob, hit_w, true, sg, x, residual, out, ws, info, cs)) return rc;
  if (nm > 0) {
    if (cudaError_t e = cudaStreamWaitEvent(cs, s->copied, 0)) return cuda_fail(e);
    if (int rc = streamer_launch(L, nm, miss_blob, miss_w, false, 1.0f, x, first ? out : residual, out, ws, info,
                                 cs))
      return rc;
  }
  ++s->steps;
  return FMOE_OK;
}

int fmoe_streamer_stats(const fmoe_streamer* s, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes) {
  if (!s) return FMOE_EINVAL;
  if (int rc = fmoe_cache_stats(s->cache, hits, misses, nullptr)) return rc;
  if (h2d_bytes) *h2d_bytes = s->h2d_bytes;
  return FMOE_OK;
}

}  // extern "C"
