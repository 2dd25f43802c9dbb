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
// The same step in two halves (fmoe_streamer_prepare: routing, slots, copies;
// fmoe_streamer_finish: the decode launches) lets a caller whose next layer's
// input is already known prepare that layer while this one decodes, so that
// its copies overlap this layer's compute.  Every slot remembers the event
// recorded after the last decode that read it, and a copy into it waits for
// that event only.
// Included at the end of fmoe_api.cu (it uses that file's internal helpers).
#pragma once

// A prepared layer: its routing decision, slots and copy event.
struct StreamerPending {
  int layer = -1;
  int n_hit = 0, n_miss = 0;
  const char* hit_blob[FMOE_MAX_TOPK];
  const char* miss_blob[FMOE_MAX_TOPK];
  float hit_w[FMOE_MAX_TOPK], miss_w[FMOE_MAX_TOPK];
  int32_t slot[FMOE_MAX_TOPK];
  float sg = 1.0f;
  cudaEvent_t copied = nullptr;
};

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
  StreamerPending pend[2];            // prepared, not yet finished layers, oldest first
  int n_pend = 0, pend_head = 0;
  std::vector<cudaEvent_t> slot_ev;  // per slot: recorded after the last decode that read it
  std::vector<char> slot_used;
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
  for (StreamerPending& p : s->pend)
    if (p.copied) cudaEventDestroy(p.copied);
  for (cudaEvent_t e : s->slot_ev)
    if (e) cudaEventDestroy(e);
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
  for (StreamerPending& p : s->pend)
    if (rc == FMOE_OK && (e = cudaEventCreateWithFlags(&p.copied, cudaEventDisableTiming)) != cudaSuccess)
      rc = cuda_fail(e);
  if (rc == FMOE_OK) {
    try {
      s->slot_ev.assign(n_slots, nullptr);
      s->slot_used.assign(n_slots, 0);
    } catch (...) {
      rc = FMOE_ENOMEM;
    }
  }
  for (int i = 0; rc == FMOE_OK && i < n_slots; ++i)
    if ((e = cudaEventCreateWithFlags(&s->slot_ev[i], cudaEventDisableTiming)) != cudaSuccess) rc = cuda_fail(e);
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

int fmoe_streamer_prepare(fmoe_streamer* s, int layer, const float* x, fmoe_stream_t route_stream,
                          fmoe_stream_t copy_stream, int32_t* idx_out_opt, float* w_out_opt) {
  if (!s || layer < 0 || layer >= (int)s->layers.size() || !x || !aligned(x, 16)) return FMOE_EINVAL;
  const fmoe_layer& L = s->layers[layer];
  const int K = L.top_k;
  // at most two layers in flight, and the pending one's experts must survive
  // this layer's evictions (the directory evicts the least recent first)
  if (s->n_pend == 2 || (s->n_pend == 1 && s->n_slots < 2 * K)) return FMOE_EINVAL;
  int dev;
  DevInfo* info;
  if (int rc = device_for(route_stream, &dev, &info)) return rc;
  if (dev != s->dev) return FMOE_EINVAL;
  if (int rc = check_stream(copy_stream, dev)) return rc;
  cudaStream_t rs = reinterpret_cast<cudaStream_t>(route_stream);
  cudaStream_t ks = reinterpret_cast<cudaStream_t>(copy_stream);
  // 1. routing on the GPU, the decision to the host
  char* d = static_cast<char*>(s->d_route);
  int32_t* d_idx = reinterpret_cast<int32_t*>(d);
  float* d_w = reinterpret_cast<float*>(d + FMOE_MAX_TOPK * 4);
  float* d_sg = reinterpret_cast<float*>(d + 2 * FMOE_MAX_TOPK * 4);
  if (int rc = fmoe_route(L.w_router, L.w_sgate, x, 1, L.hidden, L.n_experts, K, d_idx, d_w, d_sg, nullptr,
                          s->d_route_ws, s->route_ws_bytes, route_stream))
    return rc;
  if (cudaError_t e = cudaMemcpyAsync(s->h_route, s->d_route, kDecisionBytes, cudaMemcpyDeviceToHost, rs))
    return cuda_fail(e);
  if (cudaError_t e = cudaStreamSynchronize(rs)) return cuda_fail(e);
  const char* h = static_cast<const char*>(s->h_route);
  const int32_t* idx = reinterpret_cast<const int32_t*>(h);
  const float* w = reinterpret_cast<const float*>(h + FMOE_MAX_TOPK * 4);
  for (int k = 0; k < K; ++k)
    if (idx[k] < 0 || idx[k] >= L.n_experts) return FMOE_EDEVICE;  // (fmoe_route always gives valid indices)
  if (idx_out_opt) std::memcpy(idx_out_opt, idx, K * sizeof(int32_t));
  if (w_out_opt) std::memcpy(w_out_opt, w, K * sizeof(float));
  // 2. slots; each miss copied after the last decode that read its slot
  StreamerPending& p = s->pend[(s->pend_head + s->n_pend) % 2];
  int32_t miss[FMOE_MAX_TOPK];
  int n_miss = 0;
  if (int rc = fmoe_cache_lookup(s->cache, layer, idx, K, p.slot, miss, &n_miss)) return rc;
  p.layer = layer;
  p.n_hit = p.n_miss = 0;
  p.sg = *reinterpret_cast<const float*>(h + 2 * FMOE_MAX_TOPK * 4);
  for (int k = 0; k < K; ++k) {
    const int sl = p.slot[k];
    const char* dst = s->slots + (long long)sl * s->stride;
    if (miss[k]) {
      if (s->slot_used[sl])
        if (cudaError_t e = cudaStreamWaitEvent(ks, s->slot_ev[sl], 0)) return cuda_fail(e);
      const char* src = s->host[layer] + (long long)idx[k] * s->stride;
      if (cudaError_t e = cudaMemcpyAsync((void*)dst, src, s->blob_bytes, cudaMemcpyHostToDevice, ks))
        return cuda_fail(e);
      s->h2d_bytes += s->blob_bytes;
      p.miss_blob[p.n_miss] = dst;
      p.miss_w[p.n_miss++] = w[k];
    } else {
      p.hit_blob[p.n_hit] = dst;
      p.hit_w[p.n_hit++] = w[k];
    }
  }
  if (p.n_miss > 0)
    if (cudaError_t e = cudaEventRecord(p.copied, ks)) return cuda_fail(e);
  ++s->n_pend;
  return FMOE_OK;
}

int fmoe_streamer_finish(fmoe_streamer* s, int layer, const float* x, const float* residual, float* out, void* ws,
                         size_t ws_bytes, fmoe_stream_t stream) {
  if (!s || layer < 0 || layer >= (int)s->layers.size() || !ws || !aligned(ws, 256)) return FMOE_EINVAL;
  if (s->n_pend == 0 || s->pend[s->pend_head].layer != layer) return FMOE_EINVAL;  // finish in prepare order
  const fmoe_layer& L = s->layers[layer];
  if (int rc = check_layer_args(&L, x, residual, out, 1, true)) return rc;
  if (ws_bytes < fmoe_workspace_bytes(&L, 1)) return FMOE_ENOMEM;
  int dev;
  DevInfo* info;
  if (int rc = device_for(stream, &dev, &info)) return rc;
  if (dev != s->dev) return FMOE_EINVAL;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  StreamerPending& p = s->pend[s->pend_head];
  // 3. the shared expert and the hits while the copies run, then the misses
  const bool first = p.n_hit > 0 || L.shared != nullptr;
  if (first)
    if (int rc = streamer_launch(L, p.n_hit, p.hit_blob, p.hit_w, true, p.sg, x, residual, out, ws, info, cs))
      return rc;
  if (p.n_miss > 0) {
    if (cudaError_t e = cudaStreamWaitEvent(cs, p.copied, 0)) return cuda_fail(e);
    if (int rc = streamer_launch(L, p.n_miss, p.miss_blob, p.miss_w, false, 1.0f, x, first ? out : residual, out,
                                 ws, info, cs))
      return rc;
  }
  // the slots this decode read may be overwritten once it is done
  for (int k = 0; k < L.top_k; ++k) {
    if (cudaError_t e = cudaEventRecord(s->slot_ev[p.slot[k]], cs)) return cuda_fail(e);
    s->slot_used[p.slot[k]] = 1;
  }
  s->pend_head = (s->pend_head + 1) % 2;
  --s->n_pend;
  ++s->steps;
  return FMOE_OK;
}

int fmoe_streamer_decode(fmoe_streamer* s, int layer, const float* x, const float* residual, float* out, void* ws,
                         size_t ws_bytes, fmoe_stream_t stream, fmoe_stream_t copy_stream, int32_t* idx_out_opt,
                         float* w_out_opt) {
  if (!s || layer < 0 || layer >= (int)s->layers.size() || !ws || !aligned(ws, 256)) return FMOE_EINVAL;
  if (s->n_pend != 0) return FMOE_EINVAL;  // a prepared layer is waiting for its finish
  const fmoe_layer& L = s->layers[layer];
  if (int rc = check_layer_args(&L, x, residual, out, 1, true)) return rc;
  if (ws_bytes < fmoe_workspace_bytes(&L, 1)) return FMOE_ENOMEM;
  if (int rc = fmoe_streamer_prepare(s, layer, x, stream, copy_stream, idx_out_opt, w_out_opt)) return rc;
  return fmoe_streamer_finish(s, layer, x, residual, out, ws, ws_bytes, stream);
}

int fmoe_streamer_stats(const fmoe_streamer* s, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes) {
  if (!s) return FMOE_EINVAL;
  if (int rc = fmoe_cache_stats(s->cache, hits, misses, nullptr)) return rc;
  if (h2d_bytes) *h2d_bytes = s->h2d_bytes;
  return FMOE_OK;
}

}  // extern "C"
