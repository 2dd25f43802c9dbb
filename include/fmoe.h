/*
 * fmoe — quantised Mixture-of-Experts layer decode (one token or a few) on NVIDIA B200
 * (sm_100a).  C ABI of libfmoe.so.
 *
 * What the library computes is the MoE step of the Flash-MoE engine, as its
 * pages describe it:
 *   [P1] "397B MoE en MacBook: Motor Flash-MoE a 4,4 t/s" (aibit.im)
 *   [P2] "Flash-MoE: Ausführen eines 397B-Parameter-Qwen-Modells auf dem
 *        MacBook Pro mit reinem C/Metal" (openclawradar.com)
 *   [P3] "Flash-MoE - Executando um modelo de 397 bilhões de parâmetros em um
 *        notebook" (news.hada.io)
 * A router projection over the experts, softmax and top-K with renormalised
 * weights ([P2] "Pipeline-Leistung"); K routed experts plus one shared expert
 * ([P2] "Technische Implementierung"), each a gate and an up projection, a
 * fused SwiGLU and a down projection on affine group-quantised weights
 * (weight = nibble * scale + bias, evaluated as fma(nibble, scale*x, bias*x):
 * [P1] "Técnicas innovadoras" item 2, [P2] "FMA-optimierter Dequant-Kernel");
 * and a fused end step that adds the weighted expert outputs, the residual and
 * the sigmoid-gated shared expert ([P2] "Metal-Compute-Shader").  Beside it,
 * the gated delta-rule update of the model's linear-attention state
 * (fmoe_delta_update; [P2] "Accelerate-BLAS für lineare Aufmerksamkeit").
 *
 * Conventions for every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them past the call.
 *   - All work is enqueued asynchronously on the caller's stream `stream`
 *     (a cudaStream_t; NULL is the legacy default stream).  Entry points do
 *     not synchronise, except fmoe_get_status().
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns an error code and enqueues nothing.
 *   - Return values: FMOE_OK or one of the FMOE_E* codes below.
 *
 * Packed expert format (the pages fix only the affine form; the layout is this
 * library's, one reading among several):
 *   - group length 64 along a matrix's input dimension; per (row, group) one
 *     uint32 word with the bf16 scale in bits 0..15 and the bf16 bias in bits
 *     16..31; the dequantised weight is q * scale + bias with the unsigned
 *     code q in [0, 2^bits - 1];
 *   - codes: uint32 words, row-major; element k of a row is in word
 *     k / (32/bits) at bit offset bits * (k mod 32/bits), least significant
 *     bits first (8 nibbles or 16 two-bit codes per word);
 *   - an expert blob is [gate codes | gate scale/bias | up codes | up
 *     scale/bias | down codes | down scale/bias] with gate and up stored
 *     [inter][hidden] and down stored [hidden][inter]; see fmoe_blob_offsets().
 *   - Blobs must start on a 256-byte boundary.
 */
#ifndef FMOE_H
#define FMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fmoe_stream_t; /* same type as cudaStream_t */

enum {
  FMOE_OK = 0,
  FMOE_EINVAL = 1,  /* null pointer, unsupported size, bad alignment, wrong buffer size */
  FMOE_ENOMEM = 2,  /* caller-provided workspace (or output buffer) too small */
  FMOE_ECUDA = 3,   /* a CUDA runtime call or launch failed */
  FMOE_EDEVICE = 4  /* a kernel reported an error through the device status word */
};

#define FMOE_GROUP 64        /* quantisation group length */
#define FMOE_MAX_TOKENS 16   /* T limit of fmoe_route / fmoe_layer_decode */
#define FMOE_MAX_TOPK 8
#define FMOE_MAX_EXPERTS 1024
#define FMOE_MAX_HIDDEN 8192

/* Bytes of one packed expert: 3*hidden*inter*bits/8 code bytes plus 4 bytes
 * per group of 64 weights.  ([P1] "Técnicas innovadoras" item 1 and [P2]
 * "SSD-Experten-Streaming" give about 6.75 MB per 4-bit expert: this formula
 * gives 6.75 MiB = 7,077,888 bytes for hidden 4096, inter 1024, bits 4.)
 * Returns 0 for unsupported arguments (bits not 2 or 4, sizes not positive
 * multiples of 64). */
size_t fmoe_expert_bytes(int hidden, int inter, int bits);

/* Byte offsets of the six blob sections, written to off[6] in the order gate
 * codes, gate scale/bias, up codes, up scale/bias, down codes, down
 * scale/bias.  Returns FMOE_EINVAL for unsupported arguments or off == NULL. */
int fmoe_blob_offsets(int hidden, int inter, int bits, int64_t off[6]);

/* Quantise one expert from fp32 weights and pack it into blob_out.
 *   w_gate, w_up: [inter][hidden] fp32, row-major; w_down: [hidden][inter].
 *   bits: 4 or 2; group must be 64; hidden, inter: multiples of 64.
 *   blob_out: blob_bytes >= fmoe_expert_bytes(hidden, inter, bits), 256-byte
 *   aligned.
 * The pages do not describe their quantiser.  This one is affine min/max per
 * group in IEEE fp32, in this order: s = bf16(fl(fl(max - min) / (2^b - 1))),
 * bias = bf16(min), q = clamp(rint(fl(fl(w - bias) / s)), 0, 2^b - 1), q = 0
 * when s == 0; bf16 rounding is to nearest even.  Deterministic and
 * bit-reproducible.  Errors: FMOE_EINVAL, FMOE_ENOMEM (blob_bytes too small),
 * FMOE_ECUDA. */
int fmoe_quantize_expert(const float* w_gate, const float* w_up, const float* w_down, int hidden,
                         int inter, int bits, int group, void* blob_out, size_t blob_bytes,
                         fmoe_stream_t stream);

/* Workspace bytes needed by fmoe_route for T tokens and n_experts experts. */
size_t fmoe_route_workspace_bytes(int T, int n_experts);

/* Router for T tokens ([P2] "Pipeline-Leistung": router projection, then
 * softmax and top-K; [P2] "Technische Implementierung": K = 4 of 512).
 *   w_router: [n_experts][hidden] bf16 bit patterns (uint16), row-major.
 *   w_sgate:  [hidden] bf16 shared-gate vector, or NULL (then sgate = 1).
 *   x:        [T][hidden] fp32.
 *   idx:      [T][top_k] int32 out: selected experts, descending logit, lower
 *             index first on exact ties.
 *   w:        [T][top_k] fp32 out: softmax probabilities of the selected
 *             experts renormalised to sum to 1.
 *   sgate:    [T] fp32 out or NULL: sigmoid(w_sgate . x).
 *   logits_opt: [T][n_experts] fp32 out or NULL: router logits.
 *   ws:       device workspace, ws_bytes >= fmoe_route_workspace_bytes().
 * Limits: 1 <= T <= 16, 1 <= top_k <= min(8, n_experts), n_experts <= 1024,
 * hidden a multiple of 64 up to 8192.  Logits are fp32 dot products of the
 * bf16 weights (widened exactly) with fp32 x.
 * Errors: FMOE_EINVAL, FMOE_ENOMEM (workspace), FMOE_ECUDA. */
int fmoe_route(const uint16_t* w_router, const uint16_t* w_sgate, const float* x, int T, int hidden,
               int n_experts, int top_k, int32_t* idx, float* w, float* sgate, float* logits_opt,
               void* ws, size_t ws_bytes, fmoe_stream_t stream);

/* Workspace bytes needed by fmoe_expert_forward. */
size_t fmoe_expert_workspace_bytes(int hidden, int inter);

/* One expert for one token: y = Wd (silu(Wg x) * (Wu x)), where silu(z) =
 * z * sigmoid(z) ([P2] "Metal-Compute-Shader": dequantised matrix-vector
 * products and fused SwiGLU).
 *   blob: one packed expert (format above), 256-byte aligned.
 *   x: [hidden] fp32; y: [hidden] fp32 out (may not alias x).
 *   ws: device workspace of ws_bytes >= fmoe_expert_workspace_bytes(); it
 *   must be zero-filled before its first use (fmoe_workspace_init) and each
 *   call leaves it ready for the next.  Calls that share a workspace must be
 *   ordered on one stream.
 * Limits: hidden, inter multiples of 64; hidden <= 8192; inter <= 8192;
 * |x| below 2^100.  Errors: FMOE_EINVAL, FMOE_ENOMEM, FMOE_ECUDA. */
int fmoe_expert_forward(const void* blob, int hidden, int inter, int bits, const float* x, float* y,
                        void* ws, size_t ws_bytes, fmoe_stream_t stream);

/* One MoE layer. */
typedef struct {
  const uint16_t* w_router; /* [n_experts][hidden] bf16 bits */
  const uint16_t* w_sgate;  /* [hidden] bf16 bits, or NULL: shared expert ungated */
  const void* experts;      /* n_experts routed blobs; blob e at experts + e * expert_stride */
  int64_t expert_stride;    /* bytes, a multiple of 256, >= fmoe_expert_bytes(hidden, inter, bits) */
  const void* shared;       /* shared expert blob (shared_bits wide), or NULL: no shared expert */
  int hidden, inter, n_experts, top_k;
  int bits;                 /* routed experts: 4 or 2 */
  int shared_bits;          /* shared expert: 4 or 2 */
  int group;                /* must be 64 */
  /* Optional input normalisation (the "norm" that ends the previous layer's
   * step in [P2] "Verzögerte GPU-Experten-Berechnung", here fused into the
   * start of this layer): when norm_weight is non-NULL the experts and the
   * router see x / sqrt(mean(x^2) + norm_eps) * norm_weight instead of x; the
   * residual is used as given.  norm_weight: [hidden] bf16 bits, 16-byte
   * aligned; norm_eps: finite, >= 0 (1e-6 is usual). */
  const uint16_t* norm_weight;
  float norm_eps;
} fmoe_layer;

/* Workspace bytes needed by fmoe_layer_decode for T tokens. */
size_t fmoe_workspace_bytes(const fmoe_layer* L, int T);

/* Zero-fill a workspace (enqueued on stream).  Every workspace must be
 * zero-filled once before first use; fmoe_expert_forward and
 * fmoe_layer_decode leave it ready for the next call. */
int fmoe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream_t stream);

/* Decode T tokens through one MoE layer:
 *   out[t] = residual[t] + sum_k w[t][k] * E_{idx[t][k]}(x[t]) + sgate[t] * E_shared(x[t])
 * with routing as in fmoe_route and each expert as in fmoe_expert_forward
 * ([P2] "Metal-Compute-Shader": "MoE-Kombination + Rest + Sigmoid-Gate").
 *   x, residual, out: [T][hidden] fp32 (residual may be NULL: zero; out may
 *   alias residual but not x).
 *   idx_out_opt [T][top_k] int32, w_out_opt [T][top_k] fp32: optional copies
 *   of the routing decision.
 *   ws: workspace of ws_bytes >= fmoe_workspace_bytes(L, T), zero-filled
 *   before its first use; calls sharing a workspace must be stream-ordered.
 *   For T = 1 the workspace carries the launch epoch and the router logits
 *   and SwiGLU activations as words tagged with it; a workspace whose epoch
 *   is not one a launch leaves (not zero-filled) makes every wait of the next
 *   launch run out (reported, NaN results), after which it is usable again.
 * The whole layer runs on the GPU; the routing decision never returns to the
 * host.  T = 1 runs one persistent kernel.  T >= 2 groups the tokens by
 * expert: every distinct selected expert's weights are read once per call and
 * applied to each token that chose it, and the shared expert (every token)
 * runs on the tensor cores when hidden and inter are multiples of 512; each
 * token's result is the single-token result (same routing, outputs within
 * fp32 rounding).  Limits: as fmoe_route and fmoe_expert_forward, plus
 * (top_k + 1) * inter <= 10240.  Errors: FMOE_EINVAL, FMOE_ENOMEM, FMOE_ECUDA.
 * Kernel-side problems (a time-limited wait that ran out) are reported by
 * fmoe_get_status(); for T = 1 the kernel then also writes quiet NaN to the
 * out rows of every CTA whose wait ran out, hands NaN on to the rest through
 * any value it still publishes, and writes -1 / NaN to idx_out_opt /
 * w_out_opt when the routing itself was affected; for T >= 2 every unit of
 * work whose weight copy or tensor-core result did not arrive in time yields
 * NaN, which reaches the out rows of each token that uses it.  So no result
 * built on a missing value looks plausible. */
int fmoe_layer_decode(const fmoe_layer* L, const float* x, const float* residual, float* out, int T,
                      void* ws, size_t ws_bytes, int32_t* idx_out_opt, float* w_out_opt,
                      fmoe_stream_t stream);

/* The expert path of fmoe_layer_decode for one token with the routing given
 * instead of computed: out = residual + sum_k w_k * E_k(x) + shared_gate *
 * E_shared(x) ([P2] "Metal-Compute-Shader": the dequantised expert GEMVs, the
 * fused SwiGLU and the combine with the residual and the shared expert's
 * gate).  It serves experts that do not live in the layer's expert table:
 * the pages read each token's K selected experts from the SSD into memory
 * after routing ([P2] "SSD-Experten-Streaming"), and here a caller that
 * keeps experts in host memory routes with fmoe_route, copies the misses
 * into device slots (fmoe_cache_lookup) and decodes from the slots.
 *   L: shapes, code widths, the shared expert and the optional input norm
 *   (w_router, w_sgate, experts, expert_stride and n_experts are ignored;
 *   top_k is the number of routed experts).
 *   expert_blobs: HOST array of top_k device pointers, each a packed expert
 *   of L's shape and routed code width, 256-byte aligned (the same blob may
 *   appear twice).  expert_weights: HOST array of top_k combine weights (not
 *   renormalised here).  shared_gate: the shared expert's factor (1 for an
 *   ungated shared expert; ignored without a shared expert).
 *   x, residual, out, ws, ws_bytes: as fmoe_layer_decode with T = 1
 *   (ws_bytes >= fmoe_workspace_bytes(L, 1)).
 * Errors: FMOE_EINVAL, FMOE_ENOMEM, FMOE_ECUDA; kernel-side problems as
 * fmoe_layer_decode. */
int fmoe_experts_decode(const fmoe_layer* L, const void* const* expert_blobs, const float* expert_weights,
                        float shared_gate, const float* x, const float* residual, float* out, void* ws,
                        size_t ws_bytes, fmoe_stream_t stream);

/* fmoe_layer_decode without a caller-provided workspace, for callers that
 * cannot allocate device memory: code that runs where an allocator must not be
 * called (inside another library's fixed memory budget, or a host runtime that
 * hands over only the input and output buffers), or plain C callers with no
 * device allocator of their own.  The Flash-MoE pages have no counterpart:
 * this is an interface convenience of this library.
 *   Arguments, outputs and errors are those of fmoe_layer_decode, minus the
 *   workspace, for single-token decodes only: T must be 1 (FMOE_EINVAL
 *   otherwise; a grouped decode's workspace is far larger than the array).
 *   Every argument is checked before anything is enqueued, so a rejected
 *   call leaves the array untouched.  The workspace comes from one fixed
 *   128 KiB array in device memory that every GPU which loads the library
 *   keeps until the process exits; every layer that fmoe_layer_decode
 *   accepts fits it (a single-token workspace is 90,624 bytes whatever the
 *   shape), and FMOE_ENOMEM would report one that did not.
 *   The first call on a device looks the array's device address up (a
 *   synchronous runtime query); make that first call before capturing a
 *   stream into a graph.  Every call clears the array's hand-off counters and
 *   tagged words on `stream` before the layer kernel runs.
 *   All calls on a device share the one array: calls that may overlap on the
 *   GPU (different streams without ordering between them) race and give wrong
 *   results.  Nothing is allocated or freed by this call. */
int fmoe_layer_decode_noalloc(const fmoe_layer* L, const float* x, const float* residual, float* out, int T,
                              int32_t* idx_out_opt, float* w_out_opt, fmoe_stream_t stream);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device.  Returns FMOE_OK, FMOE_EDEVICE (a kernel reported a
 * problem; bits are in *bits_out if non-NULL) or FMOE_ECUDA. */
int fmoe_get_status(fmoe_stream_t stream, unsigned* bits_out);

/* The cudaError_t value of the most recent CUDA call that made an entry point
 * of this library return FMOE_ECUDA on the calling thread (0 if none). */
int fmoe_last_cuda_error(void);

/* Set the time limit of every device-side wait of the kernels launched after
 * this call (process-wide, all devices; default 2 s).  A wait that runs out
 * sets a bit of the device status word (see fmoe_get_status) and the kernel
 * carries on to its end without leaving its buffers, so the context stays
 * usable; the call's outputs are then undefined.  limit_ns must lie in
 * [1e6, 6e10] (1 ms .. 60 s), else FMOE_EINVAL and nothing changes.  The
 * previous limit is stored in *previous_opt when non-NULL.  The pages have no
 * counterpart: this is this library's watchdog.  Not synchronised with
 * launches in flight on other threads. */
int fmoe_set_wait_limit_ns(unsigned long long limit_ns, unsigned long long* previous_opt);

/* ---- Linear-attention state update (a second, independent decode step) ---- */

#define FMOE_DELTA_MAX_DIM 65536

/* Gated delta-rule update of a multi-head state for T tokens in turn, in
 * place, with the readout after each token.  Per head h and token t, in the
 * order of the routines the pages name for the GatedDeltaNet recurrence
 * (single-precision scale, matrix-vector and rank-1 update on a 64-head x
 * 128x128 state: [P2] "Accelerate-BLAS für lineare Aufmerksamkeit", [P3]
 * "Uso do Accelerate BLAS"):
 *   S_h <- alpha[t][h] * S_h
 *   u   <- S_h k[t][h]
 *   S_h <- S_h + beta[t][h] * (v[t][h] - u) k[t][h]^T
 *   o[t][h] <- S_h q[t][h]
 * i.e. S' = alpha S (I - beta k k^T) + beta v k^T, o = S' q.  How q, k, v and
 * the gates are produced from a token is outside this call.
 *   state: device [heads][dv][dk] fp32 (row i of a head: the dk key
 *          coefficients of value i), read and written once per call.
 *   q, k: device [T][heads][dk] fp32; v: [T][heads][dv]; alpha, beta:
 *          [T][heads]; o: device [T][heads][dv] fp32 out.
 * Arithmetic in fp32 (the state stays fp32 between tokens).  Limits: dk in
 * {128, 256, 384, 512}; 1 <= heads, dv, T <= FMOE_DELTA_MAX_DIM; state, q, k
 * 16-byte aligned, the rest 4-byte aligned; state and o may not overlap each
 * other or any input.  Errors: FMOE_EINVAL, FMOE_ECUDA.  Nothing is
 * allocated. */
int fmoe_delta_update(float* state, const float* q, const float* k, const float* v, const float* alpha,
                      const float* beta, float* o, int heads, int dk, int dv, int T, fmoe_stream_t stream);

/* ---- Expert cache directory (host side of streaming non-resident experts) ---- */

#define FMOE_CACHE_MAX_SLOTS (1 << 20)

/* The pages read each layer's K selected experts from the SSD on demand and
 * let the operating system's page cache, a least-recently-used cache, hold
 * them (~71 % hits: [P1] "Técnicas innovadoras" §1, [P2]
 * "SSD-Experten-Streaming", [P3] "Trust the OS").  The B200 analogue keeps
 * the experts in pinned host memory and a pool of n_slots device slots (one
 * expert blob each) as the cache.  This opaque directory decides, per layer
 * call, which selected experts are already in a slot and which slot each miss
 * goes to: never-used slots first (lowest index first), then the least
 * recently used slot over all layers.  It is host-only: it moves no data and
 * makes no CUDA call (copying a miss's blob into its slot is the caller's).
 * Not thread-safe: one directory per thread, or the caller's lock. */
typedef struct fmoe_expert_cache_s fmoe_expert_cache;

/* A directory of n_slots slots, all free.  1 <= n_slots <=
 * FMOE_CACHE_MAX_SLOTS; *cache_out is set (NULL on error).  Errors:
 * FMOE_EINVAL, FMOE_ENOMEM. */
int fmoe_cache_create(int n_slots, fmoe_expert_cache** cache_out);

/* Free a directory (NULL is accepted).  Returns FMOE_OK. */
int fmoe_cache_destroy(fmoe_expert_cache* cache);

/* For the K experts idx[0..K) selected in `layer` (host arrays): slot_out[k]
 * is the expert's slot and miss_out[k] is 1 when its blob must be copied in
 * (0 when it is there already); *n_miss_out (optional) counts the misses.
 * The touched entries become the most recently used, in k order; an expert
 * listed twice takes one slot (its second listing is a hit).  Requires
 * layer >= 0, idx[k] >= 0 and 1 <= K <= n_slots (so that no slot of this call
 * is evicted by it).  Errors: FMOE_EINVAL, FMOE_ENOMEM. */
int fmoe_cache_lookup(fmoe_expert_cache* cache, int layer, const int32_t* idx, int K, int32_t* slot_out,
                      int32_t* miss_out, int* n_miss_out);

/* Running totals since creation or the last reset (each pointer optional). */
int fmoe_cache_stats(const fmoe_expert_cache* cache, uint64_t* hits, uint64_t* misses, uint64_t* evictions);

/* Empty the directory (all slots free) and zero the totals. */
int fmoe_cache_reset(fmoe_expert_cache* cache);

/* ---- Routed experts streamed from host memory ------------------------------
 * The B200 counterpart of the pages' expert streaming ([P2] "SSD-Experten-
 * Streaming": only the K active experts of a layer are read, on demand, and
 * the OS page cache keeps the recently used ones, an LRU with ~71 % hits;
 * [P2] "Verzögerte GPU-Experten-Berechnung": the expert command is queued
 * without waiting).  The routed experts of every layer stay in page-locked
 * host memory; n_slots device slots hold the recently used ones (an
 * fmoe_expert_cache directory over (layer, expert)).  Per layer and token,
 * fmoe_streamer_decode:
 *   1. runs the router GEMV and top-K on the GPU (as fmoe_route) and copies
 *      the decision to the host, the one synchronisation of the call;
 *   2. looks the K experts up in the directory and copies every miss from
 *      host memory into its slot, one cudaMemcpyAsync each, on copy_stream;
 *   3. meanwhile decodes the shared expert and the hits on stream
 *      (out = residual + sum over hits + gated shared expert), then, once the
 *      copies have landed, adds the misses with a second launch.
 * It returns once these are queued; the result is that of fmoe_layer_decode
 * within fp32 rounding (same routing, a different summation order). */
typedef struct fmoe_streamer_s fmoe_streamer;

/* layers[0..n_layers): w_router, w_sgate, shared, shapes and code widths as
 * for fmoe_layer_decode, all with the same hidden, inter, n_experts, top_k,
 * bits and expert_stride, no norm_weight (the router reads x as given); the
 * `experts` field is ignored.  host_experts[l]: page-locked host memory
 * (cudaHostAlloc, or registered), 256-byte aligned, holding layer l's
 * n_experts blobs at expert_stride.  slots: device memory of n_slots *
 * expert_stride bytes, 256-byte aligned, top_k <= n_slots <=
 * FMOE_CACHE_MAX_SLOTS.  All stay owned by the caller and must outlive the
 * streamer.  *out is set (NULL on error).  Errors: FMOE_EINVAL (also for
 * host memory that is not page-locked), FMOE_ENOMEM, FMOE_ECUDA. */
int fmoe_streamer_create(const fmoe_layer* layers, int n_layers, const void* const* host_experts, void* slots,
                         int n_slots, fmoe_streamer** out);

/* Decode one token through layer `layer` (see above).  x, residual, out, ws,
 * ws_bytes: as fmoe_layer_decode with T = 1.  stream: the compute stream;
 * copy_stream: the stream of the host-to-device copies (may equal stream:
 * no overlap then).  Every decode of a streamer must use the same stream (a
 * slot is overwritten only after the kernels that read it, which that stream
 * orders).  The call synchronises `stream` once, so it cannot be captured
 * into a graph.  idx_out_opt, w_out_opt: optional HOST arrays [top_k] that
 * receive the routing decision.  No layer may be prepared and unfinished
 * (see fmoe_streamer_prepare).  Errors: FMOE_EINVAL, FMOE_ENOMEM,
 * FMOE_ECUDA; kernel-side problems as fmoe_layer_decode. */
int fmoe_streamer_decode(fmoe_streamer* s, int layer, const float* x, const float* residual, float* out, void* ws,
                         size_t ws_bytes, fmoe_stream_t stream, fmoe_stream_t copy_stream, int32_t* idx_out_opt,
                         float* w_out_opt);

/* fmoe_streamer_decode in two halves, for callers that know the next layer's
 * input before this layer's decode is done (independent layer inputs): a
 * layer prepared while the previous one decodes copies its misses during
 * that decode ([P2] "Verzögerte GPU-Experten-Berechnung": the host prepares
 * the next layer while the GPU computes).
 * fmoe_streamer_prepare: steps 1 and 2 for `layer` and its input x (device,
 * ready on route_stream): the routing kernels on route_stream, the decision
 * to the host (synchronises route_stream), the directory lookup and the
 * misses' copies on copy_stream, each after the last decode that read its
 * slot.  At most two layers may be prepared and not yet finished, and a
 * second one needs n_slots >= 2 * top_k (so that it cannot evict the first
 * one's experts).  idx_out_opt, w_out_opt: optional HOST arrays [top_k].
 * fmoe_streamer_finish: step 3 for the oldest prepared layer (`layer` must
 * be it; x the same input), on stream; it returns once the launches are
 * queued.  Use one copy stream for all calls of a streamer.  Errors:
 * FMOE_EINVAL (including a call out of order), FMOE_ENOMEM, FMOE_ECUDA. */
int fmoe_streamer_prepare(fmoe_streamer* s, int layer, const float* x, fmoe_stream_t route_stream,
                          fmoe_stream_t copy_stream, int32_t* idx_out_opt, float* w_out_opt);
int fmoe_streamer_finish(fmoe_streamer* s, int layer, const float* x, const float* residual, float* out, void* ws,
                         size_t ws_bytes, fmoe_stream_t stream);

/* Running totals: expert hits and misses (the directory's) and bytes copied
 * from host to device (each pointer optional). */
int fmoe_streamer_stats(const fmoe_streamer* s, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes);

/* Free a streamer (NULL is accepted); the caller's memory is untouched.
 * Returns FMOE_OK. */
int fmoe_streamer_destroy(fmoe_streamer* s);

/* How the single-token layer kernel (fmoe_layer_decode with T = 1,
 * fmoe_layer_decode_noalloc with T = 1, fmoe_expert_forward) is launched,
 * process-wide, for the calls made after this one.
 *   1 (default): programmatic dependent launch.  The grid may start while the
 *     previous kernel on the stream finishes: each CTA sets up its barriers
 *     and copies its share of the router weights before it waits for that
 *     kernel, and reads no input, output or workspace byte before.  Back-to-
 *     back layer decodes overlap one's start with the other's end.  The
 *     kernel's grid barriers need all of its CTAs resident at once; a plain
 *     launch does not promise that, so it is made only when one CTA fits on
 *     every SM (else FMOE_EINVAL), and a grid that other work keeps from
 *     becoming resident ends with a bounded-wait status bit (see
 *     fmoe_set_wait_limit_ns) instead of results.
 *   0: cooperative launch, all CTAs resident by the driver's guarantee, no
 *     overlap with the previous kernel.
 * The same setting governs the kernels of the grouped decode
 * (fmoe_layer_decode with T >= 2): with 1 each of them is a programmatic
 * dependent launch that waits for the previous kernel before its first
 * access of device memory (no grid barriers, so no residency condition);
 * with 0 they are plain launches.
 * Outputs are bit-identical either way.  enable must be 0 or 1, else
 * FMOE_EINVAL and nothing changes; the previous setting is stored in
 * *previous_opt when non-NULL.  The pages have no counterpart: launch
 * mechanics of this library.  Not synchronised with launches in flight on
 * other threads. */
int fmoe_set_dependent_launch(int enable, int* previous_opt);

/* Static, human-readable text for an error code. */
const char* fmoe_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_H */
