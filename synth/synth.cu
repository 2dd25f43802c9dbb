// Seeded synthetic expert weights drawn directly in device memory.
//
// This is input generation only (no dequantisation, GEMV or routing).  It is
// the device twin of synth/__init__.py: code words are the high 32 bits of
// output i of SplitMix64 (Steele, Lea and Flood, OOPSLA 2014; output mix with
// the constants of Vigna's public-domain splitmix64.c) seeded with a key that
// chains (tag, seed, layer, expert, matrix); (scale, bias) pairs are drawn from
// one output per group with fp32 IEEE operations in a fixed order and
// round-to-nearest-even bf16 conversion.  The test suite checks byte equality
// against the NumPy twin.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kTagCodes = 0xC0DE5ull;
constexpr uint64_t kTagSb = 0x5CA1Eull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t tag, uint64_t seed, uint64_t layer,
                                               uint64_t expert, uint64_t matrix) {
  uint64_t k = 0;
  k = mix64((k ^ tag) + kGamma);
  k = mix64((k ^ seed) + kGamma);
  k = mix64((k ^ layer) + kGamma);
  k = mix64((k ^ expert) + kGamma);
  k = mix64((k ^ matrix) + kGamma);
  return k;
}

__device__ inline uint64_t sm_output(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1ull) * kGamma);
}

__device__ inline uint32_t bf16_rne_bits(float f) {
  uint32_t u = __float_as_uint(f);
  return (uint32_t)(((uint64_t)u + 0x7FFFull + ((u >> 16) & 1u)) >> 16) & 0xFFFFu;
}

struct FillArgs {
  char* dst;
  long long stride;       // bytes between consecutive experts in dst
  long long off[6];       // byte offsets: gate codes, gate sb, up codes, up sb, down codes, down sb
  int first_expert;       // expert id of dst's first expert
  int n_experts;
  int hidden, inter, bits;
  unsigned long long seed;
  int layer;
  int expert_id_override; // >= 0: use this id for every expert (shared expert)
};

__global__ void fill_experts_kernel(FillArgs a) {
  const int em = blockIdx.y;                 // expert-local * 3 + matrix
  const int e_local = em / 3;
  const int m = em % 3;
  const int rows = (m < 2) ? a.inter : a.hidden;
  const int nin = (m < 2) ? a.hidden : a.inter;
  const long long eid = a.expert_id_override >= 0 ? a.expert_id_override
                                                  : (long long)(a.first_expert + e_local);
  char* base = a.dst + (long long)e_local * a.stride;
  const uint64_t kc = stream_key(kTagCodes, a.seed, (uint64_t)a.layer, (uint64_t)eid, (uint64_t)m);
  const uint64_t ks = stream_key(kTagSb, a.seed, (uint64_t)a.layer, (uint64_t)eid, (uint64_t)m);
  uint32_t* codes = reinterpret_cast<uint32_t*>(base + a.off[2 * m]);
  uint32_t* sb = reinterpret_cast<uint32_t*>(base + a.off[2 * m + 1]);
  const long long n_words = (long long)rows * nin * a.bits / 32;
  const long long n_groups = (long long)rows * (nin / 64);
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long i = tid; i < n_words; i += nthreads)
    codes[i] = (uint32_t)(sm_output(kc, (uint64_t)i) >> 32);
  const float two24 = 1.0f / 16777216.0f;
  const float c3e3 = __uint_as_float(0x3b449ba6u);
  const float c1e3 = __uint_as_float(0x3a83126fu);
  const float c02 = __uint_as_float(0x3e4ccccdu);
  const float c09 = __uint_as_float(0x3f666666u);
  const float negm = (a.bits == 4) ? -8.0f : -1.5f;
  for (long long i = tid; i < n_groups; i += nthreads) {
    const uint64_t h = sm_output(ks, (uint64_t)i);
    const float u = __fmul_rn((float)(uint32_t)(h >> 40), two24);
    const float u2 = __fmul_rn((float)(uint32_t)((h >> 16) & 0xFFFFFFull), two24);
    const float s32 = __fadd_rn(__fmul_rn(c3e3, u), c1e3);
    const uint32_t sbits = bf16_rne_bits(s32);
    const float sf = __uint_as_float(sbits << 16);
    const float fac = __fadd_rn(__fmul_rn(c02, u2), c09);
    const float b32 = __fmul_rn(__fmul_rn(negm, sf), fac);
    const uint32_t bbits = bf16_rne_bits(b32);
    sb[i] = sbits | (bbits << 16);
  }
}

}  // namespace

extern "C" {

// Fill n_experts consecutive expert blobs at dst (device), blob e at dst + e*stride,
// with the seeded synthetic codes and (scale, bias) words.  off[6] gives each
// section's byte offset inside a blob.  expert_id_override >= 0 draws every blob
// from that expert id's streams (used for the shared expert).  Returns a
// cudaError_t value (0 on success).
int synth_fill_experts(void* dst, long long stride, const long long* off, int first_expert,
                       int n_experts, int hidden, int inter, int bits,
                       unsigned long long seed, int layer, int expert_id_override,
                       cudaStream_t stream) {
  if (!dst || !off || n_experts <= 0 || (bits != 2 && bits != 4) || hidden % 64 || inter % 64)
    return (int)cudaErrorInvalidValue;
  FillArgs a;
  a.dst = static_cast<char*>(dst);
  a.stride = stride;
  for (int i = 0; i < 6; ++i) a.off[i] = off[i];
  a.first_expert = first_expert;
  a.n_experts = n_experts;
  a.hidden = hidden;
  a.inter = inter;
  a.bits = bits;
  a.seed = seed;
  a.layer = layer;
  a.expert_id_override = expert_id_override;
  long long words = (long long)hidden * inter * bits / 32;
  int bx = (int)((words + 256LL * 64 - 1) / (256LL * 64));
  if (bx < 1) bx = 1;
  if (bx > 4096) bx = 4096;
  // blockIdx.y is limited to 65535: launch in slices of experts.
  for (int e0 = 0; e0 < n_experts; e0 += 20000) {
    int ne = n_experts - e0 < 20000 ? n_experts - e0 : 20000;
    FillArgs s = a;
    s.dst = a.dst + (long long)e0 * stride;
    s.first_expert = first_expert + e0;
    s.n_experts = ne;
    dim3 grid(bx, ne * 3);
    fill_experts_kernel<<<grid, 256, 0, stream>>>(s);
  }
  return (int)cudaGetLastError();
}

}  // extern "C"
