// Device implementation of the synthetic input recipes (see synth/gen.py for
// the definition).  Every floating-point step is an individually rounded fp32
// operation (__fadd_rn / __fmul_rn / __fdiv_rn: no contraction into FMA), so
// the output is bit-identical to the NumPy implementation.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint32_t kTag = 7;
constexpr uint32_t kSubTarget = 0, kSubDraft = 1, kSubRot = 2, kSubHead = 3, kSubDraftToken = 4;

struct Words4 { uint32_t w[4]; };

__device__ __forceinline__ Words4 philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                         uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c1 = (uint32_t)p1;
    c3 = (uint32_t)p0;
    c0 = n0;
    c2 = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  Words4 o;
  o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
  return o;
}

__device__ __forceinline__ uint32_t word_at(uint64_t seed, uint32_t row, uint32_t sub, uint32_t pos) {
  Words4 o = philox(pos >> 2, row, sub, kTag, (uint32_t)seed, (uint32_t)(seed >> 32));
  return o.w[pos & 3];
}

__device__ __forceinline__ float normal_from_word(uint32_t w, const float* __restrict__ table) {
  const uint32_t i = w >> 20;
  const float f = __fmul_rn((float)(w & 0xFFFFFu), 9.5367431640625e-07f);  // 2^-20
  const float t0 = table[i];
  const float d = __fsub_rn(table[i + 1], t0);
  return __fadd_rn(t0, __fmul_rn(d, f));
}

__device__ __forceinline__ uint16_t bf16_rne_bits(float x) {
  const uint32_t b = __float_as_uint(x);
  return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__device__ __forceinline__ float synth_log(float x) {
  const uint32_t bits = __float_as_uint(x);
  int e = (int)(bits >> 23) - 127;
  float m = __uint_as_float((bits & 0x7FFFFFu) | 0x3F800000u);
  if (m > 1.41421356f) { m = __fmul_rn(m, 0.5f); e += 1; }
  const float s = __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f));
  const float s2 = __fmul_rn(s, s);
  float p = 2.0f / 9.0f;
  p = __fadd_rn(__fmul_rn(p, s2), 2.0f / 7.0f);
  p = __fadd_rn(__fmul_rn(p, s2), 2.0f / 5.0f);
  p = __fadd_rn(__fmul_rn(p, s2), 2.0f / 3.0f);
  p = __fadd_rn(__fmul_rn(p, s2), 2.0f);
  return __fadd_rn(__fmul_rn((float)e, 0.693147182f), __fmul_rn(s, p));
}

__device__ __forceinline__ float synth_gumbel(uint32_t w) {
  const float u = __fmul_rn(__fadd_rn((float)(w >> 9), 0.5f), 1.1920928955078125e-07f);  // 2^-23
  const float t = -synth_log(u);
  return -synth_log(t);
}

// One block per target row id.  Writes the target row (if target != null) and
// the paired draft row (if draft != null and the row has one).
__global__ void synth_rows_kernel(uint64_t seed, int bf16, int64_t nrows, int V, int64_t ld,
                                  float sigma_z, int L, const float* __restrict__ boosts,
                                  const float* __restrict__ table,
                                  const float* __restrict__ sigma_d_seq, int R, int Kd,
                                  void* target, void* draft) {
  __shared__ int head_pos[64];
  __shared__ int head_rank[64];
  const int64_t id = blockIdx.x;
  if (id >= nrows) return;
  const int bs = L > 0 ? V / L : 1;
  if (threadIdx.x < (unsigned)L) {
    const uint32_t rot = word_at(seed, (uint32_t)id, kSubRot, 0) % (uint32_t)L;
    const uint32_t off = word_at(seed, (uint32_t)id, kSubHead, threadIdx.x) % (uint32_t)bs;
    head_pos[threadIdx.x] = (int)threadIdx.x * bs + (int)off;
    head_rank[threadIdx.x] = (int)((threadIdx.x + rot) % (uint32_t)L);
  }
  __syncthreads();
  const int64_t seq = id / R;
  const int k = (int)(id % R);
  const bool has_draft = draft != nullptr && k < Kd;
  const float sd = (has_draft && sigma_d_seq) ? sigma_d_seq[seq] : 0.0f;
  const int64_t drow = seq * Kd + k;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    float zt = __fmul_rn(sigma_z, normal_from_word(word_at(seed, (uint32_t)id, kSubTarget, v), table));
    if (L > 0) {
      const int j = v / bs;
      if (j < L && head_pos[j] == v) zt = __fadd_rn(zt, boosts[head_rank[j]]);
    }
    if (target) {
      if (bf16) reinterpret_cast<uint16_t*>(target)[id * ld + v] = bf16_rne_bits(zt);
      else reinterpret_cast<float*>(target)[id * ld + v] = zt;
    }
    if (has_draft) {
      const float n2 = normal_from_word(word_at(seed, (uint32_t)id, kSubDraft, v), table);
      const float zd = __fadd_rn(zt, __fmul_rn(sd, n2));
      if (bf16) reinterpret_cast<uint16_t*>(draft)[drow * ld + v] = bf16_rne_bits(zd);
      else reinterpret_cast<float*>(draft)[drow * ld + v] = zd;
    }
  }
}

// One block per drafted token: unit u, position k < K reads draft row u*Kd + k
// (generator row id u*R + k) and writes tokens[u*K + k].
__global__ void synth_draft_tokens_kernel(uint64_t seed, int bf16, int64_t ntok, int K, int R, int Kd,
                                          int V, int64_t ld, float inv_tau, const void* draft,
                                          int32_t* tokens) {
  __shared__ float best_s[32];
  __shared__ int best_i[32];
  const int64_t j = blockIdx.x;
  if (j >= ntok) return;
  const int64_t unit = j / K;
  const int k = (int)(j % K);
  const uint32_t id = (uint32_t)(unit * R + k);
  const int64_t row = unit * Kd + k;
  float bs = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    float z;
    if (bf16) z = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(draft)[row * ld + v] << 16);
    else z = reinterpret_cast<const float*>(draft)[row * ld + v];
    const float s = __fadd_rn(__fmul_rn(z, inv_tau), synth_gumbel(word_at(seed, id, kSubDraftToken, v)));
    if (s > bs) { bs = s; bi = v; }   // v increases per thread: first max kept
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float os = __shfl_xor_sync(0xffffffffu, bs, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (os > bs || (os == bs && oi < bi)) { bs = os; bi = oi; }
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) { best_s[w] = bs; best_i[w] = bi; }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    bs = l < nw ? best_s[l] : -INFINITY;
    bi = l < nw ? best_i[l] : 0x7FFFFFFF;
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (os > bs || (os == bs && oi < bi)) { bs = os; bi = oi; }
    }
    if (l == 0) tokens[j] = bi;
  }
}

}  // namespace

extern "C" int synth_rows(uint64_t seed, int bf16, int64_t nrows, int V, int64_t ld, float sigma_z,
                          int L, const float* boosts, const float* table, const float* sigma_d_seq,
                          int R, int Kd, void* target, void* draft, void* stream) {
  if (nrows <= 0) return 0;
  if (L > 64 || V < 1 || ld < V || R < 1) return 1;
  synth_rows_kernel<<<(unsigned)nrows, 256, 0, (cudaStream_t)stream>>>(
      seed, bf16, nrows, V, ld, sigma_z, L, boosts, table, sigma_d_seq, R, Kd, target, draft);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int synth_draft_tokens(uint64_t seed, int bf16, int64_t ntok, int K, int R, int Kd, int V,
                                  int64_t ld, float inv_tau, const void* draft, int32_t* tokens,
                                  void* stream) {
  if (ntok <= 0) return 0;
  if (K < 1 || V < 1 || ld < V) return 1;
  synth_draft_tokens_kernel<<<(unsigned)ntok, 512, 0, (cudaStream_t)stream>>>(
      seed, bf16, ntok, K, R, Kd, V, ld, inv_tau, draft, tokens);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
