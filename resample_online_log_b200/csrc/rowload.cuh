// Reading logit rows (bf16 bit patterns or fp32) in 16-byte chunks, and the
// CTA-wide k-th largest of one value per thread: shared by the dense row
// kernels that select top entries (Gumbel-top-k, n-gram observations).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

// Order-preserving map of floats to signed ints (for atomicMax on a threshold).
__device__ __forceinline__ int f2ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

template <typename TIn>
__device__ __forceinline__ float ld_elem(const TIn* p, int i);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p, int i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_elem<uint16_t>(const uint16_t* p, int i) {
  return __uint_as_float((uint32_t)p[i] << 16);
}

// Eight consecutive entries of a row (one 16-byte chunk of bf16, two of fp32)
// as floats; entries at or past V read as -inf.  `hint` is the L2 policy of
// the vector loads.  The raw form (load8_raw, then unpack8) lets a thread keep
// several chunks in flight.
template <typename TIn>
__device__ __forceinline__ void load8(const TIn* row, int v0, int V, bool vec, uint64_t hint,
                                      float* z);
template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* row, int v0, int V, bool vec,
                                                uint64_t hint, float* z) {
  if (vec && v0 + 8 <= V) {
    const uint4 u = ldg_hint(row + v0, hint);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      z[2 * j] = __uint_as_float(w[j] << 16);
      z[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) z[j] = v0 + j < V ? ld_elem<uint16_t>(row, v0 + j) : -INFINITY;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* row, int v0, int V, bool vec,
                                             uint64_t hint, float* z) {
  if (vec && v0 + 8 <= V) {
    const uint4 a = ldg_hint(row + v0, hint), b = ldg_hint(row + v0 + 4, hint);
    z[0] = __uint_as_float(a.x); z[1] = __uint_as_float(a.y);
    z[2] = __uint_as_float(a.z); z[3] = __uint_as_float(a.w);
    z[4] = __uint_as_float(b.x); z[5] = __uint_as_float(b.y);
    z[6] = __uint_as_float(b.z); z[7] = __uint_as_float(b.w);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) z[j] = v0 + j < V ? row[v0 + j] : -INFINITY;
  }
}

template <typename TIn>
struct Raw8 {
  uint4 a, b;  // bf16: a only
};
template <typename TIn>
__device__ __forceinline__ Raw8<TIn> load8_raw(const TIn* row, int v0, int V, bool vec,
                                               uint64_t hint) {
  Raw8<TIn> r;
  if (vec && v0 + 8 <= V) {
    r.a = ldg_hint(row + v0, hint);
    if (sizeof(TIn) == 4) r.b = ldg_hint(row + v0 + 4, hint);
  } else {
    float zz[8];
    load8<TIn>(row, v0, V, false, hint, zz);
    if (sizeof(TIn) == 2) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = (__float_as_uint(zz[2 * j]) >> 16) | (__float_as_uint(zz[2 * j + 1]) & 0xFFFF0000u);
      r.a = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      r.a = make_uint4(__float_as_uint(zz[0]), __float_as_uint(zz[1]), __float_as_uint(zz[2]),
                       __float_as_uint(zz[3]));
      r.b = make_uint4(__float_as_uint(zz[4]), __float_as_uint(zz[5]), __float_as_uint(zz[6]),
                       __float_as_uint(zz[7]));
    }
  }
  return r;
}
template <typename TIn>
__device__ __forceinline__ void unpack8(const Raw8<TIn>& r, float* z) {
  if (sizeof(TIn) == 2) {
    const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      z[2 * j] = __uint_as_float(w[j] << 16);
      z[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    z[0] = __uint_as_float(r.a.x); z[1] = __uint_as_float(r.a.y);
    z[2] = __uint_as_float(r.a.z); z[3] = __uint_as_float(r.a.w);
    z[4] = __uint_as_float(r.b.x); z[5] = __uint_as_float(r.b.y);
    z[6] = __uint_as_float(r.b.z); z[7] = __uint_as_float(r.b.w);
  }
}
// The k-th largest of one value per thread of the CTA (-inf if fewer than k
// are finite): k rounds of warp maxima, each removing one winning lane, then
// the same over the warps' k best.
static __device__ __noinline__ float cta_kth_largest(float v, int k, float* buf /* [nwarps * k] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = 0; r < k; ++r) {
    float w = v;
    asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(w));
    const unsigned hit = __ballot_sync(0xffffffffu, v == w && w > -INFINITY);
    if (hit && lane == __ffs(hit) - 1) v = -INFINITY;
    if (lane == 0) buf[warp * k + r] = hit ? w : -INFINITY;
  }
  __syncthreads();
  float res = -INFINITY;
  if (warp == 0) {
    const int n = nw * k;  // <= 16 * 16: at most 8 per lane
    float h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = lane + 32 * i < n ? buf[lane + 32 * i] : -INFINITY;
    for (int r = 0; r < k; ++r) {
      float m = h[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) m = fmaxf(m, h[i]);
      float w = m;
      asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(w));
      const unsigned hit = __ballot_sync(0xffffffffu, m == w && w > -INFINITY);
      if (hit && lane == __ffs(hit) - 1) {
        bool done = false;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (!done && h[i] == w) {
            h[i] = -INFINITY;
            done = true;
          }
      }
      res = hit ? w : -INFINITY;
    }
    if (lane == 0) buf[0] = res;
  }
  __syncthreads();
  res = buf[0];
  __syncthreads();
  return res;
}

}  // namespace smcsd
