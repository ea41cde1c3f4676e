// Pieces shared by the logit-row kernels of libsmcsd.so (SMC-SD scoring and
// standard verification): the launch arguments, element access for bf16 /
// fp32 rows, Gumbel-max candidates with fp32 error bounds, (max, sum)
// partial combination and the host-side cluster launch helpers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

constexpr int kMaxWarps = 16;    // producer warps of one CTA (one lane each in a half-warp)
constexpr int kMaxCluster = 16;  // non-portable cluster size limit
constexpr int kEPT = 32;         // entries of each row a producer thread holds per row

struct ScoreArgs {
  const void* zT;
  const void* zD;
  int64_t ld;
  int V, K, R;
  int64_t units;
  int slice;             // entries per slice (a multiple of 8)
  int groups;            // independent warp groups per CTA
  int stages;            // ring stages
  uint32_t stage_bytes;  // bytes reserved for one tensor's slice in a stage
  int use_tma;
  float inv_tau, cT;     // 1/tau and log2(e)/tau, fp32
  double tau64, inv_tau64;
  const int32_t* draft;  // [units, K]
  uint64_t seed, round;
  const double* logw_prev;
  const double* log_potential;
  double* logw_out;
  float* tv_out;
  int32_t* bonus_out;
  int32_t* tokens_out;
  double* lse_out;
  double* lp_out;
  int32_t* acc_len;
  int32_t* out_tokens;
  uint32_t* dev_err;
};

// One slice's message for one row, pushed into every CTA of the cluster.
struct alignas(16) Msg {
  float mT, sT, mD, sD;  // (reference, sum of exps relative to it) over the slice of each row
  float zxT, zxD;        // raw logits of the draft token (owner slice only)
  float tvprev;          // a TV partial of the sender's previous row (verify)
  int aux;               // argmax entry of the sender's target slice (verify)
};

// ------------------------------------------------------------------ Gumbel-max candidates
// A screening partial: best point score, its fp32 bounds, and the largest
// upper bound of every other kept entry.  When that bound stays below the
// best's lower bound the winner is exact; otherwise it is settled in fp64.
struct Cand {
  float s, lo, hi, ohi;
  int idx, aux, pad1, pad2;  // aux: a value that travels with the candidate (-1: none)
};

struct Cand64 {
  double s;
  int idx, pad;
};

__device__ __forceinline__ Cand cand_empty() {
  Cand c;
  c.s = -INFINITY;
  c.lo = -INFINITY;
  c.hi = -INFINITY;
  c.ohi = -INFINITY;
  c.idx = 0x7FFFFFFF;
  c.aux = -1;
  c.pad1 = c.pad2 = 0;
  return c;
}
__device__ __forceinline__ Cand cand_merge(const Cand& a, const Cand& b) {
  const bool aw = a.s > b.s || (a.s == b.s && a.idx < b.idx);
  Cand w = aw ? a : b;
  const Cand& l = aw ? b : a;
  w.ohi = fmaxf(w.ohi, fmaxf(l.hi, l.ohi));
  return w;
}
__device__ __forceinline__ Cand cand_shfl(const Cand& c, int o) {
  Cand r;
  r.s = __shfl_xor_sync(0xffffffffu, c.s, o);
  r.lo = __shfl_xor_sync(0xffffffffu, c.lo, o);
  r.hi = __shfl_xor_sync(0xffffffffu, c.hi, o);
  r.ohi = __shfl_xor_sync(0xffffffffu, c.ohi, o);
  r.idx = __shfl_xor_sync(0xffffffffu, c.idx, o);
  r.aux = __shfl_xor_sync(0xffffffffu, c.aux, o);
  r.pad1 = r.pad2 = 0;
  return r;
}
__device__ __forceinline__ Cand warp_cand(Cand c) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c = cand_merge(c, cand_shfl(c, o));
  return c;
}
__device__ __forceinline__ void c64_merge(double& s, int& i, double os, int oi) {
  if (os > s || (os == s && oi < i)) {
    s = os;
    i = oi;
  }
}
__device__ __forceinline__ void warp_c64(double& s, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double os = __shfl_xor_sync(0xffffffffu, s, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    c64_merge(s, i, os, oi);
  }
}

// fp32 error bound of a score a32 + g32 (a32 = z * (1/tau) rounded, g32 from
// CUDA's logf / log1pf): contains the exact fp64 score.
__device__ __forceinline__ float score_err(float a32, float g32) {
  return 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
}

// Candidate from one kept entry with a = z / tau in fp32.
static __device__ __noinline__ Cand bonus_cand_a(float a32, float u, int v) {
  const float g32 = gumbel_f32(u);
  Cand cd;
  cd.s = a32 + g32;
  const float d = score_err(a32, g32);
  cd.lo = cd.s - d;
  cd.hi = cd.s + d;
  cd.ohi = -INFINITY;
  cd.idx = v;
  cd.aux = -1;
  cd.pad1 = cd.pad2 = 0;
  return cd;
}

constexpr float kYSkip = 5.88e-8f;  // < e^{-g_max}: even g_max cannot lift the entry to Tref

// With y = e^{a - Tref} (Tref a lower bound on the winning score), u <= 1 - y
// proves g <= Tref - a (e^{-y} >= 1 - y): the entry cannot win.  Rounding
// margins keep the test conservative.
__device__ __forceinline__ bool keep_bonus(float y, float u) {
  return y > 0.f && !(u < (1.0f - y * 1.001f) - 2.4e-7f);
}

// ------------------------------------------------------------------ element access
template <typename TIn>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float get(const float* p, int64_t i) { return p[i]; }
  static __device__ __forceinline__ void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};
template <>
struct Elem<uint16_t> {  // bf16 bit patterns
  static __device__ __forceinline__ float get(const uint16_t* p, int64_t i) {
    return __uint_as_float((uint32_t)p[i] << 16);
  }
  static __device__ __forceinline__ void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x << 16);
    o[1] = __uint_as_float(v.x & 0xFFFF0000u);
    o[2] = __uint_as_float(v.y << 16);
    o[3] = __uint_as_float(v.y & 0xFFFF0000u);
    o[4] = __uint_as_float(v.z << 16);
    o[5] = __uint_as_float(v.z & 0xFFFF0000u);
    o[6] = __uint_as_float(v.w << 16);
    o[7] = __uint_as_float(v.w & 0xFFFF0000u);
  }
};

// Combine (reference, sum) partials whose sums are relative to their own reference.
__device__ __forceinline__ float part_term(float m, float s, float M, float cT) {
  return m == -INFINITY ? 0.f : s * ex2((m - M) * cT);
}

// Paired warp reductions (two independent values per shuffle round).  Warp
// maxima in one instruction each (redux.sync on f32, sm_100a): NaN inputs are
// dropped (as fmaxf does), or with .NaN make the result NaN.
__device__ __forceinline__ void warp_max2(float& a, float& b) {
  asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(a));
  asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(b));
}
__device__ __forceinline__ void warp_max2_nan(float& a, float& b) {
  asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(a));
  asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(b));
}
__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, a, o);
    const float y = __shfl_xor_sync(0xffffffffu, b, o);
    a += x;
    b += y;
  }
}

// ------------------------------------------------------------------ host side
struct LaunchPlan {
  int C, groups, threads, stages, slice;
  uint32_t stage_bytes;
  size_t smem;
  int clusters_max;
};

// Clusters of C CTAs of this kernel that fit on the device at once (0 if none).
inline int max_active_clusters(const void* fn, int C, int threads, size_t smem) {
  cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C * 64);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Launches `fn(args)` as `nclusters` clusters of `plan.C` CTAs.
template <typename Args>
inline sd_status launch_clusters(const void* fn, const LaunchPlan& plan, int64_t nclusters,
                                 Args& args, cudaStream_t stream) {
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nclusters * plan.C));
  cfg.blockDim = dim3(plan.threads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = plan.C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  void* kargs[] = {(void*)&args};
  if (cudaLaunchKernelExC(&cfg, fn, kargs) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  return SD_OK;
}

inline bool tau_ok(float tau) { return tau > 0.f && tau < INFINITY; }

inline void fill_tau(ScoreArgs& a, float tau) {
  a.inv_tau = (float)(1.0 / (double)tau);
  a.cT = (float)(1.4426950408889634 / (double)tau);
  a.tau64 = (double)tau;
  a.inv_tau64 = 1.0 / (double)tau;
}

}  // namespace smcsd
