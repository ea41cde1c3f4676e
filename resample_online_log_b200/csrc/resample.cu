// Weight normalisation, ESS and systematic resampling: one thread block per
// sequence, all arithmetic in fp64.
//
// "Faster LLM Inference via Sequential Monte Carlo", section 2 (resampling
// step): particles with low importance weight are evicted and high-weight ones
// duplicated to form the next round's N particles.  The scheme used here is
// systematic resampling, every round or (adaptive, the usual SMC refinement
// the page's section 5 extensions build on) only when ESS < ess_frac * N:
//   W_j = exp(logw_j - max) / sum,  ESS = 1 / sum W_j^2,
//   C_j = W_0 + ... + W_j,  U_i = (i + u0) / N,  a_i = min{ j : C_j > U_i }.
// A sequence left alone keeps the identity ancestors and carries its
// log-weights to the next round (logw_next = logw; 0 after a resample).
// The order of every reduction is fixed, so results are bit-reproducible.
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

constexpr int kResampleMaxN = 8192;

__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions over <= 32 warps through a small shared scratch.
__device__ double block_sum_d(double v, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double r = 0.0;
  if (warp == 0) {
    r = lane < nw ? scratch[lane] : 0.0;
    r = warp_sum_d(r);
    if (lane == 0) scratch[32] = r;
  }
  __syncthreads();
  return scratch[32];
}
__device__ double block_max_d(double v, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max_d(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    double r = lane < nw ? scratch[lane] : -INFINITY;
    r = warp_max_d(r);
    if (lane == 0) scratch[32] = r;
  }
  __syncthreads();
  return scratch[32];
}
// Exclusive block scan of one value per thread.
__device__ double block_exclusive_scan_d(double v, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  double inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    double w = lane < nw ? scratch[lane] : 0.0;
    double wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < nw) scratch[lane] = wi - w;  // exclusive prefix of warp totals
  }
  __syncthreads();
  return scratch[warp] + (inc - v);
}

// Thread t owns particles t, t + T, t + 2T, ... so no thread ever touches two
// adjacent doubles (every shared / global access is a naturally aligned
// scalar).  The running sum is a block-wide scan over chunks of T particles
// with a carried offset.  Shared layout: [0, 40) reduction scratch, then the
// N weights / running sums, both 16-byte aligned.
// logw_next may alias logw (each entry is read before the same thread writes
// it), so neither carries __restrict__.
__global__ void resample_kernel(const double* logw, int N, double ess_frac, uint64_t seed,
                                uint64_t round, double* __restrict__ w_out,
                                double* __restrict__ ess_out, int32_t* __restrict__ anc_out,
                                int32_t* __restrict__ resampled_out, double* logw_next,
                                uint32_t* dev_err) {
  extern __shared__ __align__(16) double sh_all[];
  double* scratch = sh_all;
  double* sh = sh_all + 40;
  const int b = blockIdx.x;
  const int T = blockDim.x, t = threadIdx.x;
  const double* lw = logw + (int64_t)b * N;

  double m = -INFINITY;
  double badv = 0.0;
  for (int j = t; j < N; j += T) {
    const double v = lw[j];
    if (isnan(v) || v == INFINITY) badv = 1.0;
    m = fmax(m, v);
  }
  m = block_max_d(m, scratch);
  badv = block_max_d(badv, scratch);
  if (badv > 0.0 || m == -INFINITY) {
    for (int j = t; j < N; j += T) {
      if (w_out) w_out[(int64_t)b * N + j] = NAN;
      anc_out[(int64_t)b * N + j] = j;
      if (logw_next) logw_next[(int64_t)b * N + j] = lw[j];
    }
    if (t == 0) {
      if (ess_out) ess_out[b] = NAN;
      if (resampled_out) resampled_out[b] = 0;
      raise_err(dev_err, SD_DEV_NONFINITE);
    }
    return;
  }
  double s = 0.0;
  for (int j = t; j < N; j += T) {
    const double w = exp(lw[j] - m);
    sh[j] = w;
    s += w;
  }
  const double S = block_sum_d(s, scratch);
  double sq = 0.0;
  for (int j = t; j < N; j += T) {
    const double W = sh[j] / S;
    sh[j] = W;
    if (w_out) w_out[(int64_t)b * N + j] = W;
    sq += W * W;
  }
  const double sumsq = block_sum_d(sq, scratch);
  const double ess = 1.0 / sumsq;
  if (t == 0 && ess_out) ess_out[b] = ess;
  const bool resample = ess < ess_frac * (double)N;
  if (t == 0 && resampled_out) resampled_out[b] = resample ? 1 : 0;
  if (logw_next)
    for (int j = t; j < N; j += T) logw_next[(int64_t)b * N + j] = resample ? 0.0 : lw[j];
  if (!resample) {  // the weights carry: every particle is its own ancestor
    for (int j = t; j < N; j += T) anc_out[(int64_t)b * N + j] = j;
    return;
  }
  // running sums C_j, chunk by chunk
  double carry = 0.0;
  for (int c0 = 0; c0 < N; c0 += T) {
    const int j = c0 + t;
    const double v = j < N ? sh[j] : 0.0;
    const double ex = block_exclusive_scan_d(v, scratch);
    const double total = block_sum_d(v, scratch);
    if (j < N) sh[j] = carry + ex + v;
    carry += total;
  }
  __syncthreads();
  const Stream st(seed, round, SD_STREAM_RESAMPLE);
  const double u0 = uniform_f64(st.at(0, (uint32_t)b).x);
  for (int i = t; i < N; i += T) {
    const double U = ((double)i + u0) / (double)N;
    int lo = 0, hi = N;  // first j with C_j > U
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sh[mid] > U) hi = mid;
      else lo = mid + 1;
    }
    anc_out[(int64_t)b * N + i] = lo < N ? lo : N - 1;
  }
}

}  // namespace smcsd

using namespace smcsd;

namespace smcsd {
static sd_status launch_resample(const double* logw, int B, int N, double ess_frac, uint64_t seed,
                                 uint64_t round, double* w_out, double* ess_out,
                                 int32_t* ancestors_out, int32_t* resampled_out,
                                 double* logw_next, uint32_t* dev_err, void* stream) {
  if (B < 0 || N < 1 || !(ess_frac >= 0.0)) return SD_ERR_INVALID_ARG;
  if (N > kResampleMaxN) return SD_ERR_UNSUPPORTED;
  if (B == 0) return SD_OK;
  if (!logw || !ancestors_out) return SD_ERR_INVALID_ARG;
  int threads = (N + 31) / 32 * 32;  // one particle per thread up to 1024
  if (threads > 1024) threads = 1024;
  const size_t smem = (size_t)(N + 40) * sizeof(double);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(resample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  resample_kernel<<<B, threads, smem, (cudaStream_t)stream>>>(
      logw, N, ess_frac, seed, round, w_out, ess_out, ancestors_out, resampled_out, logw_next,
      dev_err);
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  return SD_OK;
}
}  // namespace smcsd

extern "C" sd_status smcsd_resample(const double* logw, int B, int N, uint64_t seed,
                                    uint64_t round, double* w_out, double* ess_out,
                                    int32_t* ancestors_out, uint32_t* dev_err, void* stream) {
  return launch_resample(logw, B, N, INFINITY, seed, round, w_out, ess_out, ancestors_out, nullptr,
                         nullptr, dev_err, stream);
}

extern "C" sd_status smcsd_resample_adaptive(const double* logw, int B, int N, double ess_frac,
                                             uint64_t seed, uint64_t round, double* w_out,
                                             double* ess_out, int32_t* ancestors_out,
                                             int32_t* resampled_out, double* logw_next,
                                             uint32_t* dev_err, void* stream) {
  return launch_resample(logw, B, N, ess_frac, seed, round, w_out, ess_out, ancestors_out,
                         resampled_out, logw_next, dev_err, stream);
}
