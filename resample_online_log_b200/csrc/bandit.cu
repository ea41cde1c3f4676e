// Drafter selection by a per-sequence UCB bandit (MetaSD-UCB).
//
// METASD page, section 2 (Methodology): each speculative-decoding round picks
// one of M drafters with a multi-armed bandit whose reward is the Block
// Divergence (an alignment signal from the total-variation distance between
// drafter and target next-token distributions) or the Block Efficiency (the
// accepted-token count).  The page gives no formula; the rule here is UCB1
// with rewards in [0, 1]:
//   BD = 1 - (1/K) sum_{k<K} TV_k,   BE = accepted_len / K,
//   next arm = first arm never pulled, else argmax_i S_i/n_i + sqrt(c ln t / n_i),
//   t = sum_i n_i, ties to the lowest i.
//
// One thread per sequence, fp64 throughout; the reward is summed in position
// order so it is bit-reproducible.  The state (pulls, sums) is caller-owned
// and updated in place; arm_out may alias arm_in (each thread reads its own
// entry before writing it), so neither carries __restrict__.
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

__global__ void metasd_ucb_kernel(const float* __restrict__ tv, int64_t ld_tv,
                                  const int32_t* __restrict__ accepted_len,
                                  const int32_t* arm_in, int B, int K, int M, int kind,
                                  double c, int32_t* __restrict__ pulls,
                                  double* __restrict__ sums, int32_t* arm_out,
                                  double* __restrict__ reward_out, uint32_t* dev_err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int32_t* n = pulls + (int64_t)b * M;
  double* S = sums + (int64_t)b * M;
  const int a = arm_in[b];
  double r = NAN;
  if (a < -1 || a >= M) {
    raise_err(dev_err, SD_DEV_ARM_OOB);
  } else if (a >= 0) {
    if (kind == SD_REWARD_BD) {
      const float* row = tv + (int64_t)b * ld_tv;
      double s = 0.0;
      for (int k = 0; k < K; ++k) s += (double)row[k];
      r = 1.0 - s / (double)K;
    } else {
      const int acc = accepted_len[b];
      if (acc >= 0 && acc <= K) r = (double)acc / (double)K;
    }
    if (isfinite(r)) {
      n[a] += 1;
      S[a] += r;
    } else {
      r = NAN;
      raise_err(dev_err, SD_DEV_NONFINITE);
    }
  }
  if (reward_out) reward_out[b] = r;
  int64_t t = 0;
  int pick = -1;
  for (int i = 0; i < M; ++i) {
    t += n[i];
    if (pick < 0 && n[i] == 0) pick = i;
  }
  if (pick < 0) {
    const double lt = c * log((double)t);
    double best = -INFINITY;
    for (int i = 0; i < M; ++i) {
      const double ni = (double)n[i];
      const double u = S[i] / ni + sqrt(lt / ni);
      if (pick < 0 || u > best) {
        best = u;
        pick = i;
      }
    }
  }
  arm_out[b] = pick;
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status sd_metasd_ucb(const float* tv, int64_t ld_tv, const int32_t* accepted_len,
                                   const int32_t* arm_in, int B, int K, int M, int reward_kind,
                                   double c, int32_t* pulls, double* sums, int32_t* arm_out,
                                   double* reward_out, uint32_t* dev_err, void* stream) {
  if (B < 0 || K < 1 || M < 1 || M > 4096 || !(c >= 0.0 && c < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (reward_kind != SD_REWARD_BD && reward_kind != SD_REWARD_BE) return SD_ERR_INVALID_ARG;
  if (B == 0) return SD_OK;
  if (!arm_in || !pulls || !sums || !arm_out) return SD_ERR_INVALID_ARG;
  if (reward_kind == SD_REWARD_BD && (!tv || ld_tv < K)) return SD_ERR_INVALID_ARG;
  if (reward_kind == SD_REWARD_BE && !accepted_len) return SD_ERR_INVALID_ARG;
  const int threads = 128;
  metasd_ucb_kernel<<<(B + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(
      tv, ld_tv, accepted_len, arm_in, B, K, M, reward_kind, c, pulls, sums, arm_out, reward_out,
      dev_err);
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  return SD_OK;
}
