// Gumbel-top-k sampling without replacement (dense rows and sparse top-L rows).
#include <cuda_runtime.h>

#include "common.cuh"

extern "C" sd_status gumbel_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld, int k,
                                 float tau, uint64_t seed, uint64_t round, int32_t* idx_out,
                                 float* score_out, float* logp_out, uint32_t* dev_err,
                                 void* stream) {
  (void)seed; (void)round; (void)score_out; (void)logp_out; (void)dev_err; (void)stream;
  if (rows < 0 || V < 1 || ld < V || k < 1 || k > 64 || k > V || !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (rows == 0) return SD_OK;
  if (!z || !idx_out) return SD_ERR_INVALID_ARG;
  return SD_ERR_UNSUPPORTED;
}

extern "C" sd_status gumbel_topk_sparse(const int32_t* idx, const float* prob, int rows, int L,
                                        int k, float tau, uint64_t seed, uint64_t round,
                                        int32_t* idx_out, uint32_t* dev_err, void* stream) {
  (void)seed; (void)round; (void)dev_err; (void)stream;
  if (rows < 0 || L < 1 || L > 64 || k < 1 || k > L || !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (rows == 0) return SD_OK;
  if (!idx || !prob || !idx_out) return SD_ERR_INVALID_ARG;
  return SD_ERR_UNSUPPORTED;
}
