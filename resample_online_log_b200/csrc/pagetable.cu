// KV page-table remap after resampling: a gather of page-table rows (and of
// the tokens the round commits) by ancestor index, plus optional page
// reference counts.
//
// "Faster LLM Inference via Sequential Monte Carlo", section 2 (KV cache
// management): duplicated particles share KV pages through pointer exchange
// and page-metadata copy instead of copying KV tensors.
//
// One warp per particle; rows of P int32 move as 16-byte vectors when the
// layout allows.  Reference counts use integer atomics, so their values are
// deterministic.
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

// Page ids are range-checked only when reference counts are requested (the
// call then knows num_pages).
__device__ __forceinline__ void count_page(int32_t p, int32_t* refcnt, int num_pages, bool& oob) {
  if (!refcnt) return;
  if (p >= 0 && p < num_pages) atomicAdd(&refcnt[p], 1);
  else if (p != -1) oob = true;
}

__global__ void remap_kernel(const int32_t* __restrict__ pt_in, const int32_t* __restrict__ anc,
                             int64_t particles, int N, int P, int32_t* __restrict__ pt_out,
                             const int32_t* __restrict__ tok_in, int T,
                             int32_t* __restrict__ tok_out, int32_t* refcnt, int num_pages,
                             int vec, uint32_t* dev_err) {
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= particles) return;
  const int64_t b = gw / N;
  const int a = anc[gw];
  const bool ok = a >= 0 && a < N;
  int32_t* dst = pt_out + gw * P;
  bool oob = false;
  if (!ok) {
    for (int s = lane; s < P; s += 32) dst[s] = -1;
    if (tok_out)
      for (int s = lane; s < T; s += 32) tok_out[gw * T + s] = -1;
    if (lane == 0) raise_err(dev_err, SD_DEV_ANCESTOR_OOB);
    return;
  }
  const int32_t* src = pt_in + (b * N + a) * P;
  if (vec) {
    const int4* s4 = reinterpret_cast<const int4*>(src);
    int4* d4 = reinterpret_cast<int4*>(dst);
    for (int s = lane; s < P / 4; s += 32) {
      const int4 v = s4[s];
      d4[s] = v;
      count_page(v.x, refcnt, num_pages, oob);
      count_page(v.y, refcnt, num_pages, oob);
      count_page(v.z, refcnt, num_pages, oob);
      count_page(v.w, refcnt, num_pages, oob);
    }
  } else {
    for (int s = lane; s < P; s += 32) {
      const int32_t v = src[s];
      dst[s] = v;
      count_page(v, refcnt, num_pages, oob);
    }
  }
  if (tok_out) {
    const int32_t* ts = tok_in + (b * N + a) * T;
    for (int s = lane; s < T; s += 32) tok_out[gw * T + s] = ts[s];
  }
  if (__any_sync(0xffffffffu, oob) && lane == 0) raise_err(dev_err, SD_DEV_PAGE_OOB);
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status kv_pagetable_remap(const int32_t* pt_in, const int32_t* ancestors, int B,
                                        int N, int P, int32_t* pt_out, const int32_t* tok_in,
                                        int T, int32_t* tok_out, int32_t* page_refcnt,
                                        int num_pages, uint32_t* dev_err, void* stream) {
  if (B < 0 || N < 1 || P < 0 || T < 0 || num_pages < 0) return SD_ERR_INVALID_ARG;
  if ((tok_in == nullptr) != (tok_out == nullptr)) return SD_ERR_INVALID_ARG;
  if (page_refcnt && num_pages < 1) return SD_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (B > 0 && (!ancestors || !pt_out || (P > 0 && !pt_in))) return SD_ERR_INVALID_ARG;
  const int64_t particles = (int64_t)B * N;
  if (B > 0 && P > 0 && pt_in == pt_out) return SD_ERR_INVALID_ARG;
  if (B > 0 && P > 0) {
    const int64_t lo_a = (int64_t)(uintptr_t)pt_in, hi_a = lo_a + particles * P * 4;
    const int64_t lo_b = (int64_t)(uintptr_t)pt_out, hi_b = lo_b + particles * P * 4;
    if (lo_a < hi_b && lo_b < hi_a) return SD_ERR_INVALID_ARG;  // must not alias
  }
  if (B > 0 && tok_in && T > 0) {  // the token gather is out of place too
    const int64_t lo_a = (int64_t)(uintptr_t)tok_in, hi_a = lo_a + particles * T * 4;
    const int64_t lo_b = (int64_t)(uintptr_t)tok_out, hi_b = lo_b + particles * T * 4;
    if (lo_a < hi_b && lo_b < hi_a) return SD_ERR_INVALID_ARG;
  }
  // Every argument is checked: only now is anything enqueued.
  if (page_refcnt && cudaMemsetAsync(page_refcnt, 0, (size_t)num_pages * 4, s) != cudaSuccess)
    return SD_ERR_CUDA;
  if (B == 0) return SD_OK;
  const int vec = (P % 4 == 0) && ((uintptr_t)pt_in % 16 == 0) && ((uintptr_t)pt_out % 16 == 0);
  const int threads = 256;
  const int64_t blocks = (particles * 32 + threads - 1) / threads;
  remap_kernel<<<(unsigned)blocks, threads, 0, s>>>(pt_in, ancestors, particles, N, P, pt_out,
                                                    tok_in, T, tok_out, page_refcnt, num_pages,
                                                    vec, dev_err);
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  return SD_OK;
}
