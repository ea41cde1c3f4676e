// Test-only entry points, built into libsmcsd_testing.so (not into
// libsmcsd.so):
//   * the library's own device Philox4x32-10 code -- the generator every
//     sampling kernel draws from (common.cuh: philox, philox_rk and the Stream
//     counter layout) -- run on counters the caller chooses, so that a test can
//     compare it word for word with an independent implementation and with
//     the published known-answer vectors;
//   * the bounded mbarrier wait of the kernels (common.cuh: bounded_wait) on a
//     barrier that nothing, or a second warp after a delay, completes, so a
//     test can see a wait run out and report its status without any fault.
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

// variant 0: philox (key bumped inside); variant 1: philox_rk (round keys
// computed once).  ctr [n, 4], key [n, 2], out [n, 4].
__global__ void philox_words_kernel(const uint32_t* __restrict__ ctr,
                                    const uint32_t* __restrict__ key, int n, int variant,
                                    uint32_t* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t c0 = ctr[4 * i], c1 = ctr[4 * i + 1], c2 = ctr[4 * i + 2], c3 = ctr[4 * i + 3];
  U4 w;
  if (variant == 0) {
    w = philox(c0, c1, c2, c3, key[2 * i], key[2 * i + 1]);
  } else {
    const PhiloxKeys K = philox_keys((uint64_t)key[2 * i] | ((uint64_t)key[2 * i + 1] << 32));
    w = philox_rk(c0, c1, c2, c3, K);
  }
  out[4 * i] = w.x;
  out[4 * i + 1] = w.y;
  out[4 * i + 2] = w.z;
  out[4 * i + 3] = w.w;
}

// Words 0 .. 4n-1 of one stream (seed, round, tag) for row id `row`, laid out
// as the kernels read per-entry noise: entry v uses counter word c0 = v / 4,
// output word v % 4.
__global__ void stream_words_kernel(uint64_t seed, uint64_t round, uint32_t tag, uint32_t row,
                                    int n, uint32_t* __restrict__ out) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= n) return;
  const Stream st(seed, round, tag);
  const U4 w = st.at((uint32_t)q, row);
  out[4 * q] = w.x;
  out[4 * q + 1] = w.y;
  out[4 * q + 2] = w.z;
  out[4 * q + 3] = w.w;
}

// mode bit 0: the abort flag starts set; bit 1: the wait is abortable; bit 2:
// a second warp completes the barrier delay_ns after the start.  out[0] = ns
// the wait took, out[1] = the abort flag after it.  Every wait here ends by
// itself: the waiter's after limit_ns, the second warp's after delay_ns.
__global__ void wait_kernel(uint64_t limit_ns, int mode, uint64_t delay_ns, uint32_t* err,
                            uint64_t* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ uint64_t t_start;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = mode & 1;
    t_start = globaltimer_ns();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // measured from t_start, the arriving warp's reference too, so that a wait
    // ended by an arrival after delay_ns lasts at least delay_ns
    bounded_wait(&bar, 0u, &abort_flag, err, 1u << 8, (mode & 2) != 0, limit_ns);
    out[0] = globaltimer_ns() - t_start;
    out[1] = (uint64_t)abort_flag;
  } else if (threadIdx.x == 32 && (mode & 4)) {
    while (globaltimer_ns() - t_start < delay_ns) {
    }
    mbar_arrive(&bar);
  }
}

}  // namespace smcsd

using namespace smcsd;

extern "C" __attribute__((visibility("default"))) int smcsd_testing_philox(
    const uint32_t* ctr, const uint32_t* key, int n, int variant, uint32_t* out, void* stream) {
  if (n < 0 || !ctr || !key || !out || (variant != 0 && variant != 1)) return 1;
  if (n == 0) return 0;
  philox_words_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(ctr, key, n, variant, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" __attribute__((visibility("default"))) int smcsd_testing_stream(
    uint64_t seed, uint64_t round, uint32_t tag, uint32_t row, int n, uint32_t* out, void* stream) {
  if (n < 0 || !out) return 1;
  if (n == 0) return 0;
  stream_words_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(seed, round, tag, row, n,
                                                                         out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" __attribute__((visibility("default"))) int smcsd_testing_wait(
    uint64_t limit_ns, int mode, uint64_t delay_ns, uint32_t* err, uint64_t* out, void* stream) {
  if (!out || mode < 0 || mode > 7 || limit_ns > 1000000000ull || delay_ns > 1000000000ull) return 1;
  wait_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(limit_ns, mode, delay_ns, err, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
