// Gumbel-top-k sampling without replacement: dense logit rows and sparse
// top-L (index, probability) rows.
//
// STAND, Methodology item 2: adding Gumbel noise to the log-probabilities and
// taking the k largest indices draws k tokens without replacement in
// parallel; item 1: the logit n-gram store keeps only the top-10 (index,
// probability) pairs of a row, unstored entries having probability 0.
//
// Dense kernel (one CTA per row, one streaming pass over HBM):
//   * online log-sum-exp of s = z / tau (one exp2 per entry) for the log-probs;
//   * a per-thread list of its best k+1 perturbed scores s_v + g_v under a
//     pruning threshold T that is always a lower bound on the row's (k+1)-th
//     best score (a thread's own (k+1)-th best, raised through a CTA-shared
//     maximum).  Groups of four entries with s + g_max < T skip the Philox call;
//     an entry with u <= 1 - e^{s - T} cannot reach T (e^{-y} >= 1 - y) and
//     skips the logs;
//   * the fp32 scores carry error bounds; when the order of the first k+1 is
//     not settled by them, the row is re-scored exactly in fp64.
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

constexpr int kTopkMax = 16;     // k <= 16
constexpr int kListMax = 17;     // longest per-thread list (k + 1)
constexpr int kTopkThreads = 512;
constexpr int kCandCap = 1024;   // candidates gathered per row

// Order-preserving map of floats to signed ints (for atomicMax on a threshold).
__device__ __forceinline__ int f2ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

// fp32 score error bound: a32 = z * (1/tau) and g32 from CUDA's logf / log1pf.
__device__ __forceinline__ float score_err(float a32, float g32) {
  return 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
}

struct TopkSmem {
  int thr;                 // CTA threshold (ordered int)
  int dropped;             // largest upper bound of an evicted list entry (ordered int)
  int ncand;
  int flag;
  float red_m[kTopkThreads / 32], red_s[kTopkThreads / 32];
  float cs[kCandCap];
  float cd[kCandCap];      // error bound of each candidate
  int ci[kCandCap];
  double lse;
  double s64[kTopkMax + 1];
  int i64[kTopkMax + 1];
};

template <typename TIn>
__device__ __forceinline__ float ld_elem(const TIn* p, int i);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p, int i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_elem<uint16_t>(const uint16_t* p, int i) {
  return __uint_as_float((uint32_t)p[i] << 16);
}

// Inserts (s, d, v) into a descending list of length L (ties to the lower v);
// returns the upper bound of the entry pushed out (or -inf).
template <int L>
__device__ __forceinline__ float list_insert(float (&ls)[L], float (&ld)[L], int (&li)[L], float s,
                                             float d, int v) {
#pragma unroll
  for (int j = 0; j < L; ++j) {
    const bool before = s > ls[j] || (s == ls[j] && v < li[j]);
    if (before) {
      const float ts = ls[j], td = ld[j];
      const int ti = li[j];
      ls[j] = s;
      ld[j] = d;
      li[j] = v;
      s = ts;
      d = td;
      v = ti;
    }
  }
  return v == 0x7FFFFFFF ? -INFINITY : s + d;
}

// Exact fp64 top-(k+1) of a row by a full re-scan (ambiguous fp32 order; rare).
// Every thread keeps its best k+1 fp64 scores of entries whose fp32 upper bound
// reaches `lo_star`; the CTA merges them by repeated maximum extraction.
template <typename TIn>
__device__ __noinline__ void exact_topk_row(const TIn* row, int V, int k1, float inv_tau,
                                            double tau64, float lo_star, const Stream st,
                                            uint32_t rowid, TopkSmem* sm) {
  double bs[kListMax];
  int bi[kListMax];
  for (int j = 0; j < kListMax; ++j) {
    bs[j] = -INFINITY;
    bi[j] = 0x7FFFFFFF;
  }
  for (int q = threadIdx.x; q * 4 < V; q += blockDim.x) {
    const U4 w = st.at((uint32_t)q, rowid);
    for (int j = 0; j < 4; ++j) {
      const int v = q * 4 + j;
      if (v >= V) break;
      const float z = ld_elem<TIn>(row, v);
      const float a32 = z * inv_tau;
      if (!(a32 + kGumbelMaxF + 1e-3f >= lo_star)) continue;
      const float g32 = gumbel_f32(uniform_f32(word_of(w, j)));
      if (!(a32 + g32 + score_err(a32, g32) >= lo_star)) continue;
      double s = (double)z / tau64 + gumbel_f64(uniform_f64(word_of(w, j)));
      int vi = v;
      for (int t = 0; t < kListMax && t < k1; ++t) {
        if (s > bs[t] || (s == bs[t] && vi < bi[t])) {
          const double ts = bs[t];
          const int ti = bi[t];
          bs[t] = s;
          bi[t] = vi;
          s = ts;
          vi = ti;
        }
      }
    }
  }
  // merge: k1 rounds of block-wide argmax over the threads' list heads
  __shared__ double rs[kTopkThreads / 32];
  __shared__ int ri[kTopkThreads / 32];
  int head = 0;
  for (int r = 0; r < k1; ++r) {
    double s = head < k1 ? bs[head] : -INFINITY;
    int v = head < k1 ? bi[head] : 0x7FFFFFFF;
    for (int o = 16; o > 0; o >>= 1) {
      const double os = __shfl_xor_sync(0xffffffffu, s, o);
      const int ov = __shfl_xor_sync(0xffffffffu, v, o);
      if (os > s || (os == s && ov < v)) {
        s = os;
        v = ov;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      rs[threadIdx.x >> 5] = s;
      ri[threadIdx.x >> 5] = v;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int nw = blockDim.x >> 5;
      s = threadIdx.x < nw ? rs[threadIdx.x] : -INFINITY;
      v = threadIdx.x < nw ? ri[threadIdx.x] : 0x7FFFFFFF;
      for (int o = 16; o > 0; o >>= 1) {
        const double os = __shfl_xor_sync(0xffffffffu, s, o);
        const int ov = __shfl_xor_sync(0xffffffffu, v, o);
        if (os > s || (os == s && ov < v)) {
          s = os;
          v = ov;
        }
      }
      if (threadIdx.x == 0) {
        sm->s64[r] = s;
        sm->i64[r] = v;
      }
    }
    __syncthreads();
    const int won = sm->i64[r];
    if (head < k1 && won != 0x7FFFFFFF && bi[head] == won) ++head;
    __syncthreads();
  }
}

template <typename TIn, int L>
__global__ void __launch_bounds__(kTopkThreads) topk_dense_kernel(
    const TIn* __restrict__ z, int rows, int V, int64_t ld, int k, float inv_tau, double tau64,
    uint64_t seed, uint64_t round, int vec, int32_t* __restrict__ idx_out, float* score_out,
    float* logp_out, uint32_t* dev_err) {
  __shared__ TopkSmem sm;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
  const int k1 = k + 1;
  const TIn* row = z + (int64_t)r * ld;
  const Stream st(seed, round, SD_STREAM_TOPK_DENSE);
  if (tid == 0) {
    sm.thr = f2ord(-INFINITY);
    sm.dropped = f2ord(-INFINITY);
    sm.ncand = 0;
    sm.flag = 0;
  }
  __syncthreads();

  float ls[L], ldv[L];
  int li[L];
  float dropped_hi = -INFINITY;
#pragma unroll
  for (int j = 0; j < L; ++j) {
    ls[j] = -INFINITY;
    ldv[j] = 0.f;
    li[j] = 0x7FFFFFFF;
  }
  float T = -INFINITY;        // lower bound on the row's (k+1)-th best score
  float m = -INFINITY, S = 0.f;
  bool bad = false;
  constexpr int EPC = 8;      // entries per chunk (two Philox groups)
  const int nchunks = (V + EPC - 1) / EPC;
  int iter = 0;
  for (int c = tid; c < nchunks; c += nthr, ++iter) {
    const int v0 = c * EPC;
    float s[EPC];
    if (vec && v0 + EPC <= V) {
      if (sizeof(TIn) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(row + v0);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[2 * j] = __uint_as_float(w4[j] << 16) * inv_tau;
          s[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u) * inv_tau;
        }
      } else {
        const float4 a = *reinterpret_cast<const float4*>(row + v0);
        const float4 b = *reinterpret_cast<const float4*>(row + v0 + 4);
        s[0] = a.x * inv_tau; s[1] = a.y * inv_tau; s[2] = a.z * inv_tau; s[3] = a.w * inv_tau;
        s[4] = b.x * inv_tau; s[5] = b.y * inv_tau; s[6] = b.z * inv_tau; s[7] = b.w * inv_tau;
      }
    } else {
#pragma unroll
      for (int j = 0; j < EPC; ++j) s[j] = v0 + j < V ? ld_elem<TIn>(row, v0 + j) * inv_tau : -INFINITY;
    }
    // online log-sum-exp (entries relative to the running max)
    float cm = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPC; ++j) {
      cm = fmaxf(cm, s[j]);
      bad |= (s[j] != s[j]) || (s[j] == INFINITY);
    }
    if (cm > m) {
      S = (m == -INFINITY) ? 0.f : S * ex2((m - cm) * kLog2e);
      m = cm;
    }
    if (m > -INFINITY) {
#pragma unroll
      for (int j = 0; j < EPC; ++j) S += ex2((s[j] - m) * kLog2e);
    }
    // candidates
#pragma unroll
    for (int gq = 0; gq < 2; ++gq) {
      const float gm = fmaxf(fmaxf(s[4 * gq], s[4 * gq + 1]), fmaxf(s[4 * gq + 2], s[4 * gq + 3]));
      if (!(gm + kGumbelMaxF + 1e-4f + 1e-6f * fabsf(gm) >= T)) continue;
      const U4 w = st.at((uint32_t)((v0 >> 2) + gq), (uint32_t)r);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float sv = s[4 * gq + j];
        if (!(sv > -INFINITY)) continue;
        const float u = uniform_f32(word_of(w, j));
        if (T > -INFINITY) {
          const float y = ex2((sv - T) * kLog2e) * 1.001f + 1e-30f;
          if (u < (1.0f - y) - 2.4e-7f) continue;
        }
        const float g32 = gumbel_f32(u);
        const float sc = sv + g32;
        const float d = score_err(sv, g32);
        if (!(sc + d >= T)) continue;
        dropped_hi = fmaxf(dropped_hi, list_insert<L>(ls, ldv, li, sc, d, v0 + 4 * gq + j));
        float kth = -INFINITY;  // lower bound of this thread's (k+1)-th best (-inf until held)
#pragma unroll
        for (int t = 0; t < L; ++t)
          if (t == k1 - 1) kth = ls[t] - ldv[t];
        T = fmaxf(T, kth);
      }
    }
    if ((iter & 3) == 3) {  // share / refresh the CTA threshold
      atomicMax(&sm.thr, f2ord(T));
      T = fmaxf(T, ord2f(*(volatile int*)&sm.thr));
    }
  }
  atomicMax(&sm.thr, f2ord(T));
  atomicMax(&sm.dropped, f2ord(dropped_hi));

  // lse: CTA combine of (m, S)
  float M = warp_max(m);
  float Sw = (m == -INFINITY) ? 0.f : S * ex2((m - M) * kLog2e);
  Sw = warp_sum(Sw);
  if (lane == 0) {
    sm.red_m[warp] = M;
    sm.red_s[warp] = Sw;
  }
  const int badw = __any_sync(0xffffffffu, bad);
  if (badw && lane == 0) atomicOr(&sm.flag, 1);
  __syncthreads();
  if (warp == 0) {
    const int nw = nthr >> 5;
    const float pm = lane < nw ? sm.red_m[lane] : -INFINITY;
    const float ps = lane < nw ? sm.red_s[lane] : 0.f;
    const float MM = warp_max(pm);
    const double t = (lane < nw && pm > -INFINITY) ? (double)ps * (double)ex2((pm - MM) * kLog2e) : 0.0;
    const double SS = warp_sum_d(t);
    if (lane == 0) {
      sm.lse = (double)MM + log(SS);
      if (!(MM > -INFINITY)) sm.flag |= 1;  // all -inf
    }
  }
  // gather the list entries that can still make the top k+1
  const float Tfin = ord2f(sm.thr);
#pragma unroll
  for (int j = 0; j < L; ++j) {
    if (li[j] != 0x7FFFFFFF && ls[j] + ldv[j] >= Tfin) {
      const int pos = atomicAdd(&sm.ncand, 1);
      if (pos < kCandCap) {
        sm.cs[pos] = ls[j];
        sm.cd[pos] = ldv[j];
        sm.ci[pos] = li[j];
      }
    }
  }
  __syncthreads();
  if (sm.flag & 1) {  // non-finite row
    if (tid < k) {
      idx_out[(int64_t)r * k + tid] = -1;
      if (score_out) score_out[(int64_t)r * k + tid] = NAN;
      if (logp_out) logp_out[(int64_t)r * k + tid] = NAN;
    }
    if (tid == 0) raise_err(dev_err, SD_DEV_NONFINITE);
    return;
  }
  const int n = min(sm.ncand, kCandCap);
  bool need_exact = sm.ncand > kCandCap;
  // warp 0 extracts the top k+1 (descending, ties to the lower index)
  if (warp == 0) {
    bool ambiguous = false;
    float prev_lo = INFINITY;
    for (int rnk = 0; rnk < k1; ++rnk) {
      float bs = -INFINITY, bd = 0.f;
      int bi = 0x7FFFFFFF, bp = -1;
      for (int p = lane; p < n; p += 32) {
        const float s = sm.cs[p];
        const int v = sm.ci[p];
        if (s > bs || (s == bs && v < bi)) {
          bs = s;
          bi = v;
          bd = sm.cd[p];
          bp = p;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        const float od = __shfl_xor_sync(0xffffffffu, bd, o);
        const int op = __shfl_xor_sync(0xffffffffu, bp, o);
        if (os > bs || (os == bs && oi < bi)) {
          bs = os;
          bi = oi;
          bd = od;
          bp = op;
        }
      }
      // the order between this rank and the previous one must be settled
      if (rnk > 0 && bi != 0x7FFFFFFF && !(bs + bd < prev_lo)) ambiguous = true;
      // nothing evicted from a thread's list may reach the k-th output
      if (rnk == k - 1 && !(ord2f(sm.dropped) < bs - bd)) ambiguous = true;
      prev_lo = bs - bd;
      if (lane == 0) {
        sm.s64[rnk] = bs;
        sm.i64[rnk] = bi;
        if (bp >= 0) sm.cs[bp] = -INFINITY;
      }
      __syncwarp();
    }
    if (lane == 0 && ambiguous) sm.flag |= 2;
  }
  __syncthreads();
  need_exact = need_exact || (sm.flag & 2);
  if (need_exact) {
    // lo bound of the k-th candidate: everything that can reach it is re-scored
    const float lo_k = (float)sm.s64[k - 1] - 1e-3f - 1e-5f * fabsf((float)sm.s64[k - 1]);
    __syncthreads();
    exact_topk_row<TIn>(row, V, k1, inv_tau, tau64, lo_k, st, (uint32_t)r, &sm);
    __syncthreads();
  }
  if (tid < k) {
    const int v = sm.i64[tid];
    const bool ok = v != 0x7FFFFFFF && sm.s64[tid] > -INFINITY;
    idx_out[(int64_t)r * k + tid] = ok ? v : -1;
    if (score_out) score_out[(int64_t)r * k + tid] = ok ? (float)sm.s64[tid] : NAN;
    if (logp_out)
      logp_out[(int64_t)r * k + tid] = ok ? (float)((double)ld_elem<TIn>(row, v) / tau64 - sm.lse) : NAN;
  }
}

// Sparse rows: one thread per row, fp64 throughout (L <= 64 entries).
__global__ void topk_sparse_kernel(const int32_t* __restrict__ idx, const float* __restrict__ prob,
                                   int rows, int L, int k, double tau64, uint64_t seed,
                                   uint64_t round, int32_t* __restrict__ idx_out, uint32_t* dev_err) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const Stream st(seed, round, SD_STREAM_TOPK_SPARSE);
  const float* pr = prob + (int64_t)r * L;
  bool bad = false;
  for (int l = 0; l < L; ++l) {
    const float p = pr[l];
    if (p != p || p < 0.f || p == INFINITY) bad = true;
  }
  if (bad) {
    for (int j = 0; j < k; ++j) idx_out[(int64_t)r * k + j] = -1;
    raise_err(dev_err, SD_DEV_NONFINITE);
    return;
  }
  double bs[kTopkMax];
  int bl[kTopkMax];
  int nb = 0;
  for (int q = 0; q * 4 < L; ++q) {
    const U4 w = st.at((uint32_t)q, (uint32_t)r);
    for (int j = 0; j < 4; ++j) {
      const int l = q * 4 + j;
      if (l >= L) break;
      const float p = pr[l];
      if (!(p > 0.f)) continue;  // unstored / zero probability: never drawn
      double s = log((double)p) / tau64 + gumbel_f64(uniform_f64(word_of(w, j)));
      int li = l;
      // insertion into the descending list (ties to the lower position)
      int pos = nb < k ? nb : k;
      if (nb < k) ++nb;
      for (int t = 0; t < pos; ++t) {
        if (s > bs[t] || (s == bs[t] && li < bl[t])) {
          const double ts = bs[t];
          const int tl = bl[t];
          bs[t] = s;
          bl[t] = li;
          s = ts;
          li = tl;
        }
      }
      if (pos < k) {
        bs[pos] = s;
        bl[pos] = li;
      }
    }
  }
  for (int j = 0; j < k; ++j)
    idx_out[(int64_t)r * k + j] = j < nb ? idx[(int64_t)r * L + bl[j]] : -1;
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status gumbel_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld, int k,
                                 float tau, uint64_t seed, uint64_t round, int32_t* idx_out,
                                 float* score_out, float* logp_out, uint32_t* dev_err,
                                 void* stream) {
  if (rows < 0 || V < 1 || ld < V || k < 1 || k > kTopkMax || k > V ||
      !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (rows == 0) return SD_OK;
  if (!z || !idx_out) return SD_ERR_INVALID_ARG;
  const int esize = dt == SD_BF16 ? 2 : 4;
  const int vec = ((uintptr_t)z % 16 == 0) && ((ld * esize) % 16 == 0);
  const float inv_tau = (float)(1.0 / (double)tau);
  cudaStream_t s = (cudaStream_t)stream;
  if (dt == SD_BF16) {
    if (k <= 8)
      topk_dense_kernel<uint16_t, 9><<<rows, kTopkThreads, 0, s>>>(
          (const uint16_t*)z, rows, V, ld, k, inv_tau, (double)tau, seed, round, vec, idx_out,
          score_out, logp_out, dev_err);
    else
      topk_dense_kernel<uint16_t, 17><<<rows, kTopkThreads, 0, s>>>(
          (const uint16_t*)z, rows, V, ld, k, inv_tau, (double)tau, seed, round, vec, idx_out,
          score_out, logp_out, dev_err);
  } else {
    if (k <= 8)
      topk_dense_kernel<float, 9><<<rows, kTopkThreads, 0, s>>>(
          (const float*)z, rows, V, ld, k, inv_tau, (double)tau, seed, round, vec, idx_out,
          score_out, logp_out, dev_err);
    else
      topk_dense_kernel<float, 17><<<rows, kTopkThreads, 0, s>>>(
          (const float*)z, rows, V, ld, k, inv_tau, (double)tau, seed, round, vec, idx_out,
          score_out, logp_out, dev_err);
  }
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

extern "C" sd_status gumbel_topk_sparse(const int32_t* idx, const float* prob, int rows, int L,
                                        int k, float tau, uint64_t seed, uint64_t round,
                                        int32_t* idx_out, uint32_t* dev_err, void* stream) {
  if (rows < 0 || L < 1 || L > kTopkMax || k < 1 || k > L || !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (rows == 0) return SD_OK;
  if (!idx || !prob || !idx_out) return SD_ERR_INVALID_ARG;
  const int threads = 128;
  topk_sparse_kernel<<<(rows + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(
      idx, prob, rows, L, k, (double)tau, seed, round, idx_out, dev_err);
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}
