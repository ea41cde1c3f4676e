// Gumbel-top-k sampling without replacement: dense logit rows and sparse
// top-L (index, probability) rows.
//
// STAND, Methodology item 2: adding Gumbel noise to the log-probabilities and
// taking the k largest indices draws k tokens without replacement in
// parallel; item 1: the logit n-gram store keeps only the top-10 (index,
// probability) pairs of a row, unstored entries having probability 0.
//
// Dense kernel (persistent CTAs, two per SM, each taking rows in turn): the
// row is read twice, the second time from L2 (the first read asks L2 to keep
// it) -- once for the log-sum-exp and each thread's largest logit, whose
// exact perturbed scores give a lower bound T on the row's k-th best score;
// once for the candidates under T: four entries whose s + g_max < T skip the
// Philox call, an entry with u <= 1 - e^{s - T} cannot reach T (e^{-y} >=
// 1 - y) and skips the logs.  The fp32 scores carry error bounds; when the
// order of the first k+1 is not settled by them, the row is re-scored exactly
// in fp64.
#include <algorithm>
#include <cuda_runtime.h>

#include "common.cuh"
#include "rowload.cuh"

namespace smcsd {

constexpr int kTopkMax = 16;     // k <= 16
constexpr int kListMax = 17;     // longest per-thread list (k + 1)
constexpr int kTopkThreads = 512;
constexpr int kCandCap = 1024;   // candidates gathered per row
constexpr int kTopkUnroll = 4;   // chunks a thread has in flight in the first pass

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

// Inserts (s, d, v) into a descending list of length n held in a column of
// shared memory (entry j at j * stride; ties to the lower v); returns the upper
// bound of the entry pushed out (or -inf).
__device__ __forceinline__ float list_insert_col(float* ls, float* ld, int* li, int stride, int n,
                                                 float s, float d, int v) {
  for (int j = 0; j < n; ++j) {
    const float bs = ls[j * stride];
    const int bi = li[j * stride];
    if (s > bs || (s == bs && v < bi)) {
      const float bd = ld[j * stride];
      ls[j * stride] = s;
      ld[j * stride] = d;
      li[j * stride] = v;
      s = bs;
      d = bd;
      v = bi;
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

// Dense rows.  A persistent CTA takes rows in turn and reads each twice:
//   pass 1 (HBM, kept in L2 with an evict-last hint): the row's log-sum-exp
//     (one exp2 per entry, online per thread) and each thread's largest logit;
//   threshold: the exact fp32 perturbed scores of those per-thread maxima
//     (one Philox word each, minus their error bound) -- the k-th largest of
//     them is a lower bound T on the row's k-th best score;
//   pass 2 (L2): groups of four entries that even g_max cannot lift to T skip
//     the Philox call; an entry whose word proves u <= 1 - e^{s - T} (an
//     integer leading-bit test first, then the exp2) cannot reach T and skips
//     the logs; the rest enter the thread's descending list of k+1 candidates
//     with fp32 error bounds.
// The lists merge into the first k+1 ranks; when the fp32 bounds do not settle
// their order, the row is re-scored exactly in fp64.
template <typename TIn, int L>
__global__ void __launch_bounds__(kTopkThreads, 2) topk_dense_kernel(
    const TIn* __restrict__ z, int rows, int V, int64_t ld, int k, float inv_tau, double tau64,
    uint64_t seed, uint64_t round, uint32_t tag, uint32_t row0, int vec,
    int32_t* __restrict__ idx_out, float* score_out, float* logp_out, uint32_t* dev_err) {
  __shared__ TopkSmem sm;
  __shared__ float kbuf[(kTopkThreads / 32) * kTopkMax];
  extern __shared__ float lists[];  // [3][L][blockDim.x]: scores, error bounds, indices
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
  const int k1 = k + 1;
  const Stream st(seed, round, tag);
  const PhiloxKeys K = philox_keys(seed);
  const float cT = kLog2e * inv_tau;  // log2(e) / tau
  const int nchunks = (V + 7) / 8;
  const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
  const bool vecok = vec != 0;

  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const TIn* row = z + (int64_t)r * ld;
    const uint32_t rid = row0 + (uint32_t)r;
    if (tid == 0) {
      sm.thr = f2ord(-INFINITY);
      sm.dropped = f2ord(-INFINITY);
      sm.ncand = 0;
      sm.flag = 0;
    }
    __syncthreads();
    // ---------------- pass 1: log-sum-exp and per-thread maxima
    float m = -INFINITY, S = 0.f, zmax = -INFINITY;
    int zarg = 0x7FFFFFFF;
    bool bad = false;
    for (int c0 = tid; c0 < nchunks; c0 += kTopkUnroll * nthr) {
     Raw8<TIn> raw[kTopkUnroll];
#pragma unroll
     for (int u = 0; u < kTopkUnroll; ++u)
       if (c0 + u * nthr < nchunks) raw[u] = load8_raw<TIn>(row, (c0 + u * nthr) * 8, V, vecok, keep);
#pragma unroll
     for (int u = 0; u < kTopkUnroll; ++u) {
      const int c = c0 + u * nthr;
      if (c >= nchunks) break;
      float zz[8];
      unpack8<TIn>(raw[u], zz);
      float cm = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) cm = fmax_nan(cm, zz[j]);
      bad |= cm != cm;  // a NaN, even one met while every earlier entry was -inf
      if (cm > zmax) {
        zmax = cm;
#pragma unroll
        for (int j = 7; j >= 0; --j)
          if (zz[j] == cm) zarg = c * 8 + j;
      }
      if (cm > m) {
        S = (m == -INFINITY) ? 0.f : S * ex2((m - cm) * cT);
        m = cm;
      }
      if (m > -INFINITY) {
        const float nm = -m * cT;
#pragma unroll
        for (int j = 0; j < 8; ++j) S += ex2(fmaf(zz[j], cT, nm));
      }
     }
    }
    // lse: CTA combine of (m, S) in fp64
    // a NaN entry leaves S NaN (its exp2 is NaN), a +inf entry makes m +inf
    bad = bad || m == INFINITY || S != S;
    float M = warp_max(m);
    float Sw = (m == -INFINITY) ? 0.f : S * ex2((m - M) * cT);
    Sw = warp_sum(Sw);
    if (lane == 0) {
      sm.red_m[warp] = M;
      sm.red_s[warp] = Sw;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&sm.flag, 1);
    // threshold: exact fp32 lower bounds of the per-thread maxima's perturbed scores
    float lo = -INFINITY;
    if (zarg != 0x7FFFFFFF) {
      const U4 w = philox_rk((uint32_t)(zarg >> 2), rid, st.c2, st.c3, K);
      const float a32 = zmax * inv_tau;
      const float g32 = gumbel_f32(uniform_f32(word_of(w, zarg & 3)));
      lo = a32 + g32 - score_err(a32, g32);
    }
    __syncthreads();
    if (warp == 0) {
      const int nw = nthr >> 5;
      const float pm = lane < nw ? sm.red_m[lane] : -INFINITY;
      const float ps = lane < nw ? sm.red_s[lane] : 0.f;
      const float MM = warp_max(pm);
      const double t = (lane < nw && pm > -INFINITY) ? (double)ps * (double)ex2((pm - MM) * cT) : 0.0;
      const double SS = warp_sum_d(t);
      if (lane == 0) {
        sm.lse = (double)MM / tau64 + log(SS);
        if (!(MM > -INFINITY)) sm.flag |= 1;  // all -inf
      }
    }
    const float T0 = cta_kth_largest(lo, k, kbuf);  // (syncs the CTA)
    const bool rowbad = (sm.flag & 1) != 0;

    // ---------------- pass 2: the candidates
    // this thread's descending list of its best k+1 candidates, in a column of
    // shared memory (insertions are rare: registers stay with the stream)
    float* ls = lists + tid;
    float* ldv = lists + L * nthr + tid;
    int* li = reinterpret_cast<int*>(lists + 2 * L * nthr) + tid;
    float dropped_hi = -INFINITY;
    for (int j = 0; j < L; ++j) {
      ls[j * nthr] = -INFINITY;
      ldv[j * nthr] = 0.f;
      li[j * nthr] = 0x7FFFFFFF;
    }
    float T = T0;
    if (!rowbad && tid < nchunks) {
      Raw8<TIn> nxt = load8_raw<TIn>(row, tid * 8, V, vecok, drop);
      for (int c = tid; c < nchunks; c += nthr) {
        const Raw8<TIn> cur = nxt;
        if (c + nthr < nchunks) nxt = load8_raw<TIn>(row, (c + nthr) * 8, V, vecok, drop);
        float zz[8];
        unpack8<TIn>(cur, zz);
#pragma unroll 1
        for (int gq = 0; gq < 2; ++gq) {  // one Philox block: four entries
          float z4[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) z4[j] = gq ? zz[4 + j] : zz[j];
          const float zm = fmaxf(fmaxf(z4[0], z4[1]), fmaxf(z4[2], z4[3]));
          const float am = zm * inv_tau;
          if (!(am + kGumbelMaxF + 1e-4f + 1e-6f * fabsf(am) >= T)) continue;
          const int v0 = c * 8 + 4 * gq;
          const U4 w = philox_rk((uint32_t)(v0 >> 2), rid, st.c2, st.c3, K);
          // With Xm = (max s - T) log2(e), an entry needs u > 1 - e^{s - T} >= 1 - 2^Xm;
          // u = (m + 1/2) 2^-23 with m = w >> 9, so a word with m below mstar fails for all four.
          uint32_t mstar = 0;
          if (T > -INFINITY) {
            const float thr = (1.0f - ex2(fmaf(zm, cT, -T * kLog2e)) * 1.001f) - 2.4e-7f;
            mstar = thr > 0.f ? (uint32_t)ceilf(thr * 8388608.f - 0.5f) : 0u;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t wj = word_of(w, j);
            if ((wj >> 9) < mstar) continue;
            const float sv = z4[j] * inv_tau;
            if (!(sv > -INFINITY)) continue;
            const float u = uniform_f32(wj);
            if (T > -INFINITY) {  // the entry's own test: u <= 1 - e^{s - T} cannot reach T
              const float y = ex2((sv - T) * kLog2e) * 1.001f + 1e-30f;
              if (u < (1.0f - y) - 2.4e-7f) continue;
            }
            const float g32 = gumbel_f32(u);
            const float sc = sv + g32;
            const float d = score_err(sv, g32);
            if (!(sc + d >= T)) continue;
            dropped_hi = fmaxf(dropped_hi, list_insert_col(ls, ldv, li, nthr, k1, sc, d, v0 + j));
            // lower bound of this thread's (k+1)-th best (-inf until it holds k+1)
            T = fmaxf(T, ls[(k1 - 1) * nthr] - ldv[(k1 - 1) * nthr]);
          }
        }
      }
    }
    atomicMax(&sm.thr, f2ord(T));
    atomicMax(&sm.dropped, f2ord(dropped_hi));
    __syncthreads();
    // gather the list entries that can still make the top k+1
    const float Tfin = ord2f(sm.thr);
    for (int j = 0; j < k1; ++j) {
      const float cs = ls[j * nthr], cd = ldv[j * nthr];
      const int ci = li[j * nthr];
      if (ci != 0x7FFFFFFF && cs + cd >= Tfin) {
        const int pos = atomicAdd(&sm.ncand, 1);
        if (pos < kCandCap) {
          sm.cs[pos] = cs;
          sm.cd[pos] = cd;
          sm.ci[pos] = ci;
        }
      }
    }
    __syncthreads();
    if (rowbad) {  // non-finite row
      if (tid < k) {
        idx_out[(int64_t)r * k + tid] = -1;
        if (score_out) score_out[(int64_t)r * k + tid] = NAN;
        if (logp_out) logp_out[(int64_t)r * k + tid] = NAN;
      }
      if (tid == 0) raise_err(dev_err, SD_DEV_NONFINITE);
      __syncthreads();
      continue;
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
        for (int q = lane; q < n; q += 32) {
          const float sv = sm.cs[q];
          const int v = sm.ci[q];
          if (sv > bs || (sv == bs && v < bi)) {
            bs = sv;
            bi = v;
            bd = sm.cd[q];
            bp = q;
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
      exact_topk_row<TIn>(row, V, k1, inv_tau, tau64, lo_k, st, rid, &sm);
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
    __syncthreads();  // the shared state is reused by the next row
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

namespace smcsd {

// Launches the dense kernel: k ranks of rows [rows, V] with noise stream `tag`
// and row ids row0, row0 + 1, ...
static sd_status launch_topk_dense(const void* z, sd_dtype dt, int rows, int V, int64_t ld, int k,
                                   float tau, uint64_t seed, uint64_t round, uint32_t tag,
                                   uint32_t row0, int32_t* idx_out, float* score_out,
                                   float* logp_out, uint32_t* dev_err, cudaStream_t s) {
  const int esize = dt == SD_BF16 ? 2 : 4;
  const int vec = ((uintptr_t)z % 16 == 0) && ((ld * esize) % 16 == 0);
  const float inv_tau = (float)(1.0 / (double)tau);
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const int grid = std::min(rows, 2 * nsm);  // persistent: two CTAs per SM take the rows in turn
  // the candidate lists take dynamic shared memory: 3 * L * threads * 4 bytes
  auto launch = [&](auto kern, int L, const auto* zp) {
    const int dyn = 3 * L * kTopkThreads * 4;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess)
      return;
    kern<<<grid, kTopkThreads, dyn, s>>>(zp, rows, V, ld, k, inv_tau, (double)tau, seed, round, tag,
                                         row0, vec, idx_out, score_out, logp_out, dev_err);
  };
  if (dt == SD_BF16) {
    if (k <= 8) launch(topk_dense_kernel<uint16_t, 9>, 9, (const uint16_t*)z);
    else launch(topk_dense_kernel<uint16_t, 17>, 17, (const uint16_t*)z);
  } else {
    if (k <= 8) launch(topk_dense_kernel<float, 9>, 9, (const float*)z);
    else launch(topk_dense_kernel<float, 17>, 17, (const float*)z);
  }
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

}  // namespace smcsd

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
  return launch_topk_dense(z, dt, rows, V, ld, k, tau, seed, round, SD_STREAM_TOPK_DENSE, 0u,
                           idx_out, score_out, logp_out, dev_err, (cudaStream_t)stream);
}

// Draft step: one token per row from q_D = softmax(zD / tau) by Gumbel-max, which
// is Gumbel-top-1: the dense kernel with k = 1 on its own noise stream.
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
