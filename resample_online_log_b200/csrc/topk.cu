// Gumbel-top-k sampling without replacement: dense logit rows and sparse
// top-L (index, probability) rows.
//
// STAND, Methodology item 2: adding Gumbel noise to the log-probabilities and
// taking the k largest indices draws k tokens without replacement in
// parallel; item 1: the logit n-gram store keeps only the top-10 (index,
// probability) pairs of a row, unstored entries having probability 0.
//
// Dense rows are drawn top-down over blocks of 128 entries: every block gets
// its maximum M_j = log sum_{v in j} e^{z_v/tau} + G_j (block noise), the k
// largest blocks are kept (no entry of another block can be among the k
// largest scores), and only their entries get entry noise: scores
// conditioned on the block's maximum, S_v = -log(e^{-M_j} - e^{-Z_j} +
// e^{-h_v}) with h_v = z_v/tau + g_v and Z_j = max h (Kool, van Hoof and
// Welling, "Stochastic Beams and Where to Find Them", 2019).  Independent
// per-entry Gumbels have exactly this law, so the order is Gumbel-top-k's.
//
// Dense kernel (persistent CTAs, two per SM, each taking rows in turn):
//   pass (HBM, once): a warp takes tiles of 1024 entries (32 per lane, four
//     16-byte loads of bf16); exps relative to the warp's running max R (one
//     redux per tile); each lane parks the sum of its 32 exps with the tile's
//     R; every 4 tiles the warp scores their 32 blocks, one per lane: M_j with
//     fp32 error bounds into a per-row table, and the row's log-sum-exp partial;
//   blocks: the k-th largest of the threads' best lower bounds is a lower
//     bound T on the k-th largest M, so the blocks whose upper bound reaches T
//     hold the k largest; they are ranked by their fp32 scores, settled by
//     the bounds or else re-scored in fp64; the kept blocks' M_j in fp64;
//   entries (fp64): one warp per kept block draws its entries' scores
//     conditioned on M_j; those at or above the smallest kept M_j (the k-th
//     largest score is no smaller) are ranked by counting.
#include <cuda_runtime.h>

#include "rowload.cuh"
#include "rows.cuh"

namespace smcsd {

constexpr int kTopkMax = 16;      // k <= 16 (also the sparse row length limit)
constexpr int kTThreads = 512;    // 16 warps
constexpr int kTWarps = kTThreads / 32;
constexpr int kTBlk = 128;        // entries per block
constexpr int kTBuf = 4;          // tiles a warp buffers before scoring their blocks
constexpr int kTTile = 1024;      // entries per warp tile: 32 per lane, eight blocks
constexpr int kTMaxBlocks = 2048; // V <= 262144
constexpr int kTCand = 256;       // candidate blocks gathered per row
constexpr int kTEnt = kTopkMax * kTBlk;  // entries of the kept blocks

struct TopkSmem {
  float part[kTWarps][kTBuf][32];  // per lane: sum of its 32 exps, relative to the tile's R
  float ref[kTWarps][kTBuf];
  int tile[kTWarps][kTBuf];
  float bs[kTMaxBlocks];           // block maxima M_j (fp32), -inf: empty block
  float bd[kTMaxBlocks];           // their error bounds
  float m[kTWarps], s[kTWarps];    // row lse partials
  float kbuf[kTWarps * kTopkMax];  // k-th largest scratch
  int flag;                        // bit 0: bad row; bit 1: candidate overflow
  int ncand;
  int cblk[kTCand];
  int crank[kTCand];
  int lo_ord, hi_ord;              // min lower bound of the kept, max upper bound of the rest
  int nkeep;
  int keep[kTopkMax];
  double keepM[kTopkMax];
  double cM[kTCand];               // fp64 block maxima of the candidates (when re-scored)
  double lse;
  int ne;
  double es[kTEnt];                // entries at or above the threshold: scores
  int ei[kTEnt];                   // and indices
};

// fp64 block maximum M_j = log sum_{v in j} e^{z_v/tau} + G_j by one warp
// (four entries a lane); -inf for a block with no finite entry.
template <typename TIn>
__device__ double block_max64(const TIn* row, int V, int j, double tau64, const Stream& sblk,
                              uint32_t rid) {
  const int lane = threadIdx.x & 31;
  const int v0 = j * kTBlk + 4 * lane;
  double a[4];
  double m = -INFINITY;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    a[t] = v0 + t < V ? (double)ld_elem<TIn>(row, v0 + t) / tau64 : -INFINITY;
    m = fmax(m, a[t]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (!(m > -INFINITY)) return -INFINITY;
  double sum = 0.0;
#pragma unroll
  for (int t = 0; t < 4; ++t) sum += exp(a[t] - m);
  sum = warp_sum_d(sum);
  const U4 w = sblk.at((uint32_t)(j >> 2), rid);
  return m + log(sum) + gumbel_f64(uniform_f64(word_of(w, j & 3)));
}

// The k largest block maxima of the row (kept blocks and their fp64 maxima
// into sm.keep / sm.keepM / sm.nkeep).  Every thread of the CTA calls it.
template <typename TIn>
__device__ __noinline__ void topk_keep_blocks(TopkSmem& sm, const TIn* row, int V, int nb, int k,
                                              double tau64, const Stream& sblk, uint32_t rid,
                                              bool rowbad) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---------------- blocks: the k largest maxima
  float lo_t = -INFINITY;  // this thread's best lower bound
  for (int j = tid; j < nb; j += kTThreads) lo_t = fmaxf(lo_t, sm.bs[j] - sm.bd[j]);
  const float T = cta_kth_largest(lo_t, k, sm.kbuf);  // (syncs the CTA)
  if (!rowbad) {
    for (int j = tid; j < nb; j += kTThreads) {
      if (sm.bs[j] > -INFINITY && sm.bs[j] + sm.bd[j] >= T) {
        const int pos = atomicAdd(&sm.ncand, 1);
        if (pos < kTCand) sm.cblk[pos] = j;
        else atomicOr(&sm.flag, 2);
      }
    }
  }
  __syncthreads();
  const int nc = min(sm.ncand, kTCand);
  const bool overflow = (sm.flag & 2) != 0;
  // fp32 ranks of the candidates (score, then lower block); bounds decide
  if (!rowbad && !overflow && tid < nc) {
    const int j = sm.cblk[tid];
    const float sj = sm.bs[j];
    int rk = 0;
    for (int c = 0; c < nc; ++c) {
      const int o = sm.cblk[c];
      const float so = sm.bs[o];
      rk += (so > sj || (so == sj && o < j)) ? 1 : 0;
    }
    sm.crank[tid] = rk;
    if (rk < k) atomicMin(&sm.lo_ord, f2ord(sj - sm.bd[j]));
    else atomicMax(&sm.hi_ord, f2ord(sj + sm.bd[j]));
  }
  __syncthreads();
  if (!rowbad) {
    const bool settled = !overflow && ord2f(sm.lo_ord) > ord2f(sm.hi_ord);
    if (settled) {
      // the kept blocks: the k best; their fp64 maxima, a warp each
      if (tid < nc && sm.crank[tid] < k) sm.keep[sm.crank[tid]] = sm.cblk[tid];
      if (tid == 0) sm.nkeep = min(nc, k);
      __syncthreads();
      for (int q = warp; q < sm.nkeep; q += kTWarps) {
        const double m64 = block_max64<TIn>(row, V, sm.keep[q], tau64, sblk, rid);
        if (lane == 0) sm.keepM[q] = m64;
      }
    } else if (!overflow) {
      // fp64 maxima of the candidates, ranked exactly (score, then lower block)
      for (int c = warp; c < nc; c += kTWarps) {
        const double m64 = block_max64<TIn>(row, V, sm.cblk[c], tau64, sblk, rid);
        if (lane == 0) sm.cM[c] = m64;
      }
      __syncthreads();
      if (tid < nc) {
        const int j = sm.cblk[tid];
        const double sj = sm.cM[tid];
        int rk = 0;
        for (int c = 0; c < nc; ++c) {
          const int o = sm.cblk[c];
          const double so = sm.cM[c];
          rk += (so > sj || (so == sj && o < j)) ? 1 : 0;
        }
        if (rk < k && sj > -INFINITY) {
          sm.keep[rk] = j;
          sm.keepM[rk] = sj;
        }
      }
      if (tid == 0) {
        int n = 0;
        for (int c = 0; c < nc; ++c) n += sm.cM[c] > -INFINITY ? 1 : 0;
        sm.nkeep = min(n, k);
      }
    } else {
      // more candidates than the table holds (ties flooding the bound):
      // fp64 maxima of every block (in the entry table), k rounds of arg-max
      for (int j = warp; j < nb; j += kTWarps) {
        const double m64 = block_max64<TIn>(row, V, j, tau64, sblk, rid);
        if (lane == 0) sm.es[j] = m64;
      }
      __syncthreads();
      if (warp == 0) {
        int taken = 0;
        for (int q = 0; q < k; ++q) {
          double best = -INFINITY;
          int bi = 0x7FFFFFFF;
          for (int j = lane; j < nb; j += 32) {
            bool used = false;
            for (int p = 0; p < taken; ++p) used |= sm.keep[p] == j;
            if (!used) c64_merge(best, bi, sm.es[j], j);
          }
          warp_c64(best, bi);
          if (bi == 0x7FFFFFFF || !(best > -INFINITY)) break;
          if (lane == 0) {
            sm.keep[taken] = bi;
            sm.keepM[taken] = best;
          }
          __syncwarp();
          ++taken;
        }
        if (lane == 0) sm.nkeep = taken;
      }
    }
  }
  __syncthreads();
}

// Entry scores of the kept blocks conditioned on their maxima, fp64, a warp
// per block; those at or above the smallest kept maximum go to sm.es / sm.ei.
template <typename TIn>
__device__ __noinline__ void topk_kept_entries(TopkSmem& sm, const TIn* row, int V, int k,
                                               double tau64, const Stream& sent, uint32_t rid,
                                               bool rowbad) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // ---------------- entries of the kept blocks (fp64), a warp per block
  const int nk = rowbad ? 0 : sm.nkeep;
  double Tm = INFINITY;  // the k-th largest score is no smaller than the smallest kept maximum
  for (int q = 0; q < nk; ++q) Tm = fmin(Tm, sm.keepM[q]);
  if (nk < k) Tm = -INFINITY;  // fewer live blocks than k: every entry counts
  for (int q = warp; q < nk; q += kTWarps) {
    const int j = sm.keep[q];
    const double Mj = sm.keepM[q];
    const int v0 = j * kTBlk + 4 * lane;
    double h[4];
    U4 w = U4{0u, 0u, 0u, 0u};
    if (v0 < V) w = sent.at((uint32_t)(v0 >> 2), rid);
    double Z = -INFINITY;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float zv = v0 + t < V ? ld_elem<TIn>(row, v0 + t) : -INFINITY;
      h[t] = zv > -INFINITY ? (double)zv / tau64 + gumbel_f64(uniform_f64(word_of(w, t))) : -INFINITY;
      Z = fmax(Z, h[t]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Z = fmax(Z, __shfl_xor_sync(0xffffffffu, Z, o));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (!(h[t] > -INFINITY)) continue;
      // S = -log(e^{-M} - e^{-Z} + e^{-h}) = M - softplus(M - h + log(1 - e^{h - Z}))
      double sv = Mj;
      const double d = h[t] - Z;
      if (d != 0.0) {
        const double u = Mj - h[t] + log(-expm1(d));
        sv = Mj - (fmax(u, 0.0) + log1p(exp(-fabs(u))));
      }
      if (sv >= Tm) {
        const int pos = atomicAdd(&sm.ne, 1);
        sm.es[pos] = sv;
        sm.ei[pos] = v0 + t;
      }
    }
  }
}

template <typename TIn>
__global__ void __launch_bounds__(kTThreads, 2) topk_block_kernel(
    const TIn* __restrict__ z, int rows, int V, int64_t ld, int k, float inv_tau, float cT,
    double tau64, uint64_t seed, uint64_t round, int vec, int32_t* __restrict__ idx_out,
    float* __restrict__ score_out, float* __restrict__ logp_out, uint32_t* dev_err) {
  constexpr int kUnroll = 1;  // tiles in flight: 64 bytes a lane (bf16)
  extern __shared__ __align__(16) unsigned char topk_smem[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = (V + kTTile - 1) / kTTile;
  const int nb = (V + kTBlk - 1) / kTBlk;
  const Stream sblk(seed, round, SD_STREAM_TOPK_BLOCK);
  const Stream sent(seed, round, SD_STREAM_TOPK_DENSE);
  const uint64_t pol = policy_evict_first();
  const bool vecok = vec != 0;

  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const TIn* row = z + (int64_t)r * ld;
    const uint32_t rid = (uint32_t)r;
    if (tid == 0) {
      sm.flag = 0;
      sm.ncand = 0;
      sm.ne = 0;
      sm.lo_ord = f2ord(INFINITY);
      sm.hi_ord = f2ord(-INFINITY);
    }
    __syncthreads();
    // ---------------- pass over the row: block maxima and the lse partials
    float M = -INFINITY, S = 0.f, R = -INFINITY;
    bool bad = false;
    int nbuf = 0;
    auto score_blocks = [&]() {
      __syncwarp();
      const int q = lane >> 3, h = lane & 7;  // lane: block h of buffered tile q
      if (q < nbuf) {
        float sb = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) sb += sm.part[warp][q][4 * h + i];
        const float rb = sm.ref[warp][q];
        const int j = 8 * sm.tile[warp][q] + h;
        float mj = -INFINITY, dj = 0.f;
        if (sb > 0.f && sb < INFINITY) {
          if (rb > M) {
            S = (M == -INFINITY) ? 0.f : S * ex2((M - rb) * cT);
            M = rb;
          }
          S += sb * ex2((rb - M) * cT);
          // ln(sum) from exps whose arguments were rounded in fp32 (2^-24 of
          // |R c| and of |t| <= 130), ex2.approx and the 128-term sum
          const U4 w = sblk.at((uint32_t)(j >> 2), rid);
          const float g32 = gumbel_f32(uniform_f32(word_of(w, j & 3)));
          const float lam = logf(sb) + rb * inv_tau;
          mj = lam + g32;
          dj = score_err(lam, g32) + 2e-5f + 2e-7f * fabsf(rb * cT);
        }
        // a block more than ~87 nats below R flushed to 0: the block holding
        // R beats it by more than block noise can span (< 20), so -inf is safe
        if (j < nb) {
          sm.bs[j] = mj;
          sm.bd[j] = dj;
        }
      }
      __syncwarp();
      nbuf = 0;
    };
    for (int t0 = warp; t0 < nt; t0 += kUnroll * kTWarps) {
      Raw8<TIn> raw[kUnroll][4];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int t = t0 + u * kTWarps;
        if (t < nt) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            raw[u][h] = load8_raw<TIn>(row, t * kTTile + 32 * lane + 8 * h, V, vecok, pol);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int t = t0 + u * kTWarps;
        if (t >= nt) break;  // warp-uniform
        float mq[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float zz[8];
          unpack8<TIn>(raw[u][h], zz);
          mq[h] = fmax_nan(fmax_nan(fmax_nan(zz[0], zz[1]), fmax_nan(zz[2], zz[3])),
                           fmax_nan(fmax_nan(zz[4], zz[5]), fmax_nan(zz[6], zz[7])));
        }
        const float m8 = fmax_nan(fmax_nan(mq[0], mq[1]), fmax_nan(mq[2], mq[3]));
        bad |= m8 != m8;
        float mt = m8 != m8 ? -INFINITY : m8;
        asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(mt));
        bad |= mt == INFINITY;
        R = fmaxf(R, mt);
        float sl = 0.f;
        if (R > -INFINITY && R < INFINITY) {
          const float2 c2 = f2(cT), n2 = f2(-R * cT);
          float2 acc = f2(0.f), acc2 = f2(0.f);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            float zz[8];
            unpack8<TIn>(raw[u][h], zz);
#pragma unroll
            for (int i = 0; i < 8; i += 4) {
              const float2 ta = __ffma2_rn(make_float2(zz[i], zz[i + 1]), c2, n2);
              const float2 tb = __ffma2_rn(make_float2(zz[i + 2], zz[i + 3]), c2, n2);
              acc = __fadd2_rn(acc, make_float2(ex2(ta.x), ex2(ta.y)));
              acc2 = __fadd2_rn(acc2, make_float2(ex2(tb.x), ex2(tb.y)));
            }
          }
          sl = (acc.x + acc.y) + (acc2.x + acc2.y);
        }
        sm.part[warp][nbuf][lane] = sl;
        if (lane == 0) {
          sm.ref[warp][nbuf] = R;
          sm.tile[warp][nbuf] = t;
        }
        if (++nbuf == kTBuf) score_blocks();
      }
    }
    score_blocks();
    {
      const float Mw = warp_max(M);
      float Sw = (M == -INFINITY) ? 0.f : S * ex2((M - Mw) * cT);
      Sw = warp_sum(Sw);
      if (lane == 0) {
        sm.m[warp] = Mw;
        sm.s[warp] = Sw;
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&sm.flag, 1);
    }
    __syncthreads();
    if (warp == 0) {
      const float pm = lane < kTWarps ? sm.m[lane] : -INFINITY;
      const float ps = lane < kTWarps ? sm.s[lane] : 0.f;
      const float MM = warp_max(pm);
      const double tt = (lane < kTWarps && pm > -INFINITY) ? (double)ps * (double)ex2((pm - MM) * cT) : 0.0;
      const double SS = warp_sum_d(tt);
      if (lane == 0) {
        sm.lse = (double)MM / tau64 + log(SS);
        if (!(MM > -INFINITY)) sm.flag |= 1;  // every entry -inf
      }
    }
    __syncthreads();
    const bool rowbad = (sm.flag & 1) != 0;
    topk_keep_blocks<TIn>(sm, row, V, nb, k, tau64, sblk, rid, rowbad);
    __syncthreads();
    topk_kept_entries<TIn>(sm, row, V, k, tau64, sent, rid, rowbad);
    __syncthreads();
    const int ne = rowbad ? 0 : sm.ne;
    for (int e = tid; e < ne; e += kTThreads) {  // ranks by counting (score, then lower index)
      const double se = sm.es[e];
      const int ve = sm.ei[e];
      int rk = 0;
      for (int c = 0; c < ne; ++c) {
        const double so = sm.es[c];
        rk += (so > se || (so == se && sm.ei[c] < ve)) ? 1 : 0;
      }
      if (rk < k) {
        idx_out[(int64_t)r * k + rk] = ve;
        if (score_out) score_out[(int64_t)r * k + rk] = (float)se;
        if (logp_out)
          logp_out[(int64_t)r * k + rk] = (float)((double)ld_elem<TIn>(row, ve) / tau64 - sm.lse);
      }
    }
    if (tid >= min(ne, k) && tid < k) {  // ranks with no finite entry left
      idx_out[(int64_t)r * k + tid] = -1;
      if (score_out) score_out[(int64_t)r * k + tid] = NAN;
      if (logp_out) logp_out[(int64_t)r * k + tid] = NAN;
    }
    if (rowbad && tid == 0) raise_err(dev_err, SD_DEV_NONFINITE);
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

extern "C" sd_status gumbel_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld, int k,
                                 float tau, uint64_t seed, uint64_t round, int32_t* idx_out,
                                 float* score_out, float* logp_out, uint32_t* dev_err,
                                 void* stream) {
  if (rows < 0 || V < 1 || ld < V || k < 1 || k > kTopkMax || k > V ||
      !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (V > kTMaxBlocks * kTBlk) return SD_ERR_UNSUPPORTED;
  if (rows == 0) return SD_OK;
  if (!z || !idx_out) return SD_ERR_INVALID_ARG;
  const int esize = dt == SD_BF16 ? 2 : 4;
  const int vec = ((uintptr_t)z % 16 == 0) && ((ld * esize) % 16 == 0);
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const int grid = rows < 2 * nsm ? rows : 2 * nsm;  // persistent: two CTAs per SM
  const int smem = (int)sizeof(TopkSmem);
  const float inv_tau = (float)(1.0 / (double)tau);
  const float cT = (float)(1.4426950408889634 / (double)tau);
  cudaStream_t s = (cudaStream_t)stream;
  auto launch = [&](auto kern, const auto* zp) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return;
    kern<<<grid, kTThreads, smem, s>>>(zp, rows, V, ld, k, inv_tau, cT, (double)tau, seed, round, vec,
                                       idx_out, score_out, logp_out, dev_err);
  };
  if (dt == SD_BF16) launch(topk_block_kernel<uint16_t>, (const uint16_t*)z);
  else launch(topk_block_kernel<float>, (const float*)z);
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
