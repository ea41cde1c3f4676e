// The draft step's sampler: one token per draft row drawn from the drafter's
// distribution q = softmax(zD / tau), with log q of the draw.
//
// "Faster LLM Inference via Sequential Monte Carlo", section 2 (draft step):
// the draft model extends each particle by sampling its own distribution;
// STAND, Methodology item 1: drafting samples the distribution rather than
// taking its argmax.  The sampler is an exact two-level Gumbel-max: the block
// of 128 entries j* = argmax_j (log sum_{v in j} e^{z_v/tau} + G_j), G from
// Philox stream 10, then the entry v* = argmax_{v in j*} (z_v/tau + g_v), g
// from stream 8 (row id row0 + r, counter entry j or v, ties to the lower
// index).  It samples q exactly, like a one-level Gumbel-max, but needs noise
// for the blocks and one block's entries only -- so one pass over the row
// does it, at HBM speed.
//
// Kernel: persistent CTAs of 512 threads (two per SM) take rows in turn.  A
// warp takes tiles of 1024 entries (32 per lane, four 16-byte loads of bf16);
// every exp is relative to the warp's running max R (one redux per tile, so no
// exp can overflow), and each lane parks the sum of its 32 exps in shared
// memory with the tile's R.  Every 4 tiles the warp scores their 32 blocks one
// per lane: the block's sum from its 4 lanes' partials, then
// ln(sum) + R/tau + G_j with fp32 error bounds, folded into the row's (max,
// sum) partial for the log-sum-exp.  The CTA merges the block candidates; a
// block decision the fp32 bounds do not settle is redone in fp64 over the
// row (rare).  One warp then draws the entry inside the chosen block (fp32
// bounds, fp64 on a near-tie) and writes the token and log q.
#include <cuda_runtime.h>

#include "rowload.cuh"
#include "rows.cuh"

namespace smcsd {

constexpr int kDThreads = 512;  // 16 warps
constexpr int kDBlk = 128;      // entries per block of the draw
constexpr int kDBuf = 4;        // tiles a warp buffers before scoring their blocks
constexpr int kDTile = 1024;    // entries per warp tile: 32 per lane, eight blocks

struct DraftSmem {
  float part[kDThreads / 32][kDBuf][32];  // per lane: sum of its 32 exps, relative to the tile's R
  float ref[kDThreads / 32][kDBuf];       // the tile's reference R (the warp's running max)
  int tile[kDThreads / 32][kDBuf];
  Cand cand[kDThreads / 32];
  float m[kDThreads / 32], s[kDThreads / 32];
  int flag;
  int block;
  double lse;
  double s64[kDThreads / 32];
  int i64[kDThreads / 32];
};

template <typename TIn>
__global__ void __launch_bounds__(kDThreads, 2) draft_block_kernel(
    const TIn* __restrict__ z, int rows, int V, int64_t ld, float inv_tau, float cT, double tau64,
    uint64_t seed, uint64_t round, uint32_t row0, int vec, int32_t* __restrict__ tokens_out,
    float* __restrict__ logq_out, uint32_t* dev_err) {
  constexpr int kDUnroll = 1;  // tiles in flight: 64 bytes a lane (bf16)
  __shared__ DraftSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = kDThreads / 32;
  const int nt = (V + kDTile - 1) / kDTile;  // tiles of 512 entries (four blocks)
  const Stream sblk(seed, round, SD_STREAM_DRAFT_BLOCK);
  const Stream sent(seed, round, SD_STREAM_DRAFT);
  const uint64_t pol = policy_evict_first();
  const bool vecok = vec != 0;

  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const TIn* row = z + (int64_t)r * ld;
    const uint32_t rid = row0 + (uint32_t)r;
    if (tid == 0) sm.flag = 0;
    __syncthreads();
    Cand best = cand_empty();
    float M = -INFINITY, S = 0.f;  // this lane's (max, sum) partial of the row
    float R = -INFINITY;           // the warp's running max: every exp is taken relative to it
    bool bad = false;
    int nbuf = 0;  // tiles in this warp's buffer (warp-uniform)
    // Scores the buffered tiles' blocks, one block per lane: its sum from the
    // 16 lanes' partials, the row's (max, sum) partial, and the block's score
    // ln(sum) + R/tau + G_j with fp32 bounds (ln(sum) from exps whose
    // arguments were rounded in fp32: 2^-24 of |R c| and of |t| <= 130;
    // ex2.approx; the 128-term sum).  A block more than ~87 nats below R has
    // flushed to 0 and is dropped: the block holding R beats it by more than
    // the block noise can span (< 20).
    auto score_blocks = [&]() {
      __syncwarp();
      const int q = lane >> 3, h = lane & 7;  // lane: block h of buffered tile q
      if (q < nbuf) {
        float sb = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) sb += sm.part[warp][q][4 * h + i];
        const float rb = sm.ref[warp][q];
        if (sb > 0.f && sb < INFINITY) {
          if (rb > M) {
            S = (M == -INFINITY) ? 0.f : S * ex2((M - rb) * cT);
            M = rb;
          }
          S += sb * ex2((rb - M) * cT);
          const int j = 8 * sm.tile[warp][q] + h;
          const U4 w = sblk.at((uint32_t)(j >> 2), rid);
          const float g32 = gumbel_f32(uniform_f32(word_of(w, j & 3)));
          const float lam = logf(sb) + rb * inv_tau;
          const float sc = lam + g32;
          const float d = score_err(lam, g32) + 2e-5f + 2e-7f * fabsf(rb * cT);
          Cand c;
          c.s = sc;
          c.lo = sc - d;
          c.hi = sc + d;
          c.ohi = -INFINITY;
          c.idx = j;
          c.aux = -1;
          c.pad1 = c.pad2 = 0;
          best = cand_merge(best, c);
        }
      }
      __syncwarp();
      nbuf = 0;
    };
    for (int t0 = warp; t0 < nt; t0 += kDUnroll * nw) {
      Raw8<TIn> raw[kDUnroll][4];
#pragma unroll
      for (int u = 0; u < kDUnroll; ++u) {
        const int t = t0 + u * nw;
        if (t < nt) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            raw[u][h] = load8_raw<TIn>(row, t * kDTile + 32 * lane + 8 * h, V, vecok, pol);
        }
      }
#pragma unroll
      for (int u = 0; u < kDUnroll; ++u) {
        const int t = t0 + u * nw;
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
        if (++nbuf == kDBuf) score_blocks();
      }
    }
    score_blocks();
    // ---------------- CTA: the row's lse, the block
    best = warp_cand(best);
    const float Mw = warp_max(M);
    float Sw = (M == -INFINITY) ? 0.f : S * ex2((M - Mw) * cT);
    Sw = warp_sum(Sw);
    if (lane == 0) {
      sm.cand[warp] = best;
      sm.m[warp] = Mw;
      sm.s[warp] = Sw;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&sm.flag, 1);
    __syncthreads();
    if (warp == 0) {
      const float pm = lane < nw ? sm.m[lane] : -INFINITY;
      const float ps = lane < nw ? sm.s[lane] : 0.f;
      const float MM = warp_max(pm);
      const double tt = (lane < nw && pm > -INFINITY) ? (double)ps * (double)ex2((pm - MM) * cT) : 0.0;
      const double SS = warp_sum_d(tt);
      Cand c = lane < nw ? sm.cand[lane] : cand_empty();
      c = warp_cand(c);
      if (lane == 0) {
        sm.lse = (double)MM / tau64 + log(SS);
        if (!(MM > -INFINITY)) sm.flag |= 1;  // every entry -inf
        // -1: settle the block in fp64 below; -2: no block (a bad row)
        sm.block = c.idx == 0x7FFFFFFF ? -2 : (c.ohi < c.lo ? c.idx : -1);
      }
    }
    __syncthreads();
    const bool rowbad = (sm.flag & 1) != 0;
    int jb = sm.block;
    if (!rowbad && jb == -1) {
      // fp64 block scores over the whole row (rare): lambda_j = log sum exp(z/tau)
      const int nb = (V + kDBlk - 1) / kDBlk;
      double bs = -INFINITY;
      int bi = 0x7FFFFFFF;
      for (int j = tid; j < nb; j += kDThreads) {
        const int v0 = j * kDBlk, v1 = min(v0 + kDBlk, V);
        double m = -INFINITY;
        for (int v = v0; v < v1; ++v) m = fmax(m, (double)ld_elem<TIn>(row, v) / tau64);
        if (!(m > -INFINITY)) continue;
        double sum = 0.0;
        for (int v = v0; v < v1; ++v) sum += exp((double)ld_elem<TIn>(row, v) / tau64 - m);
        const U4 w = sblk.at((uint32_t)(j >> 2), rid);
        c64_merge(bs, bi, m + log(sum) + gumbel_f64(uniform_f64(word_of(w, j & 3))), j);
      }
      warp_c64(bs, bi);
      if (lane == 0) {
        sm.s64[warp] = bs;
        sm.i64[warp] = bi;
      }
      __syncthreads();
      if (warp == 0) {
        double s2 = lane < nw ? sm.s64[lane] : -INFINITY;
        int i2 = lane < nw ? sm.i64[lane] : 0x7FFFFFFF;
        warp_c64(s2, i2);
        if (lane == 0) sm.block = i2 == 0x7FFFFFFF ? -2 : i2;
      }
      __syncthreads();
      jb = sm.block;
    }
    // ---------------- the entry inside block jb (warp 0)
    if (warp == 0) {
      int x = -1;
      if (!rowbad && jb >= 0) {
        const int v0 = jb * kDBlk + 4 * lane;
        float zz[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        U4 w = U4{0u, 0u, 0u, 0u};
        Cand ce = cand_empty();
        if (v0 < V) {
          w = sent.at((uint32_t)(v0 >> 2), rid);
#pragma unroll
          for (int q = 0; q < 4; ++q) zz[q] = v0 + q < V ? ld_elem<TIn>(row, v0 + q) : -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (zz[q] > -INFINITY)
              ce = cand_merge(ce, bonus_cand_a(zz[q] * inv_tau, uniform_f32(word_of(w, q)), v0 + q));
        }
        ce = warp_cand(ce);
        if (ce.idx != 0x7FFFFFFF && ce.ohi < ce.lo) {
          x = ce.idx;
        } else {
          double bs = -INFINITY;
          int bi = 0x7FFFFFFF;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (zz[q] > -INFINITY)
              c64_merge(bs, bi, (double)zz[q] / tau64 + gumbel_f64(uniform_f64(word_of(w, q))), v0 + q);
          warp_c64(bs, bi);
          x = bi == 0x7FFFFFFF ? -1 : bi;
        }
      }
      if (lane == 0) {
        tokens_out[r] = x;
        if (logq_out)
          logq_out[r] = x >= 0 ? (float)((double)ld_elem<TIn>(row, x) / tau64 - sm.lse) : NAN;
        if (rowbad) raise_err(dev_err, SD_DEV_NONFINITE);
      }
    }
    __syncthreads();
  }
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status sd_draft_sample(const void* zD, sd_dtype dt, int rows, int V, int64_t ld,
                                     float tau, uint64_t seed, uint64_t round, uint32_t row0,
                                     int32_t* tokens_out, float* logq_out, uint32_t* dev_err,
                                     void* stream) {
  if (rows < 0 || V < 1 || ld < V || !(tau > 0.f && tau < INFINITY)) return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (rows == 0) return SD_OK;
  if (!zD || !tokens_out) return SD_ERR_INVALID_ARG;
  if ((uint64_t)row0 + (uint64_t)rows > 0x100000000ull) return SD_ERR_INVALID_ARG;
  const int esize = dt == SD_BF16 ? 2 : 4;
  const int vec = ((uintptr_t)zD % 16 == 0) && ((ld * esize) % 16 == 0);
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const float inv_tau = (float)(1.0 / (double)tau);
  const float cT = (float)(1.4426950408889634 / (double)tau);
  cudaStream_t s = (cudaStream_t)stream;
  const int grid = rows < 2 * nsm ? rows : 2 * nsm;  // persistent: two CTAs per SM
  if (dt == SD_BF16)
    draft_block_kernel<uint16_t><<<grid, kDThreads, 0, s>>>(
        (const uint16_t*)zD, rows, V, ld, inv_tau, cT, (double)tau, seed, round, row0, vec,
        tokens_out, logq_out, dev_err);
  else
    draft_block_kernel<float><<<grid, kDThreads, 0, s>>>((const float*)zD, rows, V, ld, inv_tau, cT,
                                                         (double)tau, seed, round, row0, vec,
                                                         tokens_out, logq_out, dev_err);
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}
