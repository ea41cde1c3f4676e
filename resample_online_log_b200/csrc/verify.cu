// Standard speculative-decoding verification (N = 1), row-parallel.
//
// What it computes (include/smcsd.h, sd_verify_reject): per sequence, K
// drafted tokens are checked in order against the target; the first rejection
// discards the rest and draws one token from the residual max(p - q, 0); if all
// K are accepted a bonus token is drawn from the target row K+1.  Sources:
// "Faster LLM Inference via Sequential Monte Carlo", section 1 (standard SD,
// rejection, KV rollback); METASD section 1 (background) and section 2 (TV
// block divergence reported per position).  Both draws are exact two-level
// Gumbel-max draws over blocks of 128 entries (the block by its log-mass plus
// block noise, then the entry inside it).
//
// Design (B200, sm_100a).  Every (sequence, position) row is independent until
// the first rejection is known, so all rows are scored at once:
//   verify_rows_kernel: persistent CTAs of 512 threads (two per SM) take rows
//     in turn, streaming each row twice with 16-byte loads, several in flight:
//     pass 1 (HBM, tiles of 256 entries, 8 per lane; the row stays in L2):
//       the log-sum-exp of the target and
//       draft rows, exps relative to each lane's running max (the warp
//       combines its lanes once, after the row); the accept test
//       u q(x) < p(x) in fp64;
//     pass 2 (L2, tiles of 512 entries: 16 per lane): p and q per entry,
//       TV = 1/2 sum |p - q|, and the block masses the row's draw needs --
//       residual sum max(p - q, 0) after a rejection (with the error bound
//       7.7e-6 (p + q) per entry), target mass on the last row -- parked per
//       lane and scored per block one per lane every 8 tiles; the CTA merges
//       the block candidates (a near-tie, or no residual mass in fp32, goes to
//       fp64 over the row's blocks), and one warp draws the entry inside the
//       chosen block in fp64.
//     Each row's outcome is encoded in its own slot of out_tokens.
//   verify_finalize_kernel: per sequence, the first rejection decides the
//     accepted length and the emitted tokens; slots past it become -1.
// Work for rows past the first rejection is spent speculatively; nothing but
// the outputs is written to global memory.
#include <cuda_runtime.h>

#include "rowload.cuh"
#include "rows.cuh"

namespace smcsd {

constexpr int kVThreads = 512;
constexpr int kVPerSM = 2;
constexpr int kVWarps = kVThreads / 32;
constexpr int kVBlk = 128;
constexpr int kVBuf = 8;   // pass-2 tiles a warp buffers before scoring their blocks
constexpr int kVTile2 = 512;  // pass-2 warp tile: 16 entries a lane, four blocks

struct VerifyArgs {
  const void* zT;
  const void* zD;
  int64_t ld;
  int B, V, K, R;
  int vec;  // 16-byte loads allowed
  float inv_tau, cT;
  double tau64;
  const int32_t* draft;
  uint64_t seed, round;
  int32_t* out_tokens;
  int32_t* acc_len;
  float* tv_out;
  uint32_t* dev_err;
};

struct VSmem {
  float part[kVWarps][kVBuf][32];  // per lane: its 16 entries' block mass (residual or target)
  float pq[kVWarps][kVBuf][32];    // per lane: its 16 entries' p + q (residual error bounds)
  int tile[kVWarps][kVBuf];
  float rm[2][kVWarps], rs[2][kVWarps];  // lse partials (target, draft)
  float tv[kVWarps];
  Cand cand[kVWarps];
  double s64[kVWarps];
  int i64[kVWarps];
  double lse[2];
  int flag;   // bit 0: target bad, 1: draft bad, 2: accept, 3: draft token out of range
  int block;  // chosen block, -1: settle in fp64, -2: none
};

// Encoding of a row's outcome in its out_tokens slot, decoded by the finalize
// kernel: an accepted draft keeps its id (>= 0); a row whose rows are not
// finite is -1; a rejection is -2 - (token | oob << 29 | zero_residual << 30).
constexpr int kCodeBad = -1;
__device__ __forceinline__ int encode_reject(int tok, bool oob, bool zr) {
  return -2 - (tok | (oob ? (1 << 29) : 0) | (zr ? (1 << 30) : 0));
}

// fp64 log-weight of entry v for the row's draw: mode 1 the residual
// log max(p - q, 0) (-inf where zero), else the target's z/tau.
template <typename TIn>
__device__ __forceinline__ double draw_weight64(const TIn* rT, const TIn* rD, int v, int mode,
                                                double tau64, double lseT, double lseD) {
  const double a = (double)ld_elem<TIn>(rT, v) / tau64;
  if (mode != 1) return a;
  const double r = exp(a - lseT) - exp((double)ld_elem<TIn>(rD, v) / tau64 - lseD);
  return r > 0.0 ? log(r) : -INFINITY;
}

// The block of the draw in fp64 over the whole row (a near-tie the fp32 bounds
// could not settle, or no residual mass in fp32; rare): every thread takes
// whole blocks.  Returns the block, or -1 if no block has positive mass.
template <typename TIn>
__device__ __noinline__ int exact_block(VSmem& sm, const TIn* rT, const TIn* rD, int V, int mode,
                                        double tau64, double lseT, double lseD, const Stream& sb,
                                        uint32_t rid) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nb = (V + kVBlk - 1) / kVBlk;
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int j = tid; j < nb; j += kVThreads) {
    const int v0 = j * kVBlk, v1 = min(v0 + kVBlk, V);
    double m = -INFINITY;
    for (int v = v0; v < v1; ++v) m = fmax(m, draw_weight64<TIn>(rT, rD, v, mode, tau64, lseT, lseD));
    if (!(m > -INFINITY)) continue;
    double sum = 0.0;
    for (int v = v0; v < v1; ++v) sum += exp(draw_weight64<TIn>(rT, rD, v, mode, tau64, lseT, lseD) - m);
    const U4 w = sb.at((uint32_t)(j >> 2), rid);
    c64_merge(best, bi, m + log(sum) + gumbel_f64(uniform_f64(word_of(w, j & 3))), j);
  }
  warp_c64(best, bi);
  if (lane == 0) {
    sm.s64[warp] = best;
    sm.i64[warp] = bi;
  }
  __syncthreads();
  if (warp == 0) {
    best = lane < kVWarps ? sm.s64[lane] : -INFINITY;
    bi = lane < kVWarps ? sm.i64[lane] : 0x7FFFFFFF;
    warp_c64(best, bi);
    if (lane == 0) sm.block = bi == 0x7FFFFFFF ? -1 : bi;
  }
  __syncthreads();
  return sm.block;
}

// The entry inside block j, in fp64 (one warp, four entries a lane).
template <typename TIn>
__device__ __noinline__ int exact_in_block(const TIn* rT, const TIn* rD, int V, int j, int mode,
                                           double tau64, double lseT, double lseD,
                                           const Stream& se, uint32_t rid) {
  const int lane = threadIdx.x & 31;
  const int v0 = j * kVBlk + 4 * lane;
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  if (v0 < V) {
    const U4 w = se.at((uint32_t)(v0 >> 2), rid);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (v0 + t >= V) break;
      const double wv = draw_weight64<TIn>(rT, rD, v0 + t, mode, tau64, lseT, lseD);
      if (wv > -INFINITY) c64_merge(best, bi, wv + gumbel_f64(uniform_f64(word_of(w, t))), v0 + t);
    }
  }
  warp_c64(best, bi);
  return bi == 0x7FFFFFFF ? -1 : bi;
}

// Pass 1 over a row pair (HBM; the rows are left in L2 for pass 2): each lane
// keeps its own running max and sum of exps relative to it for the target and
// draft rows (no cross-lane step inside the loop), then the warp combines
// them; the warp's (max, sum) pairs and NaN / +inf flags go to shared memory.
template <typename TIn>
__device__ __noinline__ void verify_pass1(VSmem& sm, const TIn* rT, const TIn* rD, int V, int nt,
                                          bool hasD, float cT, bool vec, uint64_t keep) {
  constexpr int kUnroll = sizeof(TIn) == 2 ? 2 : 1;  // tiles in flight per tensor (32 bytes a lane)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float RT = -INFINITY, RD = -INFINITY, ST = 0.f, SD = 0.f;
  bool badT = false, badD = false;
  for (int t0 = warp; t0 < nt; t0 += kUnroll * kVWarps) {
    Raw8<TIn> xt[kUnroll], xd[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = t0 + u * kVWarps;
      if (t < nt) {
        xt[u] = load8_raw<TIn>(rT, t * 256 + 8 * lane, V, vec, keep);
        if (hasD) xd[u] = load8_raw<TIn>(rD, t * 256 + 8 * lane, V, vec, keep);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (t0 + u * kVWarps >= nt) break;  // warp-uniform
      float zt[8], zd[8];
      unpack8<TIn>(xt[u], zt);
      float mt = fmax_nan(fmax_nan(fmax_nan(zt[0], zt[1]), fmax_nan(zt[2], zt[3])),
                          fmax_nan(fmax_nan(zt[4], zt[5]), fmax_nan(zt[6], zt[7])));
      badT |= mt != mt || mt == INFINITY;
      if (mt > RT) {
        ST = RT == -INFINITY ? 0.f : ST * ex2((RT - mt) * cT);
        RT = mt;
      }
      if (RT > -INFINITY && RT < INFINITY) {
        const float n = -RT * cT;
#pragma unroll
        for (int i = 0; i < 8; ++i) ST += ex2(fmaf(zt[i], cT, n));
      }
      if (hasD) {
        unpack8<TIn>(xd[u], zd);
        float md = fmax_nan(fmax_nan(fmax_nan(zd[0], zd[1]), fmax_nan(zd[2], zd[3])),
                            fmax_nan(fmax_nan(zd[4], zd[5]), fmax_nan(zd[6], zd[7])));
        badD |= md != md || md == INFINITY;
        if (md > RD) {
          SD = RD == -INFINITY ? 0.f : SD * ex2((RD - md) * cT);
          RD = md;
        }
        if (RD > -INFINITY && RD < INFINITY) {
          const float n = -RD * cT;
#pragma unroll
          for (int i = 0; i < 8; ++i) SD += ex2(fmaf(zd[i], cT, n));
        }
      }
    }
  }
  {
    // the warp's pair from the lanes' pairs (a lane's reference is finite or -inf)
    float MT = RT, MD = RD;
    warp_max2(MT, MD);
    float st = RT == -INFINITY ? 0.f : ST * ex2((RT - MT) * cT);
    float sd = RD == -INFINITY ? 0.f : SD * ex2((RD - MD) * cT);
    warp_sum2(st, sd);
    if (lane == 0) {
      sm.rm[0][warp] = MT;
      sm.rs[0][warp] = st;
      sm.rm[1][warp] = MD;
      sm.rs[1][warp] = sd;
    }
    if (__any_sync(0xffffffffu, badT) && lane == 0) atomicOr(&sm.flag, 1);
    if (__any_sync(0xffffffffu, badD) && lane == 0) atomicOr(&sm.flag, 2);
  }
}

// Pass 2 (L2): p and q per entry from the rows' lse (exponents LT, LD in
// log2 units), TV, and the block masses of the row's draw (mode 1 residual,
// 2 target), scored per block; the warp's TV and best block go to shared memory.
template <typename TIn>
__device__ __noinline__ void verify_pass2(VSmem& sm, const TIn* rT, const TIn* rD, int V, int nt,
                                          bool hasD, int mode, bool badTr, bool badDr, float cT,
                                          float LT, float LD, bool vec, uint64_t drop,
                                          const Stream& sblk, uint32_t rid) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float tvp = 0.f;
  Cand best = cand_empty();
  int nbuf = 0;
  auto score_blocks = [&]() {
    __syncwarp();
    const int q = lane >> 2, h = lane & 3;  // lane: block h of buffered tile q
    if (q < nbuf) {
      float m = 0.f, e = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m += sm.part[warp][q][8 * h + i];
      if (mode == 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) e += sm.pq[warp][q][8 * h + i];
        e = 7.7e-6f * e + 1e-35f;  // |fp32 r - r| <= 7.7e-6 (p + q) per entry
      }
      const int jb = 4 * sm.tile[warp][q] + h;
      if (m + e > 0.f) {
        const U4 w = sblk.at((uint32_t)(jb >> 2), rid);
        const float g32 = gumbel_f32(uniform_f32(word_of(w, jb & 3)));
        Cand c;
        if (mode == 1) {
          const float lh = logf(m + e), lm = m > 0.f ? logf(m) : -INFINITY;
          const float d = score_err(lh, g32);
          c.s = lm + g32;
          c.hi = lh + g32 + d;
          c.lo = m - e > 0.f ? logf(m - e) + g32 - d : -INFINITY;
        } else {
          // the target's block mass from exps with arguments rounded in fp32
          // (2^-24 of |z c| and of |lse log2 e|), ex2.approx and the sum
          const float lm = logf(m);
          const float d = score_err(lm, g32) + 2e-5f + 2e-7f * fabsf(LT);
          c.s = lm + g32;
          c.lo = c.s - d;
          c.hi = c.s + d;
        }
        c.ohi = -INFINITY;
        c.idx = jb;
        c.aux = -1;
        c.pad1 = c.pad2 = 0;
        best = cand_merge(best, c);
      }
    }
    __syncwarp();
    nbuf = 0;
  };
  if (hasD || mode == 2) {
    const int nt2 = (V + kVTile2 - 1) / kVTile2;
    for (int t = warp; t < nt2; t += kVWarps) {
      Raw8<TIn> xt[2], xd[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        xt[u] = load8_raw<TIn>(rT, t * kVTile2 + 16 * lane + 8 * u, V, vec, drop);
        if (hasD) xd[u] = load8_raw<TIn>(rD, t * kVTile2 + 16 * lane + 8 * u, V, vec, drop);
      }
      float bm = 0.f, bpq = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float zt[8], zd[8];
        unpack8<TIn>(xt[u], zt);
        if (hasD) unpack8<TIn>(xd[u], zd);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float p = badTr ? 0.f : ex2(fmaf(zt[i], cT, -LT));
          if (hasD) {
            const float q = badDr ? 0.f : ex2(fmaf(zd[i], cT, -LD));
            tvp += fabsf(p - q);
            bm += fmaxf(p - q, 0.f);
            bpq += p + q;
          } else {
            bm += p;
          }
        }
      }
      if (mode != 0) {
        sm.part[warp][nbuf][lane] = bm;
        if (mode == 1) sm.pq[warp][nbuf][lane] = bpq;
        if (lane == 0) sm.tile[warp][nbuf] = t;
        if (++nbuf == kVBuf) score_blocks();
      }
    }
    if (mode != 0) score_blocks();
  }
  tvp = warp_sum(tvp);
  best = warp_cand(best);
  if (lane == 0) {
    sm.tv[warp] = tvp;
    sm.cand[warp] = best;
  }
}

template <typename TIn>
__global__ void __launch_bounds__(kVThreads, kVPerSM) verify_rows_kernel(const VerifyArgs a) {
  extern __shared__ __align__(16) unsigned char vsmem[];
  VSmem& sm = *reinterpret_cast<VSmem*>(vsmem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int V = a.V;
  const int nt = (V + 255) / 256;
  const float cT = a.cT;
  const bool vec = a.vec != 0;
  const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
  const int64_t nrows = (int64_t)a.B * a.R;

  for (int64_t j = blockIdx.x; j < nrows; j += gridDim.x) {
    const int b = (int)(j / a.R), k = (int)(j % a.R);
    const bool hasD = k < a.K;
    const TIn* rT = (const TIn*)a.zT + j * a.ld;
    const TIn* rD = hasD ? (const TIn*)a.zD + ((int64_t)b * a.K + k) * a.ld : rT;
    if (tid == 0) sm.flag = 0;
    __syncthreads();

    verify_pass1<TIn>(sm, rT, rD, V, nt, hasD, cT, vec, keep);
    __syncthreads();
    if (warp == 0) {  // lse of both rows (fp64 combine): half-warp 0 the target, 1 the draft
      const int h = lane >> 4, w = lane & 15;
      const float pm = w < kVWarps ? sm.rm[h][w] : -INFINITY, ps = w < kVWarps ? sm.rs[h][w] : 0.f;
      float MM = pm;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) MM = fmaxf(MM, __shfl_xor_sync(0xffffffffu, MM, o));
      double t = pm > -INFINITY ? (double)ps * (double)ex2((pm - MM) * cT) : 0.0;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      const double lse = (double)MM / a.tau64 + log(t);
      if (w == 0) {
        sm.lse[h] = lse;
        if (!(MM > -INFINITY) && (h == 0 || hasD)) atomicOr(&sm.flag, h == 0 ? 1 : 2);
      }
      __syncwarp();
      if (lane == 0 && hasD && !(sm.flag & 3)) {  // the accept test, fp64
        const int x = a.draft[(int64_t)b * a.K + k];
        if (x >= 0 && x < V) {
          const double p = exp((double)ld_elem<TIn>(rT, x) / a.tau64 - sm.lse[0]);
          const double q = exp((double)ld_elem<TIn>(rD, x) / a.tau64 - sm.lse[1]);
          const Stream sa(a.seed, a.round, SD_STREAM_ACCEPT);
          const double uu = uniform_f64(sa.at(0, (uint32_t)j).x);
          if (uu * q < p) atomicOr(&sm.flag, 4);
        } else {
          atomicOr(&sm.flag, 8);
        }
      }
    }
    __syncthreads();
    const int flag = sm.flag;
    const bool badTr = (flag & 1) != 0, badDr = hasD && (flag & 2) != 0;
    const bool bad = badTr || badDr;
    const bool accept = (flag & 4) != 0;
    const double lseT = sm.lse[0], lseD = sm.lse[1];
    // the draw this row needs: 1 the residual (a rejection), 2 the bonus (the last row)
    const int mode = bad ? 0 : (hasD ? (accept ? 0 : 1) : 2);

    const float LT = (float)(lseT * 1.4426950408889634), LD = (float)(lseD * 1.4426950408889634);
    const Stream sblk(a.seed, a.round, mode == 1 ? SD_STREAM_RESIDUAL_BLOCK : SD_STREAM_BONUS_BLOCK);
    const uint32_t rid = mode == 1 ? (uint32_t)j : (uint32_t)b;
    verify_pass2<TIn>(sm, rT, rD, V, nt, hasD, mode, badTr, badDr, cT, LT, LD, vec, drop, sblk, rid);
    // ---------------- the row's TV and block
    __syncthreads();
    if (warp == 0) {
      float tv = lane < kVWarps ? sm.tv[lane] : 0.f;
      tv = warp_sum(tv);
      Cand c = lane < kVWarps ? sm.cand[lane] : cand_empty();
      c = warp_cand(c);
      if (lane == 0) {
        if (hasD && a.tv_out) a.tv_out[(int64_t)b * a.K + k] = bad ? NAN : 0.5f * tv;
        // -2: no candidate; -1: settle in fp64; else the block
        sm.block = c.idx == 0x7FFFFFFF ? -2 : (c.ohi < c.lo ? c.idx : -1);
      }
    }
    __syncthreads();
    int code = kCodeBad;
    if (mode != 0) {
      int dmode = mode;  // 1 residual, 2 bonus, 0 target after a zero residual
      bool zr = false;
      int jb = sm.block;
      const Stream sb_res(a.seed, a.round, SD_STREAM_RESIDUAL_BLOCK);
      if (jb < 0) {
        jb = exact_block<TIn>(sm, rT, rD, V, dmode, a.tau64, lseT, lseD, sblk, rid);
        if (jb < 0 && mode == 1) {  // the exact residual is zero everywhere: draw from p
          zr = true;
          dmode = 0;
          jb = exact_block<TIn>(sm, rT, rD, V, 0, a.tau64, lseT, lseD, sb_res, rid);
        }
      }
      if (warp == 0) {
        const Stream se(a.seed, a.round, mode == 1 ? SD_STREAM_RESIDUAL : SD_STREAM_BONUS);
        const int tok = jb >= 0 ? exact_in_block<TIn>(rT, rD, V, jb, dmode, a.tau64, lseT, lseD, se, rid) : -1;
        if (mode == 1) code = encode_reject(max(tok, 0), (flag & 8) != 0, zr);
        else code = tok;
      }
    } else if (hasD && !bad) {
      code = a.draft[(int64_t)b * a.K + k];  // accepted
    }
    if (tid == 0) {
      if (hasD && bad) raise_err(a.dev_err, SD_DEV_NONFINITE);
      a.out_tokens[j] = code;
    }
    __syncthreads();  // shared state is reused by the next row
  }
}

// Per sequence: the first rejection (or the end) decides the accepted length
// and the emitted tokens from the rows' encoded outcomes.
__global__ void verify_finalize_kernel(int B, int K, int32_t* out_tokens, int32_t* acc_len,
                                       uint32_t* dev_err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int R = K + 1;
  int32_t* o = out_tokens + (int64_t)b * R;
  int first = K;
  for (int k = 0; k < K; ++k)
    if (o[k] < 0) {
      first = k;
      break;
    }
  acc_len[b] = first;
  const int code = o[first];
  int tok;
  if (code == kCodeBad || (first == K && code < 0)) {
    tok = -1;
    raise_err(dev_err, SD_DEV_NONFINITE);  // the row the sequence reached is not finite
  } else if (first == K) {
    tok = code;  // the bonus token
  } else {
    const int dec = -2 - code;
    tok = dec & ((1 << 29) - 1);
    if (dec & (1 << 29)) raise_err(dev_err, SD_DEV_TOKEN_OOB);
    if (dec & (1 << 30)) raise_err(dev_err, SD_DEV_ZERO_RESIDUAL);
  }
  o[first] = tok;
  for (int k = first + 1; k < R; ++k) o[k] = -1;
}

template <typename TIn>
static sd_status launch_verify(VerifyArgs& a, int B, cudaStream_t stream) {
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const int64_t rows = (int64_t)B * a.R;
  const int grid = (int)(rows < kVPerSM * nsm ? rows : kVPerSM * nsm);  // persistent CTAs
  const int smem = (int)sizeof(VSmem);
  const void* fn = (const void*)verify_rows_kernel<TIn>;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  verify_rows_kernel<TIn><<<grid, kVThreads, smem, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  verify_finalize_kernel<<<(B + 127) / 128, 128, 0, stream>>>(B, a.K, a.out_tokens, a.acc_len,
                                                               a.dev_err);
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  return SD_OK;
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status sd_verify_reject(const void* zT, const void* zD, sd_dtype dt, int B, int K,
                                      int V, int64_t ld, const int32_t* draft_tokens, float tau,
                                      uint64_t seed, uint64_t round, int32_t* accepted_len,
                                      int32_t* out_tokens, float* tv_out, uint32_t* dev_err,
                                      void* stream) {
  if (B < 0 || K < 1 || V < 1 || ld < V || !tau_ok(tau)) return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (B == 0) return SD_OK;
  if (!zT || !zD || !draft_tokens || !accepted_len || !out_tokens) return SD_ERR_INVALID_ARG;
  if ((int64_t)B * (K + 1) >= (int64_t)1 << 31) return SD_ERR_UNSUPPORTED;
  if (V > 262144) return SD_ERR_UNSUPPORTED;
  VerifyArgs a = {};
  a.zT = zT;
  a.zD = zD;
  a.ld = ld;
  a.B = B;
  a.V = V;
  a.K = K;
  a.R = K + 1;
  const int esize = dt == SD_BF16 ? 2 : 4;
  a.vec = ((uintptr_t)zT % 16 == 0) && ((uintptr_t)zD % 16 == 0) && ((ld * esize) % 16 == 0);
  a.inv_tau = (float)(1.0 / (double)tau);
  a.cT = (float)(1.4426950408889634 / (double)tau);
  a.tau64 = (double)tau;
  a.draft = draft_tokens;
  a.seed = seed;
  a.round = round;
  a.out_tokens = out_tokens;
  a.acc_len = accepted_len;
  a.tv_out = tv_out;
  a.dev_err = dev_err;
  cudaStream_t s = (cudaStream_t)stream;
  return dt == SD_BF16 ? launch_verify<uint16_t>(a, B, s) : launch_verify<float>(a, B, s);
}
