// Standard speculative-decoding verification (N = 1), row-parallel.
//
// What it computes (include/smcsd.h, sd_verify_reject): per sequence, K
// drafted tokens are checked in order against the target; the first rejection
// discards the rest and draws one token from the residual max(p - q, 0); if all
// K are accepted a bonus token is drawn from the target row K+1.  Sources:
// "Faster LLM Inference via Sequential Monte Carlo", section 1 (standard SD,
// rejection, KV rollback); METASD section 1 (background) and section 2 (TV
// block divergence reported per position).
//
// Design (B200, sm_100a).  Every (sequence, position) row is independent until
// the first rejection is known, so each is scored on its own, all at once:
//   verify_rows_kernel: one CTA of 1024 threads per row (a thread-block cluster
//     of C CTAs when V exceeds one CTA's slice, the CTAs exchanging partials
//     through distributed shared memory); each thread holds 32 bf16 (16 fp32)
//     entries of the target and draft rows in registers, loaded with 16-byte
//     vector loads.  Per row: the log-sum-exp of both rows (fp64 combine), the
//     accept test u q(x) < p(x) in fp64, TV = 1/2 sum |p - q| (exps recomputed
//     from the registers), and -- only if the row rejects its draft token --
//     the residual draw argmax_{r_v > 0} (log r_v + g_v), r = max(p - q, 0);
//     the last row draws the bonus token argmax (z/tau + g).  The draws are
//     exact: an fp32 screen with rigorous error bounds keeps only entries that
//     can still win, near-ties are re-scored in fp64 over the whole row.  Each
//     row's outcome is encoded in its own slot of out_tokens.
//   verify_finalize_kernel: per sequence, the first rejection decides the
//     accepted length and the emitted tokens; slots past it become -1.
// Work for rows past the first rejection is spent speculatively; nothing but
// the outputs is written to global memory.
#include <algorithm>
#include <cuda_runtime.h>

#include "rows.cuh"

namespace smcsd {

constexpr int kVThreads = 1024;
constexpr int kVWarps = kVThreads / 32;
constexpr int kVChunks = 4;  // 16-byte chunks of each row per thread

struct VerifyArgs {
  const void* zT;
  const void* zD;
  int64_t ld;
  int V, K, R;
  int slice;   // entries of a row per CTA
  int vec;     // 16-byte loads allowed
  float inv_tau, cT;
  double tau64;
  const int32_t* draft;
  uint64_t seed, round;
  int32_t* out_tokens;
  int32_t* acc_len;
  float* tv_out;
  uint32_t* dev_err;
};

// What a CTA publishes to the other CTAs of its row's cluster.
struct alignas(16) VExch {
  float mT, sT, mD, sD;  // (max, sum of exps relative to it) over the CTA's slice
  float zxT, zxD;        // raw logits of the draft token (its owner CTA only)
  int own, pad0;
  float tvp, pad1, pad2, pad3;  // TV partial
  Cand cand;             // best candidate of the CTA's screen
};

struct VSmem {
  float red[4][kVWarps];
  Cand wc[kVWarps];
  Cand64 w64[kVWarps];
  VExch ex;
  double lse[2];
  int flag;
};

// Encoding of a row's outcome in its out_tokens slot, decoded by the finalize
// kernel: an accepted draft keeps its id (>= 0); a row whose rows are not
// finite is -1; a rejection is -2 - (token | oob << 29 | zero_residual << 30).
constexpr int kCodeBad = -1;
__device__ __forceinline__ int encode_reject(int tok, bool oob, bool zr) {
  return -2 - (tok | (oob ? (1 << 29) : 0) | (zr ? (1 << 30) : 0));
}

template <typename TIn>
struct VT;
template <>
struct VT<uint16_t> {
  static constexpr int EPC = 8;  // entries per 16-byte chunk
  static __device__ __forceinline__ float get(const uint4& v, int j) {
    const uint32_t w = (j >> 1) == 0 ? v.x : ((j >> 1) == 1 ? v.y : ((j >> 1) == 2 ? v.z : v.w));
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
  static __device__ __forceinline__ uint4 load(const uint16_t* g, int e0, int len, bool vec) {
    if (vec && e0 + 8 <= len) return *reinterpret_cast<const uint4*>(g + e0);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = e0 + 2 * j < len ? (uint32_t)g[e0 + 2 * j] : 0xFF80u;
      const uint32_t hi = e0 + 2 * j + 1 < len ? (uint32_t)g[e0 + 2 * j + 1] : 0xFF80u;
      w[j] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct VT<float> {
  static constexpr int EPC = 4;
  static __device__ __forceinline__ float get(const uint4& v, int j) {
    return __uint_as_float(j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w)));
  }
  static __device__ __forceinline__ uint4 load(const float* g, int e0, int len, bool vec) {
    if (vec && e0 + 4 <= len) return *reinterpret_cast<const uint4*>(g + e0);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = e0 + j < len ? __float_as_uint(g[e0 + j]) : 0xFF800000u;
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// CTA-wide reductions of four values (max, NaN-propagating) / (sum) through shared memory.
__device__ __forceinline__ float4 cta_max4_nan(float4 v, VSmem* sm) {
  float a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(a[i]));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0)
    for (int i = 0; i < 4; ++i) sm->red[i][warp] = a[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i] = sm->red[i][lane];
    asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(a[i]));
  }
  return make_float4(a[0], a[1], a[2], a[3]);
}
__device__ __forceinline__ float4 cta_sum4(float4 v, VSmem* sm) {
  float a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = warp_sum(a[i]);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0)
    for (int i = 0; i < 4; ++i) sm->red[i][warp] = a[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = warp_sum(sm->red[i][lane]);
  return make_float4(a[0], a[1], a[2], a[3]);
}
__device__ __forceinline__ Cand cta_cand(Cand c, VSmem* sm) {
  c = warp_cand(c);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sm->wc[warp] = c;
  __syncthreads();
  return warp_cand(sm->wc[lane]);
}

// Exact fp64 draw over a whole row, by the whole CTA (a near-tie the fp32
// screens could not settle, or a zero residual; rare).  mode 0: argmax z/tau +
// g; mode 1: argmax over max(p - q, 0) > 0 of log(p - q) + g.  Entries whose
// fp32 upper bound stays below lo_star cannot win and are not re-scored.
template <typename TIn>
__device__ __noinline__ int exact_draw_row(const TIn* rT, const TIn* rD, int V, int mode,
                                           double lseT, double lseD, const VerifyArgs& a,
                                           float lo_star, const Stream st, uint32_t rowid,
                                           VSmem* sm) {
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int q = threadIdx.x; q * 4 < V; q += blockDim.x) {
    const U4 w = st.at((uint32_t)q, rowid);
    for (int j = 0; j < 4; ++j) {
      const int v = q * 4 + j;
      if (v >= V) break;
      const float zt = Elem<TIn>::get(rT, v);
      const float u = uniform_f32(word_of(w, j));
      float hi;
      if (mode == 0) {
        const float a32 = zt * a.inv_tau;
        if (!(a32 + kGumbelMaxF + 1e-3f >= lo_star)) continue;
        const float g32 = gumbel_f32(u);
        hi = a32 + g32 + score_err(a32, g32);
      } else {
        const float p = (float)exp((double)zt / a.tau64 - lseT);
        const float q = (float)exp((double)Elem<TIn>::get(rD, v) / a.tau64 - lseD);
        const float r = p - q, eb = 7.7e-6f * (p + q) + 1e-37f;
        if (!(r + eb > 0.f)) continue;
        const float lh = logf(r + eb);
        if (!(lh + kGumbelMaxF + 1e-3f >= lo_star)) continue;
        const float g32 = gumbel_f32(u);
        hi = lh + g32 + score_err(lh, g32);
      }
      if (!(hi >= lo_star)) continue;
      const double g64 = gumbel_f64(uniform_f64(word_of(w, j)));
      double sv;
      if (mode == 0) {
        sv = (double)zt / a.tau64 + g64;
      } else {
        const double rr = exp((double)zt / a.tau64 - lseT) - exp((double)Elem<TIn>::get(rD, v) / a.tau64 - lseD);
        sv = rr > 0.0 ? log(rr) + g64 : -INFINITY;
      }
      c64_merge(best, bi, sv, v);
    }
  }
  warp_c64(best, bi);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) {
    sm->w64[warp].s = best;
    sm->w64[warp].idx = bi;
  }
  __syncthreads();
  double s = lane < (int)(blockDim.x >> 5) ? sm->w64[lane].s : -INFINITY;
  int i = lane < (int)(blockDim.x >> 5) ? sm->w64[lane].idx : 0x7FFFFFFF;
  warp_c64(s, i);
  return i == 0x7FFFFFFF ? -1 : i;
}

template <typename TIn>
__global__ void __launch_bounds__(kVThreads, 1) verify_rows_kernel(const VerifyArgs a) {
  using T8 = VT<TIn>;
  constexpr int EPC = T8::EPC;
  __shared__ VSmem sm;
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const int j = (int)cluster_id();  // row unit: sequence b, position k
  const int b = j / a.R, k = j % a.R;
  const bool hasD = k < a.K;
  const int s0 = (int)rank * a.slice;
  const int len = max(0, min(a.slice, a.V - s0));
  const TIn* rT = (const TIn*)a.zT + ((int64_t)b * a.R + k) * a.ld;
  const TIn* rD = hasD ? (const TIn*)a.zD + ((int64_t)b * a.K + k) * a.ld : rT;
  const TIn* gT = rT + s0;
  const TIn* gD = rD + s0;
  const bool vec = a.vec != 0;
  const float cT = a.cT;

  // ---------------- the row slices into registers
  uint4 xT[kVChunks], xD[kVChunks];
#pragma unroll
  for (int c = 0; c < kVChunks; ++c) {
    const int e0 = (tid + c * kVThreads) * EPC;
    xT[c] = T8::load(gT, e0, len, vec);
    xD[c] = hasD ? T8::load(gD, e0, len, vec) : xT[c];
  }
  const int x = hasD ? a.draft[(int64_t)b * a.K + k] : -1;
  const bool x_ok = hasD && x >= 0 && x < a.V;

  // ---------------- CTA maxima, then sums of exps relative to them
  float mt = -INFINITY, md = -INFINITY;
#pragma unroll
  for (int c = 0; c < kVChunks; ++c)
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      mt = fmax_nan(mt, T8::get(xT[c], e));
      md = fmax_nan(md, T8::get(xD[c], e));
    }
  const float4 mx = cta_max4_nan(make_float4(mt, md, 0.f, 0.f), &sm);
  const float MtC = mx.x == -INFINITY ? 0.f : mx.x, MdC = mx.y == -INFINITY ? 0.f : mx.y;
  const float nT = -MtC * cT, nD = -MdC * cT;
  float st = 0.f, sd = 0.f;
#pragma unroll
  for (int c = 0; c < kVChunks; ++c)
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      st += ex2(fmaf(T8::get(xT[c], e), cT, nT));
      sd += ex2(fmaf(T8::get(xD[c], e), cT, nD));
    }
  const float4 sums = cta_sum4(make_float4(st, sd, 0.f, 0.f), &sm);
  if (tid == 0) {
    sm.ex.mT = mx.x;
    sm.ex.sT = sums.x;
    sm.ex.mD = mx.y;
    sm.ex.sD = sums.y;
    sm.ex.own = x_ok && x >= s0 && x < s0 + len;
    if (sm.ex.own) {
      sm.ex.zxT = Elem<TIn>::get(rT, x);
      sm.ex.zxD = Elem<TIn>::get(rD, x);
    }
  }
  // ---------------- the row's normalisers from every CTA of the cluster
  cluster_sync();
  float MT, ST, MD, SD, zxT = 0.f, zxD = 0.f;
  double lseT, lseD;
  {
    const int lane = tid & 31;
    const bool has = lane < (int)C;
    float pm1 = -INFINITY, ps1 = 0.f, pm2 = -INFINITY, ps2 = 0.f;
    int own = 0;
    float zt = 0.f, zd = 0.f;
    if (has) {
      const uint32_t base = peer_addr(&sm.ex, (uint32_t)lane);
      pm1 = ld_peer_f32(base + offsetof(VExch, mT));
      ps1 = ld_peer_f32(base + offsetof(VExch, sT));
      pm2 = ld_peer_f32(base + offsetof(VExch, mD));
      ps2 = ld_peer_f32(base + offsetof(VExch, sD));
      own = ld_peer_s32(base + offsetof(VExch, own));
      if (own) {
        zt = ld_peer_f32(base + offsetof(VExch, zxT));
        zd = ld_peer_f32(base + offsetof(VExch, zxD));
      }
    }
    float m1 = pm1, m2 = pm2;
    warp_max2_nan(m1, m2);
    MT = m1;
    MD = m2;
    float t1 = part_term(pm1, ps1, MT, cT), t2 = part_term(pm2, ps2, MD, cT);
    warp_sum2(t1, t2);
    ST = t1;
    SD = t2;
    const unsigned ob = __ballot_sync(0xffffffffu, own != 0);
    if (ob) {
      zxT = __shfl_sync(0xffffffffu, zt, __ffs(ob) - 1);
      zxD = __shfl_sync(0xffffffffu, zd, __ffs(ob) - 1);
    }
    // fp64 log-sum-exp: the slice factors in fp32, their sums and the log in fp64
    double d1 = (has && pm1 > -INFINITY) ? (double)ps1 * (double)ex2((pm1 - MT) * cT) : 0.0;
    double d2 = (has && pm2 > -INFINITY) ? (double)ps2 * (double)ex2((pm2 - MD) * cT) : 0.0;
    d1 = warp_sum_d(d1);
    d2 = warp_sum_d(d2);
    lseT = (double)MT / a.tau64 + log(d1);
    lseD = (double)MD / a.tau64 + log(d2);
  }
  const bool badT = !(MT > -INFINITY && MT < INFINITY && ST > 0.f && ST < INFINITY);
  const bool badD = hasD && !(MD > -INFINITY && MD < INFINITY && SD > 0.f && SD < INFINITY);
  const bool bad = badT || badD;

  // ---------------- the accept test (every CTA of the row takes it alike)
  bool accept = false;
  if (hasD && !bad && x_ok) {
    const double p = exp((double)zxT / a.tau64 - lseT);
    const double q = exp((double)zxD / a.tau64 - lseD);
    const Stream sa(a.seed, a.round, SD_STREAM_ACCEPT);
    const double u = uniform_f64(sa.at(0, (uint32_t)j).x);
    accept = u * q < p;
  }

  // ---------------- TV, and the draw this row needs
  // per-thread scale factors turning the CTA-relative exps into probabilities
  const float scT = (!badT && mx.x > -INFINITY) ? ex2((MtC - MT) * cT) / ST : 0.f;
  const float scD = (hasD && !badD && mx.y > -INFINITY) ? ex2((MdC - MD) * cT) / SD : 0.f;
  const bool draw_resid = hasD && !bad && !accept;
  const bool draw_bonus = !hasD && !badT;
  const Stream sr(a.seed, a.round, draw_resid ? SD_STREAM_RESIDUAL : SD_STREAM_BONUS);
  const uint32_t rowid = draw_resid ? (uint32_t)j : (uint32_t)b;
  float tvp = 0.f;
  Cand best = cand_empty();
  if (hasD && !draw_resid) {
#pragma unroll
    for (int c = 0; c < kVChunks; ++c)
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        const float p = ex2(fmaf(T8::get(xT[c], e), cT, nT)) * scT;
        const float q = ex2(fmaf(T8::get(xD[c], e), cT, nD)) * scD;
        tvp += fabsf(p - q);
      }
  } else if (draw_resid) {
    // TV and the residual screen in one pass.  Tr, a lower bound on the
    // winner's score, is the best fp32 lower bound among the entries this thread
    // has scored so far (any entry's score bounds the winner's from below; -inf
    // at first).  With y = (r + eb) e^{-Tr}, u <= 1 - y proves log r + g <= Tr
    // (e^{-y} >= 1 - y): the entry cannot win and takes no log; four entries
    // whose y all stay below e^{-g_max} skip the Philox call.
    float Tr = -INFINITY, eTr = INFINITY;
#pragma unroll 1
    for (int c = 0; c < kVChunks; ++c) {
#pragma unroll 1
      for (int h = 0; h < EPC / 4; ++h) {
        float r4[4], eb4[4], ymax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float zt = T8::get(xT[c], 4 * h + e), zd = T8::get(xD[c], 4 * h + e);
          const float p = ex2(fmaf(zt, cT, nT)) * scT, q = ex2(fmaf(zd, cT, nD)) * scD;
          tvp += fabsf(p - q);
          r4[e] = p - q;
          eb4[e] = 7.7e-6f * (p + q) + 1e-37f;
          ymax = fmaxf(ymax, (r4[e] + eb4[e]) * eTr);
        }
        const int v0 = s0 + (tid + c * kVThreads) * EPC + 4 * h;
        if (!(ymax >= kYSkip) || v0 >= s0 + len) continue;
        const U4 w = sr.at((uint32_t)(v0 >> 2), rowid);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float ub = r4[e] + eb4[e];
          if (!(ub > 0.f) || v0 + e >= s0 + len) continue;
          const float u = uniform_f32(word_of(w, e));
          if (Tr > -INFINITY && !keep_bonus(ub * eTr, u)) continue;
          const float g32 = gumbel_f32(u);
          const float hl = logf(ub);
          const float d = score_err(hl, g32);
          Cand cd;
          cd.hi = hl + g32 + d;
          if (!(cd.hi >= Tr)) continue;
          cd.s = r4[e] > 0.f ? logf(r4[e]) + g32 : -INFINITY;
          cd.lo = r4[e] - eb4[e] > 0.f ? logf(r4[e] - eb4[e]) + g32 - d : -INFINITY;
          cd.ohi = -INFINITY;
          cd.idx = v0 + e;
          cd.aux = -1;
          cd.pad1 = cd.pad2 = 0;
          best = cand_merge(best, cd);
          if (cd.lo > Tr) {
            Tr = cd.lo;
            eTr = ex2(-Tr * kLog2e) * 1.001f;  // (rounded up: keeps the tests conservative)
          }
        }
      }
    }
  } else if (draw_bonus) {
    // T = M/tau + g_min - margin bounds the winning score from below; an entry
    // whose uniform proves u <= 1 - e^{a - T} cannot win (integer leading-bit
    // test first), four entries that even g_max cannot lift to T skip Philox.
    const float aM = MT * a.inv_tau;
    const float Tc = (aM + kGumbelMinF - (1e-5f + 2e-7f * fabsf(aM))) * kLog2e;
#pragma unroll 1
    for (int c = 0; c < kVChunks; ++c) {
#pragma unroll 1
      for (int h = 0; h < EPC / 4; ++h) {
        float z4[4], X4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          z4[e] = T8::get(xT[c], 4 * h + e);
          X4[e] = fmaf(z4[e], cT, -Tc);
        }
        if (!(fmaxf(fmaxf(X4[0], X4[1]), fmaxf(X4[2], X4[3])) > -24.05f)) continue;
        const int v0 = s0 + (tid + c * kVThreads) * EPC + 4 * h;
        const U4 w = sr.at((uint32_t)(v0 >> 2), rowid);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t wj = word_of(w, e);
          const uint32_t Rr = 0x7FFFFFu - (wj >> 9);
          const int hb = Rr ? 31 - __clz((int)Rr) : -1;
          if (!(X4[e] > (float)(hb - 23) - 0.01f) || v0 + e >= s0 + len) continue;
          const float u = uniform_f32(wj);
          if (keep_bonus(ex2(X4[e]), u)) best = cand_merge(best, bonus_cand_a(z4[e] * a.inv_tau, u, v0 + e));
        }
      }
    }
  }
  // ---------------- the row's TV and candidates, gathered at the leader CTA
  const float4 tvs = cta_sum4(make_float4(tvp, 0.f, 0.f, 0.f), &sm);
  best = cta_cand(best, &sm);
  if (tid == 0) {
    sm.ex.tvp = tvs.x;
    sm.ex.cand = best;
  }
  cluster_sync();
  if (rank == 0 && tid < 32) {
    const int lane = tid;
    const bool has = lane < (int)C;
    float tv = 0.f;
    Cand cd = cand_empty();
    if (has) {
      const uint32_t base = peer_addr(&sm.ex, (uint32_t)lane);
      tv = ld_peer_f32(base + offsetof(VExch, tvp));
      cd.s = ld_peer_f32(base + offsetof(VExch, cand) + offsetof(Cand, s));
      cd.lo = ld_peer_f32(base + offsetof(VExch, cand) + offsetof(Cand, lo));
      cd.hi = ld_peer_f32(base + offsetof(VExch, cand) + offsetof(Cand, hi));
      cd.ohi = ld_peer_f32(base + offsetof(VExch, cand) + offsetof(Cand, ohi));
      cd.idx = ld_peer_s32(base + offsetof(VExch, cand) + offsetof(Cand, idx));
    }
    tv = warp_sum(tv);
    cd = warp_cand(cd);
    if (lane == 0) {
      if (hasD && a.tv_out) a.tv_out[(int64_t)b * a.K + k] = bad ? NAN : 0.5f * tv;
      sm.wc[0] = cd;
    }
  }
  cluster_sync();  // every CTA's exchange slot has been read: peers may finish
  if (rank != 0) return;

  // ---------------- the leader encodes the row's outcome
  int code;
  if (hasD) {
    if (bad) {
      code = kCodeBad;
      if (tid == 0) raise_err(a.dev_err, SD_DEV_NONFINITE);
    } else if (accept) {
      code = x;
    } else {
      const Cand cd = sm.wc[0];
      int tok;
      bool zr = false;
      if (cd.idx == 0x7FFFFFFF) {  // no residual mass in fp32: decide exactly
        tok = exact_draw_row<TIn>(rT, rD, a.V, 1, lseT, lseD, a, -INFINITY, sr, rowid, &sm);
        if (tok < 0) {  // the exact residual is zero everywhere: draw from p
          zr = true;
          tok = exact_draw_row<TIn>(rT, rD, a.V, 0, lseT, lseD, a, -INFINITY, sr, rowid, &sm);
        }
      } else if (cd.ohi < cd.lo) {
        tok = cd.idx;
      } else {  // near-tie: exact fp64 re-score of every entry that can still win
        tok = exact_draw_row<TIn>(rT, rD, a.V, 1, lseT, lseD, a, cd.lo, sr, rowid, &sm);
      }
      code = encode_reject(max(tok, 0), !x_ok, zr);
    }
  } else {
    if (badT) {
      code = kCodeBad;
    } else {
      const Cand cd = sm.wc[0];
      if (cd.idx == 0x7FFFFFFF) code = -1;
      else if (cd.ohi < cd.lo) code = cd.idx;
      else code = exact_draw_row<TIn>(rT, rT, a.V, 0, lseT, lseD, a, cd.lo, sr, rowid, &sm);
    }
  }
  if (tid == 0) a.out_tokens[(int64_t)b * a.R + k] = code;
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
  a.slice = kVThreads * kVChunks * VT<TIn>::EPC;
  const int C = (a.V + a.slice - 1) / a.slice;
  if (C > kMaxCluster) return SD_ERR_UNSUPPORTED;
  a.slice = ((a.V + C - 1) / C + 7) / 8 * 8;  // balanced slices (multiples of 8 entries)
  const void* fn = (const void*)verify_rows_kernel<TIn>;
  if (C > 8 && cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  LaunchPlan p{C, 1, kVThreads, 0, a.slice, 0, 0, 0};
  const sd_status st = launch_clusters(fn, p, (int64_t)B * a.R, a, stream);
  if (st != SD_OK) return st;
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
