// Logit-row scoring kernel for SMC-SD rounds and standard SD verification.
//
// What it computes (see include/smcsd.h for the full contract):
//   "Faster LLM Inference via Sequential Monte Carlo", section 2 -- per
//   particle the importance log-weight sum_k [log p_T(x) - log q_D(x)] and
//   the bonus token drawn from the target at position K+1;
//   METASD section 2 -- per row the total-variation distance 1/2 |p - q|_1;
//   SMC-SD section 1 / METASD section 1 -- standard verification with the
//   residual max(p - q, 0).
//
// Design (B200, sm_100a):
//   * One unit of work = one particle (SMC-SD) or one sequence (verify):
//     K+1 row pairs processed in order by one thread-block cluster of C CTAs.
//     The vocabulary is split into C slices (split-V); CTA r owns slice r of
//     both the target and the draft row.
//   * Rows stream HBM -> shared memory with bulk async copies
//     (cp.async.bulk, no multicast) into a ring of stages completed on
//     mbarriers; thread 0 refills a stage as soon as the CTA has moved it to
//     registers.  The ring keeps several rows in flight per SM.
//   * Each thread holds 32 entries of each row in registers and computes one
//     exp2 per element (relative to its warp's max).  The per-CTA partial
//     (max, sum) is exchanged through distributed shared memory after one
//     cluster barrier per row; every CTA rebuilds the row's normalisers from
//     the C partials.  TV then comes from the exps still held in registers,
//     so every element is read from HBM once and exponentiated once.
//   * lse, log-probs and log-weights are combined in fp64 from the fp32
//     partials; the accept test of verification is taken in fp64.
//   * Gumbel-max draws (bonus token, residual token) are exact: an fp32 screen
//     over the register-resident exps with rigorous error bounds keeps only
//     the entries that can still win (most are pruned before any Philox call
//     or log), and near-ties are re-scored in fp64 from the logits in HBM.
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>
#include <cuda_runtime.h>

#include "common.cuh"

namespace smcsd {

constexpr int kMaxWarps = 16;
constexpr int kMaxCluster = 16;
constexpr int kMaxThreads = 512;
constexpr int kEPT = 32;  // entries per thread per row

struct ScoreArgs {
  const void* zT;
  const void* zD;
  int64_t ld;
  int V, K, R;
  int64_t units;
  int slice;
  int stages;
  uint32_t stage_bytes;  // bytes reserved for one tensor's slice in a stage
  int use_tma;
  float inv_tau, cT;     // 1/tau and log2(e)/tau, fp32
  double tau64;
  const int32_t* draft;  // [units, K]
  uint64_t seed, round;
  const double* logw_prev;
  double* logw_out;
  float* tv_out;
  int32_t* bonus_out;
  int32_t* tokens_out;
  double* lse_out;
  double* lp_out;
  int32_t* acc_len;
  int32_t* out_tokens;
  uint32_t* dev_err;
};

struct XSlot {  // one CTA's per-row partials
  float mT, sT, mD, sD;
  float zxT, zxD, pad0, pad1;
};

struct Cand {  // screening partial: best point score, its bounds, best bound of the rest
  float s, lo, hi, ohi;
  int idx, pad0, pad1, pad2;
};

struct Cand64 {
  double s;
  int idx, pad;
};

struct Tail {
  uint64_t full[8];
  XSlot xs[2];
  float4 wpart[kMaxWarps];
  float tvp[2][kMaxCluster][kMaxWarps];
  Cand wcand[kMaxWarps];
  Cand xc;
  Cand64 wc64[kMaxWarps];
  Cand64 xc64;
  double lse64[2];
  int flag[4];
};

__device__ __forceinline__ Cand cand_empty() {
  Cand c;
  c.s = -INFINITY;
  c.lo = -INFINITY;
  c.hi = -INFINITY;
  c.ohi = -INFINITY;
  c.idx = 0x7FFFFFFF;
  c.pad0 = c.pad1 = c.pad2 = 0;
  return c;
}
__device__ __forceinline__ Cand cand_merge(const Cand& a, const Cand& b) {
  const bool aw = a.s > b.s || (a.s == b.s && a.idx < b.idx);
  Cand w = aw ? a : b;
  const Cand& l = aw ? b : a;
  w.ohi = fmaxf(w.ohi, fmaxf(l.hi, l.ohi));
  return w;
}
__device__ __forceinline__ Cand cand_shfl(const Cand& c, int o) {
  Cand r;
  r.s = __shfl_xor_sync(0xffffffffu, c.s, o);
  r.lo = __shfl_xor_sync(0xffffffffu, c.lo, o);
  r.hi = __shfl_xor_sync(0xffffffffu, c.hi, o);
  r.ohi = __shfl_xor_sync(0xffffffffu, c.ohi, o);
  r.idx = __shfl_xor_sync(0xffffffffu, c.idx, o);
  r.pad0 = r.pad1 = r.pad2 = 0;
  return r;
}
__device__ __forceinline__ Cand warp_cand(Cand c) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c = cand_merge(c, cand_shfl(c, o));
  return c;
}
__device__ __forceinline__ void c64_merge(double& s, int& i, double os, int oi) {
  if (os > s || (os == s && oi < i)) {
    s = os;
    i = oi;
  }
}
__device__ __forceinline__ void warp_c64(double& s, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double os = __shfl_xor_sync(0xffffffffu, s, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    c64_merge(s, i, os, oi);
  }
}

// ------------------------------------------------------------------ element access
template <typename TIn>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float get(const float* p, int64_t i) { return p[i]; }
  static __device__ __forceinline__ void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};
template <>
struct Elem<uint16_t> {  // bf16 bit patterns
  static __device__ __forceinline__ float get(const uint16_t* p, int64_t i) {
    return __uint_as_float((uint32_t)p[i] << 16);
  }
  static __device__ __forceinline__ void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x << 16);
    o[1] = __uint_as_float(v.x & 0xFFFF0000u);
    o[2] = __uint_as_float(v.y << 16);
    o[3] = __uint_as_float(v.y & 0xFFFF0000u);
    o[4] = __uint_as_float(v.z << 16);
    o[5] = __uint_as_float(v.z & 0xFFFF0000u);
    o[6] = __uint_as_float(v.w << 16);
    o[7] = __uint_as_float(v.w & 0xFFFF0000u);
  }
};

// Moves this thread's entries of one row slice into registers; returns their max.
// Entry e of the slice lives in chunk e / EPC; thread t owns chunks t, t + nthr, ...
template <typename TIn, int CPT>
__device__ __forceinline__ float load_slice(float* x, const TIn* st, const TIn* g, int len,
                                            int tma_len, int tid, int nthr) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  float m = -INFINITY;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int e0 = (tid + c * nthr) * EPC;
    if (e0 + EPC <= tma_len) {
      const uint4 v = *reinterpret_cast<const uint4*>(st + e0);
      Elem<TIn>::unpack(v, &x[c * EPC]);
    } else {
#pragma unroll
      for (int j = 0; j < EPC; ++j) {
        const int e = e0 + j;
        x[c * EPC + j] =
            e < tma_len ? Elem<TIn>::get(st, e) : (e < len ? Elem<TIn>::get(g, e) : -INFINITY);
      }
    }
#pragma unroll
    for (int j = 0; j < EPC; ++j) m = fmaxf(m, x[c * EPC + j]);
  }
  return m;
}

// In place: x <- 2^((x - m) cT); returns the sum.  Entries at -inf become 0.
template <int N>
__device__ __forceinline__ float exp_slice(float* x, float m, float cT) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    x[i] = ex2((x[i] - m) * cT);
    x[i + 1] = ex2((x[i + 1] - m) * cT);
    x[i + 2] = ex2((x[i + 2] - m) * cT);
    x[i + 3] = ex2((x[i + 3] - m) * cT);
    s0 += x[i];
    s1 += x[i + 1];
    s2 += x[i + 2];
    s3 += x[i + 3];
  }
  return (s0 + s1) + (s2 + s3);
}

// Combine (max, sum) partials whose sums are relative to their own max.
__device__ __forceinline__ float part_term(float m, float s, float M, float cT) {
  return m == -INFINITY ? 0.f : s * ex2((m - M) * cT);
}

// ------------------------------------------------------------------ Gumbel screens
// Mode 0: score = a_v + g_v (bonus token; zero-residual fallback).  xt holds
//   2^((x - mw) cT); y_v = xt * rho = e^{a_v - Tref} with Tref a lower bound on
//   the winning score, so u_v <= 1 - y_v proves g_v <= Tref - a_v (since
//   e^-y >= 1 - y) and the entry cannot win: no log is taken.  Groups of four
//   entries whose y are all below e^{-g_max} skip the Philox call too.
// Mode 1: score = log r_v + g_v, r = max(p - q, 0), p = xt*scT, q = xd*scD,
//   with an fp32 error bound eb on r; every entry whose upper bound on r is
//   positive is screened.
// Each kept entry carries [lo, hi] bounds on its exact score.  The partials
// merge to (best point score, its bounds, the largest upper bound of all
// others); when that upper bound stays below the best lower bound the winner
// is exact, otherwise `rescore_exact` settles it in fp64.
struct ScreenCtx {
  int s0, len, tid, nthr;
  uint32_t rowid;
  float mw_a;        // (warp max of the target) / tau
  float rho;         // mode 0
  float scT, scD;    // mode 1
  float mwT, mwD, cT;
  const void* gT;    // this CTA's slice of the target / draft row in HBM
  const void* gD;
  double tau64, lseT, lseD;
};

constexpr float kYSkip = 5.88e-8f;  // < e^{-g_max}: even g_max cannot lift the entry to Tref

__device__ __forceinline__ bool keep_bonus(float y, float u) {
  return y > 0.f && !(u < (1.0f - y * 1.001f) - 2.4e-7f);
}

template <int CPT, int EPC, int MODE>
__device__ __forceinline__ void screen(const float* xt, const float* xd, const ScreenCtx& cx,
                                       const Stream& st, Cand& out) {
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int e0 = (cx.tid + c * cx.nthr) * EPC;
    if (e0 >= cx.len) continue;
#pragma unroll
    for (int gq = 0; gq < EPC / 4; ++gq) {
      const int base = c * EPC + gq * 4;
      const int v0 = cx.s0 + e0 + gq * 4;
      float y[4], r[4], eb[4];
      float ymax = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (MODE == 0) {
          y[j] = xt[base + j] * cx.rho;
          ymax = fmaxf(ymax, y[j]);
        } else {
          const float p = xt[base + j] * cx.scT, q = xd[base + j] * cx.scD;
          r[j] = p - q;
          eb[j] = 7.7e-6f * (p + q);  // > 2^-17 (p + q): fp32 error bound of p - q
          ymax = fmaxf(ymax, r[j] + eb[j]);
        }
      }
      if (MODE == 0 ? (ymax < kYSkip) : !(ymax > 0.f)) continue;
      const U4 w = st.at((uint32_t)(v0 >> 2), cx.rowid);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (e0 + gq * 4 + j >= cx.len) continue;
        const float u = uniform_f32(word_of(w, j));
        Cand cd;
        if (MODE == 0) {
          if (!keep_bonus(y[j], u)) continue;
          const float g32 = gumbel_f32(u);
          const float a32 = cx.mw_a + logf(xt[base + j]);
          cd.s = a32 + g32;
          const float d = 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
          cd.lo = cd.s - d;
          cd.hi = cd.s + d;
        } else {
          if (!(r[j] + eb[j] > 0.f)) continue;
          const float g32 = gumbel_f32(u);
          const float lh = logf(r[j] + eb[j]);
          const float d = 4e-6f + 4.8e-7f * (fabsf(lh) + 2.f * fabsf(g32));
          cd.hi = lh + g32 + d;
          cd.s = r[j] > 0.f ? logf(r[j]) + g32 : -INFINITY;
          cd.lo = r[j] - eb[j] > 0.f ? logf(r[j] - eb[j]) + g32 - d : -INFINITY;
        }
        cd.ohi = -INFINITY;
        cd.idx = v0 + j;
        cd.pad0 = cd.pad1 = cd.pad2 = 0;
        out = cand_merge(out, cd);
      }
    }
  }
}

// Exact fp64 maximum over the entries the screen keeps whose upper bound
// reaches lo_star.  Recomputes the screen's fp32 values from the logits in HBM
// (same operations, same inputs, so the same entries are kept) and scores the
// survivors in fp64 exactly as the definition does.  Runs only on near-ties.
template <typename TIn, int CPT>
__device__ __noinline__ void rescore_exact(const ScreenCtx cx, const Stream st, int mode,
                                           float lo_star, double* s_out, int* i_out) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  const TIn* gT = (const TIn*)cx.gT;
  const TIn* gD = (const TIn*)cx.gD;
  for (int c = 0; c < CPT; ++c) {
    const int e0 = (cx.tid + c * cx.nthr) * EPC;
    if (e0 >= cx.len) continue;
    for (int gq = 0; gq < EPC / 4; ++gq) {
      const int v0 = cx.s0 + e0 + gq * 4;
      const U4 w = st.at((uint32_t)(v0 >> 2), cx.rowid);
      for (int j = 0; j < 4; ++j) {
        const int le = e0 + gq * 4 + j;
        if (le >= cx.len) continue;
        const float zt = Elem<TIn>::get(gT, le);
        const float et = ex2((zt - cx.mwT) * cx.cT);
        const float u = uniform_f32(word_of(w, j));
        float hi;
        if (mode == 0) {
          if (!keep_bonus(et * cx.rho, u)) continue;
          const float g32 = gumbel_f32(u);
          const float a32 = cx.mw_a + logf(et);
          const float d = 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
          hi = a32 + g32 + d;
        } else {
          const float zd = Elem<TIn>::get(gD, le);
          const float p = et * cx.scT, q = ex2((zd - cx.mwD) * cx.cT) * cx.scD;
          const float r = p - q, eb = 7.7e-6f * (p + q);
          if (!(r + eb > 0.f)) continue;
          const float g32 = gumbel_f32(u);
          const float lh = logf(r + eb);
          hi = lh + g32 + 4e-6f + 4.8e-7f * (fabsf(lh) + 2.f * fabsf(g32));
        }
        if (!(hi >= lo_star)) continue;
        const double g64 = gumbel_f64(uniform_f64(word_of(w, j)));
        const double a64 = (double)zt / cx.tau64;
        double sv;
        if (mode == 0) {
          sv = a64 + g64;
        } else {
          const double b64 = (double)Elem<TIn>::get(gD, le) / cx.tau64;
          const double rr = exp(a64 - cx.lseT) - exp(b64 - cx.lseD);
          sv = rr > 0.0 ? log(rr) + g64 : -INFINITY;
        }
        c64_merge(best, bi, sv, v0 + j);
      }
    }
  }
  *s_out = best;
  *i_out = bi;
}

// Screen from the logits in HBM (both modes): the same fp32 values a register
// screen would use (identical operations on identical inputs), recomputed so
// the once-per-sequence draws of verification do not hold the
// register-resident exps of the main loop.
template <typename TIn, int CPT>
__device__ __noinline__ void screen_global(const ScreenCtx cx, const Stream st, int mode,
                                           Cand* out) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  Cand best = cand_empty();
  const TIn* gT = (const TIn*)cx.gT;
  const TIn* gD = (const TIn*)cx.gD;
  for (int c = 0; c < CPT; ++c) {
    const int e0 = (cx.tid + c * cx.nthr) * EPC;
    if (e0 >= cx.len) continue;
    for (int gq = 0; gq < EPC / 4; ++gq) {
      const int v0 = cx.s0 + e0 + gq * 4;
      float r[4], eb[4], et[4];
      float ymax = 0.f;
      for (int j = 0; j < 4; ++j) {
        const int le = e0 + gq * 4 + j;
        r[j] = 0.f;
        eb[j] = 0.f;
        et[j] = 0.f;
        if (le >= cx.len) continue;
        et[j] = ex2((Elem<TIn>::get(gT, le) - cx.mwT) * cx.cT);
        if (mode == 0) {
          ymax = fmaxf(ymax, et[j] * cx.rho);
        } else {
          const float p = et[j] * cx.scT;
          const float q = ex2((Elem<TIn>::get(gD, le) - cx.mwD) * cx.cT) * cx.scD;
          r[j] = p - q;
          eb[j] = 7.7e-6f * (p + q);
          ymax = fmaxf(ymax, r[j] + eb[j]);
        }
      }
      if (mode == 0 ? (ymax < kYSkip) : !(ymax > 0.f)) continue;
      const U4 w = st.at((uint32_t)(v0 >> 2), cx.rowid);
      for (int j = 0; j < 4; ++j) {
        if (e0 + gq * 4 + j >= cx.len) continue;
        const float u = uniform_f32(word_of(w, j));
        Cand cd;
        if (mode == 0) {
          if (!keep_bonus(et[j] * cx.rho, u)) continue;
          const float g32 = gumbel_f32(u);
          const float a32 = cx.mw_a + logf(et[j]);
          cd.s = a32 + g32;
          const float d = 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
          cd.lo = cd.s - d;
          cd.hi = cd.s + d;
        } else {
          if (!(r[j] + eb[j] > 0.f)) continue;
          const float g32 = gumbel_f32(u);
          const float lh = logf(r[j] + eb[j]);
          const float d = 4e-6f + 4.8e-7f * (fabsf(lh) + 2.f * fabsf(g32));
          cd.hi = lh + g32 + d;
          cd.s = r[j] > 0.f ? logf(r[j]) + g32 : -INFINITY;
          cd.lo = r[j] - eb[j] > 0.f ? logf(r[j] - eb[j]) + g32 - d : -INFINITY;
        }
        cd.ohi = -INFINITY;
        cd.idx = v0 + j;
        cd.pad0 = cd.pad1 = cd.pad2 = 0;
        best = cand_merge(best, cd);
      }
    }
  }
  *out = best;
}

// fp64 log-sum-exp of a row from its C per-CTA partials (one per lane).
__device__ __noinline__ double row_lse64(float m, float s, float M, bool has, double tau64) {
  const double t = (has && m > -INFINITY) ? (double)s * exp(((double)m - (double)M) / tau64) : 0.0;
  return (double)M / tau64 + log(warp_sum_d(t));
}

// Accept test of verification in fp64: u * q(x) < p(x).
__device__ __noinline__ int accept_test(double zxT, double zxD, double lseT, double lseD,
                                        double tau64, uint64_t seed, uint64_t round,
                                        uint32_t rowid) {
  const double p = exp(zxT / tau64 - lseT);
  const double q = exp(zxD / tau64 - lseD);
  const Stream st(seed, round, SD_STREAM_ACCEPT);
  const double u = uniform_f64(st.at(0, rowid).x);
  return u * q < p ? 1 : 0;
}

// ------------------------------------------------------------------ the kernel
template <typename TIn, int CPT, bool VERIFY>
__global__ void __launch_bounds__(kMaxThreads, 1) score_kernel(const ScoreArgs a) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  constexpr int EPT = CPT * EPC;
  static_assert(EPT == kEPT, "entries per thread");
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x, nwarps = nthr >> 5;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const uint32_t cid = cluster_id(), G = num_clusters();
  Tail* tl = reinterpret_cast<Tail*>(smem + (size_t)a.stages * 2 * a.stage_bytes);

  const int s0 = (int)rank * a.slice;
  const int len = max(0, min(a.slice, a.V - s0));
  const int tma_len = a.use_tma ? ((len * (int)sizeof(TIn)) & ~15) / (int)sizeof(TIn) : 0;
  const uint32_t tma_bytes = (uint32_t)tma_len * (uint32_t)sizeof(TIn);
  const int64_t my_units = (int64_t)cid < a.units ? (a.units - 1 - cid) / G + 1 : 0;
  const int64_t nrows = my_units * a.R;
  const bool leader = rank == 0;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) mbar_init(&tl->full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  cluster_sync();

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int64_t it) {
    const int s = (int)(it % a.stages);
    const int64_t unit = cid + (it / a.R) * G;
    const int k = (int)(it % a.R);
    const bool hasD = !VERIFY || k < a.K;
    const int64_t rowT = unit * a.R + k;
    const int64_t rowD = VERIFY ? unit * a.K + k : rowT;
    unsigned char* stg = smem + (size_t)s * 2 * a.stage_bytes;
    mbar_arrive_expect_tx(&tl->full[s], tma_bytes * (hasD ? 2u : 1u));
    if (tma_bytes) {
      bulk_load(stg, (const TIn*)a.zT + rowT * a.ld + s0, tma_bytes, &tl->full[s], pol);
      if (hasD)
        bulk_load(stg + a.stage_bytes, (const TIn*)a.zD + rowD * a.ld + s0, tma_bytes, &tl->full[s],
                  pol);
    }
  };
  if (tid == 0)
    for (int64_t it = 0; it < nrows && it < a.stages; ++it) issue(it);

  // Per-unit state.  Decisions are computed identically in every CTA of the
  // cluster, so control flow (and the number of cluster barriers) matches.
  double logw_acc = 0.0;  // leader, warp 0
  bool unit_bad = false;  // leader, warp 0: some lp / lq invalid
  bool done = false;      // verify: sequence finished
  int acc_len = 0;        // verify
  int emitted = -1;       // verify: the drawn token
  int64_t prev_tv_idx = -1;
  bool prev_bad = false;

  float xt[EPT], xd[EPT];

  for (int64_t it = 0; it < nrows; ++it) {
    const int s = (int)(it % a.stages);
    const uint32_t ph = (uint32_t)((it / a.stages) & 1);
    const int par = (int)(it & 1);
    const int64_t unit = cid + (it / a.R) * G;
    const int k = (int)(it % a.R);
    const bool hasD = !VERIFY || k < a.K;
    const int64_t rowT = unit * a.R + k;
    const int64_t rowD = VERIFY ? unit * a.K + k : rowT;
    if (k == 0) {
      logw_acc = 0.0;
      unit_bad = false;
      done = false;
      acc_len = 0;
      emitted = -1;
    }
    const int x = k < a.K ? a.draft[unit * a.K + k] : -1;
    const bool x_ok = k < a.K && x >= 0 && x < a.V;

    if (!mbar_wait(&tl->full[s], ph)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
    const TIn* stT = reinterpret_cast<const TIn*>(smem + (size_t)s * 2 * a.stage_bytes);
    const TIn* stD = reinterpret_cast<const TIn*>(smem + (size_t)s * 2 * a.stage_bytes + a.stage_bytes);
    const TIn* gT = (const TIn*)a.zT + rowT * a.ld + s0;
    const TIn* gD = (const TIn*)a.zD + rowD * a.ld + s0;

    const float mt = load_slice<TIn, CPT>(xt, stT, gT, len, tma_len, tid, nthr);
    float md = -INFINITY;
    if (hasD) md = load_slice<TIn, CPT>(xd, stD, gD, len, tma_len, tid, nthr);
    // the owner of the draft token's entry records its raw logits
    if (x_ok && x >= s0 && x < s0 + len) {
      const int le = x - s0;
      if (((le / EPC) % nthr) == tid) {
        tl->xs[par].zxT = le < tma_len ? Elem<TIn>::get(stT, le) : Elem<TIn>::get(gT, le);
        tl->xs[par].zxD = le < tma_len ? Elem<TIn>::get(stD, le) : Elem<TIn>::get(gD, le);
      }
    }
    const float mwT = warp_max(mt);
    const float mwD = hasD ? warp_max(md) : -INFINITY;
    const float mwTs = mwT == -INFINITY ? 0.f : mwT;
    const float mwDs = mwD == -INFINITY ? 0.f : mwD;
    float sT = exp_slice<EPT>(xt, mwTs, a.cT);
    float sD = 0.f;
    if (hasD) sD = exp_slice<EPT>(xd, mwDs, a.cT);
    sT = warp_sum(sT);
    if (hasD) sD = warp_sum(sD);
    if (lane == 0) tl->wpart[warp] = make_float4(mwT, sT, mwD, sD);
    __syncthreads();  // (A) the stage is now free; warp partials are visible
    if (tid == 0 && it + a.stages < nrows) issue(it + a.stages);
    if (warp == 0) {
      const float4 wp = lane < nwarps ? tl->wpart[lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      const float M1 = warp_max(wp.x), M2 = warp_max(wp.z);
      const float S1 = warp_sum(part_term(wp.x, wp.y, M1, a.cT));
      const float S2 = warp_sum(part_term(wp.z, wp.w, M2, a.cT));
      if (lane == 0) {
        tl->xs[par].mT = M1;
        tl->xs[par].sT = S1;
        tl->xs[par].mD = M2;
        tl->xs[par].sD = S2;
      }
    }
    cluster_sync();  // (B) all CTAs' partials of this row are visible

    // Rebuild the row's normalisers from the C partials (every warp, same order).
    float pm1 = -INFINITY, ps1 = 0.f, pm2 = -INFINITY, ps2 = 0.f;
    if (lane < (int)C) {
      const uint32_t pa = peer_addr(&tl->xs[par], lane);
      pm1 = ld_peer_f32(pa + 0);
      ps1 = ld_peer_f32(pa + 4);
      pm2 = ld_peer_f32(pa + 8);
      ps2 = ld_peer_f32(pa + 12);
    }
    const float MT = warp_max(pm1);
    const float ST = warp_sum(part_term(pm1, ps1, MT, a.cT));
    const float MD = hasD ? warp_max(pm2) : 0.f;
    const float SD = hasD ? warp_sum(part_term(pm2, ps2, MD, a.cT)) : 1.f;
    const bool badT = !(MT > -INFINITY && MT < INFINITY && ST > 0.f && ST < INFINITY);
    const bool badD = hasD && !(MD > -INFINITY && MD < INFINITY && SD > 0.f && SD < INFINITY);
    const bool bad = badT || badD;

    // fp64 lse of both rows (warp 0 of every CTA; lanes < C hold the partials)
    double lse64T = 0.0, lse64D = 0.0, zxT = 0.0, zxD = 0.0;
    if (warp == 0) {
      lse64T = row_lse64(pm1, ps1, MT, lane < (int)C, a.tau64);
      if (hasD) lse64D = row_lse64(pm2, ps2, MD, lane < (int)C, a.tau64);
      if (x_ok) {
        const uint32_t oa = peer_addr(&tl->xs[par], (uint32_t)(x / a.slice));
        zxT = (double)ld_peer_f32(oa + 16);
        zxD = (double)ld_peer_f32(oa + 20);
      }
    }

    // Leader bookkeeping: TV of the previous row, lse / lp / log-weight of this one.
    if (leader && warp == 0) {
      if (prev_tv_idx >= 0) {
        float acc = 0.f;
        if (lane < nwarps)
          for (int c = 0; c < (int)C; ++c) acc += tl->tvp[par ^ 1][c][lane];
        acc = warp_sum(acc);
        if (lane == 0) a.tv_out[prev_tv_idx] = prev_bad ? NAN : 0.5f * acc;
      }
      if (lane == 0) {
        if (bad && (!VERIFY || k < a.K || !done)) raise_err(a.dev_err, SD_DEV_NONFINITE);
        if (!VERIFY) {
          if (a.lse_out) {
            a.lse_out[rowT * 2 + 0] = badT ? NAN : lse64T;
            a.lse_out[rowT * 2 + 1] = badD ? NAN : lse64D;
          }
          if (k < a.K) {
            double lp = NAN, lq = NAN;
            if (!x_ok) raise_err(a.dev_err, SD_DEV_TOKEN_OOB);
            if (x_ok && !bad) {
              lp = zxT / a.tau64 - lse64T;
              lq = zxD / a.tau64 - lse64D;
            } else {
              unit_bad = true;
            }
            logw_acc += lp - lq;
            if (a.lp_out) {
              a.lp_out[(unit * a.K + k) * 2 + 0] = lp;
              a.lp_out[(unit * a.K + k) * 2 + 1] = lq;
            }
          }
        }
      }
    }
    const bool want_tv = hasD && a.tv_out != nullptr;
    if (leader && warp == 0) {
      prev_tv_idx = want_tv ? (VERIFY ? rowD : rowT) : -1;
      prev_bad = bad;
    }

    // Per-warp scales turning register exps into normalised probabilities.
    const float scT = (mwT > -INFINITY && !badT) ? ex2((mwT - MT) * a.cT) / ST : 0.f;
    const float scD = (hasD && mwD > -INFINITY && !badD) ? ex2((mwD - MD) * a.cT) / SD : 0.f;

    if (want_tv) {
      float tv = 0.f;
#pragma unroll
      for (int i = 0; i < EPT; ++i) tv += fabsf(__fmul_rn(xt[i], scT) - __fmul_rn(xd[i], scD));
      tv = warp_sum(tv);
      if (lane == 0) st_peer_f32(peer_addr(&tl->tvp[par][rank][warp], 0), tv);
    }

    // ---------------- verification: accept test (CTA-uniform, fp64) ----------------
    bool draw_residual = false;
    if (VERIFY && k < a.K && !done) {
      if (warp == 0 && lane == 0) {
        int acc = 0;
        if (!bad && x_ok)
          acc = accept_test(zxT, zxD, lse64T, lse64D, a.tau64, a.seed, a.round, (uint32_t)rowT);
        tl->flag[0] = acc;
        tl->lse64[0] = lse64T;
        tl->lse64[1] = lse64D;
        if (leader && !x_ok) raise_err(a.dev_err, SD_DEV_TOKEN_OOB);
      }
      __syncthreads();
      const bool accept = tl->flag[0] != 0;
      if (bad) {
        done = true;
        acc_len = k;
        emitted = -1;
      } else if (accept) {
        acc_len = k + 1;
      } else {
        draw_residual = true;
      }
    }

    // ---------------- Gumbel-max draws: bonus token / residual token ----------------
    const bool draw_bonus = (k == a.K) && !badT && (!VERIFY || !done);
    if (draw_bonus || draw_residual) {
      ScreenCtx cx;
      cx.s0 = s0;
      cx.len = len;
      cx.tid = tid;
      cx.nthr = nthr;
      cx.gT = gT;
      cx.gD = gD;
      cx.tau64 = a.tau64;
      cx.mw_a = mwTs * a.inv_tau;
      // Tref = M/tau + g_min - margin <= exact score of the row's max entry.
      const float margin = 1e-5f + 2e-7f * fabsf(MT * a.inv_tau);
      cx.rho = (mwT > -INFINITY) ? ex2((mwT - MT) * a.cT + (-kGumbelMinF + margin) * kLog2e) : 0.f;
      cx.scT = scT;
      cx.scD = scD;
      cx.mwT = mwTs;
      cx.mwD = mwDs;
      cx.cT = a.cT;
      if (draw_residual) {
        cx.lseT = tl->lse64[0];
        cx.lseD = tl->lse64[1];
      }
      const uint32_t tag = draw_bonus ? SD_STREAM_BONUS : SD_STREAM_RESIDUAL;
      cx.rowid = draw_bonus ? (uint32_t)unit : (uint32_t)rowT;
      const Stream st(a.seed, a.round, tag);
      int mode = draw_bonus ? 0 : 1;
      for (int pass = 0; pass < 2; ++pass) {
        // pass 0: residual (mode 1) or bonus (mode 0); pass 1 only for an
        // all-zero residual: draw from p with the same stream.
        Cand cd = cand_empty();
        if (!VERIFY)
          screen<CPT, EPC, 0>(xt, xd, cx, st, cd);
        else
          screen_global<TIn, CPT>(cx, st, mode, &cd);
        cd = warp_cand(cd);
        if (lane == 0) tl->wcand[warp] = cd;
        __syncthreads();
        if (warp == 0) {
          Cand c2 = lane < nwarps ? tl->wcand[lane] : cand_empty();
          c2 = warp_cand(c2);
          if (lane == 0) tl->xc = c2;
        }
        cluster_sync();  // (C1)
        if (warp == 0) {
          Cand c3 = cand_empty();
          if (lane < (int)C) {
            const uint32_t pa = peer_addr(&tl->xc, lane);
            c3.s = ld_peer_f32(pa + 0);
            c3.lo = ld_peer_f32(pa + 4);
            c3.hi = ld_peer_f32(pa + 8);
            c3.ohi = ld_peer_f32(pa + 12);
            c3.idx = ld_peer_s32(pa + 16);
          }
          c3 = warp_cand(c3);
          if (lane == 0) {
            const bool none = c3.idx == 0x7FFFFFFF;
            tl->flag[1] = none ? 2 : (c3.ohi < c3.lo ? 0 : 1);  // 0 clear, 1 near-tie, 2 nothing
            tl->flag[2] = c3.idx;
            reinterpret_cast<float*>(&tl->flag[3])[0] = c3.lo;
          }
        }
        __syncthreads();
        const int decision = tl->flag[1];
        int winner = tl->flag[2];
        if (decision == 2 && mode == 1) {  // all-zero residual: sample p instead
          if (leader && tid == 0) raise_err(a.dev_err, SD_DEV_ZERO_RESIDUAL);
          mode = 0;
          continue;
        }
        if (decision == 1) {  // near-tie: exact fp64 re-score of every entry that can still win
          const float lo_star = reinterpret_cast<const float*>(&tl->flag[3])[0];
          double s64 = -INFINITY;
          int i64 = 0x7FFFFFFF;
          rescore_exact<TIn, CPT>(cx, st, mode, lo_star, &s64, &i64);
          warp_c64(s64, i64);
          if (lane == 0) {
            tl->wc64[warp].s = s64;
            tl->wc64[warp].idx = i64;
          }
          __syncthreads();
          if (warp == 0) {
            double ss = lane < nwarps ? tl->wc64[lane].s : -INFINITY;
            int ii = lane < nwarps ? tl->wc64[lane].idx : 0x7FFFFFFF;
            warp_c64(ss, ii);
            if (lane == 0) {
              tl->xc64.s = ss;
              tl->xc64.idx = ii;
            }
          }
          cluster_sync();  // (C2)
          if (warp == 0) {
            double ss = -INFINITY;
            int ii = 0x7FFFFFFF;
            if (lane < (int)C) {
              const uint32_t pa = peer_addr(&tl->xc64, lane);
              ss = ld_peer_f64(pa);
              ii = ld_peer_s32(pa + 8);
            }
            warp_c64(ss, ii);
            if (lane == 0) tl->flag[2] = ii;
          }
          __syncthreads();
          winner = tl->flag[2];
          if (winner == 0x7FFFFFFF && mode == 1) {  // exact residual is zero everywhere
            if (leader && tid == 0) raise_err(a.dev_err, SD_DEV_ZERO_RESIDUAL);
            mode = 0;
            continue;
          }
        }
        if (winner == 0x7FFFFFFF) winner = -1;
        if (VERIFY) {
          emitted = winner;
          done = true;
          if (draw_bonus) acc_len = a.K;
        } else if (leader && tid == 0) {
          a.bonus_out[unit] = winner;
          if (a.tokens_out) a.tokens_out[unit * a.R + a.K] = winner;
        }
        break;
      }
    }

    // ---------------- end of unit: write per-particle / per-sequence outputs ----------------
    if (k == a.K && leader && tid == 0) {
      if (!VERIFY) {
        if (badT) {
          a.bonus_out[unit] = -1;
          if (a.tokens_out) a.tokens_out[unit * a.R + a.K] = -1;
        }
        const double prev = a.logw_prev ? a.logw_prev[unit] : 0.0;
        a.logw_out[unit] = unit_bad ? NAN : prev + logw_acc;
        if (a.tokens_out)
          for (int j = 0; j < a.K; ++j) a.tokens_out[unit * a.R + j] = a.draft[unit * a.K + j];
      } else {
        a.acc_len[unit] = acc_len;
        for (int j = 0; j < a.R; ++j) {
          int tok = -1;
          if (j < acc_len) tok = a.draft[unit * a.K + j];
          else if (j == acc_len) tok = emitted;
          a.out_tokens[unit * a.R + j] = tok;
        }
      }
    }
  }

  cluster_sync();  // (F) last row's TV partials are in; no peer reads our smem after this
  if (leader && warp == 0 && prev_tv_idx >= 0) {
    const int par = (int)((nrows - 1) & 1);
    float acc = 0.f;
    if (lane < nwarps)
      for (int c = 0; c < (int)C; ++c) acc += tl->tvp[par][c][lane];
    acc = warp_sum(acc);
    if (lane == 0) a.tv_out[prev_tv_idx] = prev_bad ? NAN : 0.5f * acc;
  }
}

// ------------------------------------------------------------------ host side
struct LaunchPlan {
  int C, threads, stages, slice;
  uint32_t stage_bytes;
  size_t smem;
  int clusters_max;
};

template <typename TIn, bool VERIFY>
void* kernel_ptr() {
  return (void*)score_kernel<TIn, (int)(kEPT * sizeof(TIn) / 16), VERIFY>;
}

static int max_active_clusters(const void* fn, int C, int threads, size_t smem) {
  cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C * 64);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Chooses the cluster size C that keeps the most SMs busy for this many units:
// each CTA must hold its slice in 32 registers per thread (<= 512 threads) and
// at least two ring stages must fit in shared memory.  Plans are cached per
// (kernel, device, V, element size, unit count clipped at 4096).
static bool make_plan(const void* fn, int V, int esize, int64_t units, LaunchPlan& best) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, int, int64_t>, LaunchPlan> cache;
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t ukey = std::min<int64_t>(units, 4096);
  const auto key = std::make_tuple(fn, dev, V, esize, ukey);
  auto hit = cache.find(key);
  if (hit != cache.end()) {
    best = hit->second;
    return true;
  }
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t tail = sizeof(Tail) + 128;
  bool found = false;
  int64_t best_score = -1;
  for (int C = 1; C <= kMaxCluster; ++C) {
    const int slice = (int)(((int64_t)(V + C - 1) / C + 7) / 8 * 8);
    const int threads = std::max(32, (int)(((slice + kEPT - 1) / kEPT + 31) / 32 * 32));
    if (threads > kMaxThreads) continue;
    const uint32_t sb = (uint32_t)(((int64_t)slice * esize + 127) / 128 * 128);
    int stages = 0;
    for (int s = 4; s >= 2; --s)
      if ((size_t)s * 2 * sb + tail <= (size_t)optin) {
        stages = s;
        break;
      }
    if (stages == 0) continue;
    const size_t smem = (size_t)stages * 2 * sb + tail;
    const int nc = max_active_clusters(fn, C, threads, smem);
    if (nc <= 0) continue;
    const int64_t score = std::min<int64_t>(ukey, nc) * C;
    if (score > best_score) {
      best_score = score;
      best = LaunchPlan{C, threads, stages, slice, sb, smem, nc};
      found = true;
    }
  }
  if (found) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)best.smem);
    cache[key] = best;
  }
  return found;
}

template <typename TIn, bool VERIFY>
static sd_status launch_score(ScoreArgs& a, cudaStream_t stream) {
  const void* fn = kernel_ptr<TIn, VERIFY>();
  LaunchPlan p;
  if (!make_plan(fn, a.V, (int)sizeof(TIn), a.units, p)) return SD_ERR_UNSUPPORTED;
  a.slice = p.slice;
  a.stages = p.stages;
  a.stage_bytes = p.stage_bytes;
  const bool aligned = ((uintptr_t)a.zT % 16 == 0) && ((uintptr_t)a.zD % 16 == 0) &&
                       ((a.ld * (int64_t)sizeof(TIn)) % 16 == 0);
  a.use_tma = aligned ? 1 : 0;
  const int64_t nclusters = std::min<int64_t>(a.units, p.clusters_max);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nclusters * p.C));
  cfg.blockDim = dim3(p.threads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = p.C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, score_kernel<TIn, (int)(kEPT * sizeof(TIn) / 16), VERIFY>, a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  return SD_OK;
}

static bool tau_ok(float tau) { return tau > 0.f && tau < INFINITY; }

static void fill_common(ScoreArgs& a, float tau) {
  a.inv_tau = (float)(1.0 / (double)tau);
  a.cT = (float)(1.4426950408889634 / (double)tau);
  a.tau64 = (double)tau;
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status smcsd_score(const void* zT, const void* zD, sd_dtype dt, int B, int N, int K,
                                 int V, int64_t ld, const int32_t* draft_tokens, float tau,
                                 uint64_t seed, uint64_t round, const double* logw_prev,
                                 double* logw_out, int32_t* bonus_out, float* tv_out,
                                 int32_t* tokens_out, double* lse_out, double* lp_out,
                                 uint32_t* dev_err, void* stream) {
  if (B < 0 || N < 1 || K < 0 || V < 1 || ld < V || !tau_ok(tau)) return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (B == 0) return SD_OK;
  if (!zT || !zD || !logw_out || !bonus_out || (K > 0 && !draft_tokens)) return SD_ERR_INVALID_ARG;
  if ((int64_t)B * N * (K + 1) >= (int64_t)1 << 31) return SD_ERR_UNSUPPORTED;
  if (V > 262144) return SD_ERR_UNSUPPORTED;
  ScoreArgs a = {};
  a.zT = zT;
  a.zD = zD;
  a.ld = ld;
  a.V = V;
  a.K = K;
  a.R = K + 1;
  a.units = (int64_t)B * N;
  fill_common(a, tau);
  a.draft = draft_tokens;
  a.seed = seed;
  a.round = round;
  a.logw_prev = logw_prev;
  a.logw_out = logw_out;
  a.tv_out = tv_out;
  a.bonus_out = bonus_out;
  a.tokens_out = tokens_out;
  a.lse_out = lse_out;
  a.lp_out = lp_out;
  a.dev_err = dev_err;
  cudaStream_t s = (cudaStream_t)stream;
  return dt == SD_BF16 ? launch_score<uint16_t, false>(a, s) : launch_score<float, false>(a, s);
}

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
  ScoreArgs a = {};
  a.zT = zT;
  a.zD = zD;
  a.ld = ld;
  a.V = V;
  a.K = K;
  a.R = K + 1;
  a.units = B;
  fill_common(a, tau);
  a.draft = draft_tokens;
  a.seed = seed;
  a.round = round;
  a.tv_out = tv_out;
  a.acc_len = accepted_len;
  a.out_tokens = out_tokens;
  a.dev_err = dev_err;
  cudaStream_t s = (cudaStream_t)stream;
  return dt == SD_BF16 ? launch_score<uint16_t, true>(a, s) : launch_score<float, true>(a, s);
}
