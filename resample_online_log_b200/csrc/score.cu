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
#include <cstdlib>
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
  int slice;             // entries per group slice (a multiple of 8)
  int groups;            // independent warp groups per CTA (1..3)
  int stages;            // ring stages
  uint32_t stage_bytes;  // bytes reserved for one tensor's slice in a stage
  int use_tma;
  float inv_tau, cT;     // 1/tau and log2(e)/tau, fp32
  double tau64, inv_tau64;
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

struct Cand {  // screening partial: best point score, its bounds, best bound of the rest
  float s, lo, hi, ohi;
  int idx, pad0, pad1, pad2;
};

struct Cand64 {
  double s;
  int idx, pad;
};

constexpr int kMaxGroups = 3;
constexpr int kMaxSlices = 32;  // cluster size x groups

// One group's message for one row, pushed into every CTA of the cluster.
struct alignas(16) Msg {
  float mT, sT, mD, sD;  // (max, sum of exps relative to it) over its slice of each row
  float zxT, zxD;        // raw logits of the draft token (owner slice only)
  float tvprev;          // this group's TV partial of its previous row
  int aux;               // argmax entry of its target slice (rows that draw a token)
};

constexpr int kLogN = 4;
// Row record handed from the leader's group 0 to its bookkeeping warp.
struct alignas(16) LogEntry {
  Msg m[kMaxSlices];
  int64_t unit;
  int k, x;
};

struct alignas(16) GroupState {  // scratch of one warp group
  float4 wpart[kMaxWarps];
  float tvw[kMaxWarps];
  float wargv[kMaxWarps];
  int wargi[kMaxWarps];
  Cand wcand[kMaxWarps];
  Cand64 wc64[kMaxWarps];
  float zx[2][2];
  double lse64[2];
  int flag[4];
};

struct alignas(128) Tail {
  uint64_t full[4];           // ring stages (bulk copies)
  uint64_t rbar[2];           // row messages, by row parity
  uint64_t cbar[2], dbar[2];  // candidate / fp64 messages, by use parity
  uint64_t fbar, pad_bar;
  uint64_t logfull[kLogN], logempty[kLogN];
  int stage_cnt[4];           // groups done with each stage
  int pad_cnt[4];
  Msg recv[2][kMaxSlices];
  Cand crecv[2][kMaxSlices];
  Cand64 drecv[2][kMaxSlices];
  float frecv[kMaxSlices];
  GroupState gs[kMaxGroups];
  LogEntry log[kLogN];
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
// Work split: a cluster of C CTAs scores one row pair at a time; each CTA runs
// `groups` independent warp groups, and group g of CTA q owns vocabulary slice
// j = q*groups + g (J = C*groups slices per row).  The groups of a CTA share the
// bulk-copy ring but otherwise run unsynchronised, so one group's exp2 phase
// overlaps another group's exchange, TV and bookkeeping of the same or the
// previous row (ping-pong), which keeps MUFU and the issue slots busy.
//
// Message exchange: after its group-level reduction a group pushes one 32-byte
// Msg into slot [j] of every CTA of the cluster with st.async, which completes
// transaction bytes on the receiver's mbarrier; group 0 of each CTA arms the
// CTA's barrier for J messages per row and every group waits on it.  No
// cluster-wide barrier or fence sits on the per-row path.  Slots and barriers
// alternate by row parity: a group can only send row r+2 after every group has
// sent row r+1, which each does only after reading its row r slots.

__device__ __forceinline__ void send_row_msg(Tail* tl, int par, int j, uint32_t C, int lane,
                                             const Msg& m) {
  if (lane < (int)C) {  // lane l -> slot j of CTA l
    const uint32_t ra = peer_addr(&tl->recv[par][j], (uint32_t)lane);
    const uint32_t rb = peer_addr(&tl->rbar[par], (uint32_t)lane);
    st_async_v4(ra, m.mT, m.sT, m.mD, m.sD, rb);
    st_async_v4(ra + 16, m.zxT, m.zxD, m.tvprev, __int_as_float(m.aux), rb);
  }
}

// Candidate scoring of one kept entry (rare; kept out of line to keep the hot
// loop small).
__device__ __noinline__ Cand bonus_cand(float e, float u, float mw_a, int v) {
  const float g32 = gumbel_f32(u);
  const float a32 = mw_a + logf(e);
  Cand cd;
  cd.s = a32 + g32;
  const float d = 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
  cd.lo = cd.s - d;
  cd.hi = cd.s + d;
  cd.ohi = -INFINITY;
  cd.idx = v;
  cd.pad0 = cd.pad1 = cd.pad2 = 0;
  return cd;
}

// Register screen for the bonus token (SMC-SD): entries of this thread, exps
// xt relative to its warp max; see the Gumbel-screen notes above.
template <int CPT, int EPC>
__device__ __forceinline__ void screen_bonus(const float* xt, const ScreenCtx& cx,
                                             const Stream& st, Cand& out) {
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int e0 = (cx.tid + c * cx.nthr) * EPC;
    if (e0 >= cx.len) continue;
#pragma unroll
    for (int gq = 0; gq < EPC / 4; ++gq) {
      const int base = c * EPC + gq * 4;
      const int v0 = cx.s0 + e0 + gq * 4;
      const float y0 = xt[base] * cx.rho, y1 = xt[base + 1] * cx.rho;
      const float y2 = xt[base + 2] * cx.rho, y3 = xt[base + 3] * cx.rho;
      if (fmaxf(fmaxf(y0, y1), fmaxf(y2, y3)) < kYSkip) continue;
      const U4 w = st.at((uint32_t)(v0 >> 2), cx.rowid);
      const float u0 = uniform_f32(w.x), u1 = uniform_f32(w.y);
      const float u2 = uniform_f32(w.z), u3 = uniform_f32(w.w);
      const bool k0 = keep_bonus(y0, u0) && e0 + gq * 4 + 0 < cx.len;
      const bool k1 = keep_bonus(y1, u1) && e0 + gq * 4 + 1 < cx.len;
      const bool k2 = keep_bonus(y2, u2) && e0 + gq * 4 + 2 < cx.len;
      const bool k3 = keep_bonus(y3, u3) && e0 + gq * 4 + 3 < cx.len;
      if (k0 | k1 | k2 | k3) {
        if (k0) out = cand_merge(out, bonus_cand(xt[base], u0, cx.mw_a, v0));
        if (k1) out = cand_merge(out, bonus_cand(xt[base + 1], u1, cx.mw_a, v0 + 1));
        if (k2) out = cand_merge(out, bonus_cand(xt[base + 2], u2, cx.mw_a, v0 + 2));
        if (k3) out = cand_merge(out, bonus_cand(xt[base + 3], u3, cx.mw_a, v0 + 3));
      }
    }
  }
}

// Bookkeeping warp of the leader CTA: fp64 lse, log-probs, log-weights, TV and
// per-particle outputs, fed row by row through a small shared-memory ring so
// that none of this sits on the compute warps' critical path.
template <bool VERIFY>
__device__ void bookkeep(const ScoreArgs& a, Tail* tl, uint32_t J, int64_t nrows, bool want_tv) {
  const int lane = threadIdx.x & 31;
  double logw_acc = 0.0;
  bool unit_bad = false;
  int64_t prev_tv_idx = -1;
  bool prev_bad = false;
  const int64_t entries = nrows + ((want_tv && nrows > 0) ? 1 : 0);
  for (int64_t it = 0; it < entries; ++it) {
    const int slot = (int)(it % kLogN);
    if (!mbar_wait(&tl->logfull[slot], (uint32_t)((it / kLogN) & 1)))
      raise_err(a.dev_err, SD_DEV_TIMEOUT);
    const LogEntry& e = tl->log[slot];
    if (prev_tv_idx >= 0) {  // every message carries its group's TV partial of the previous row
      float v = lane < (int)J ? e.m[lane].tvprev : 0.f;
      v = warp_sum(v);
      if (lane == 0) a.tv_out[prev_tv_idx] = prev_bad ? NAN : 0.5f * v;
    }
    if (it == nrows) {  // final record: only the last row's TV
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->logempty[slot]);
      break;
    }
    const int64_t unit = e.unit;
    const int k = e.k, x = e.x;
    const bool hasD = !VERIFY || k < a.K;
    const float pm1 = lane < (int)J ? e.m[lane].mT : -INFINITY;
    const float ps1 = lane < (int)J ? e.m[lane].sT : 0.f;
    const float pm2 = lane < (int)J ? e.m[lane].mD : -INFINITY;
    const float ps2 = lane < (int)J ? e.m[lane].sD : 0.f;
    const float MT = warp_max(pm1);
    const float ST = warp_sum(part_term(pm1, ps1, MT, a.cT));
    const float MD = hasD ? warp_max(pm2) : 0.f;
    const float SD = hasD ? warp_sum(part_term(pm2, ps2, MD, a.cT)) : 1.f;
    const bool badT = !(MT > -INFINITY && MT < INFINITY && ST > 0.f && ST < INFINITY);
    const bool badD = hasD && !(MD > -INFINITY && MD < INFINITY && SD > 0.f && SD < INFINITY);
    const bool bad = badT || badD;
    const int64_t rowT = unit * a.R + k;
    const int64_t rowD = VERIFY ? unit * a.K + k : rowT;
    if (!VERIFY) {
      if (k == 0) {
        logw_acc = 0.0;
        unit_bad = false;
      }
      const double lse64T = row_lse64(pm1, ps1, MT, lane < (int)J, a.tau64);
      const double lse64D = row_lse64(pm2, ps2, MD, lane < (int)J, a.tau64);
      if (lane == 0) {
        if (bad) raise_err(a.dev_err, SD_DEV_NONFINITE);
        if (a.lse_out) {
          a.lse_out[rowT * 2 + 0] = badT ? NAN : lse64T;
          a.lse_out[rowT * 2 + 1] = badD ? NAN : lse64D;
        }
        if (k < a.K) {
          const bool x_ok = x >= 0 && x < a.V;
          double lp = NAN, lq = NAN;
          if (!x_ok) raise_err(a.dev_err, SD_DEV_TOKEN_OOB);
          if (x_ok && !bad) {
            const Msg& o = e.m[x / a.slice];
            lp = (double)o.zxT / a.tau64 - lse64T;
            lq = (double)o.zxD / a.tau64 - lse64D;
          } else {
            unit_bad = true;
          }
          logw_acc += lp - lq;
          if (a.lp_out) {
            a.lp_out[(unit * a.K + k) * 2 + 0] = lp;
            a.lp_out[(unit * a.K + k) * 2 + 1] = lq;
          }
        } else {
          const double prev = a.logw_prev ? a.logw_prev[unit] : 0.0;
          a.logw_out[unit] = unit_bad ? NAN : prev + logw_acc;
          if (a.tokens_out)
            for (int jj = 0; jj < a.K; ++jj)
              a.tokens_out[unit * a.R + jj] = a.draft[unit * a.K + jj];
        }
      }
    }
    prev_tv_idx = (want_tv && hasD) ? (VERIFY ? rowD : rowT) : -1;
    prev_bad = bad;
    __syncwarp();
    if (lane == 0) mbar_arrive(&tl->logempty[slot]);
  }
}

template <typename TIn, int CPT, bool VERIFY>
__global__ void __launch_bounds__(kMaxThreads, 1) score_kernel(const ScoreArgs a) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  constexpr int EPT = CPT * EPC;
  static_assert(EPT == kEPT, "entries per thread");
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ncomp = blockDim.x - 32;          // last warp: service (bookkeeping)
  const uint32_t NG = (uint32_t)a.groups;
  const int gthr = ncomp / (int)NG;           // threads per group
  const int grp = tid / gthr;                 // this thread's group (== NG for the service warp)
  const int gtid = tid - grp * gthr, gwarp = gtid >> 5, gnw = gthr >> 5;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const uint32_t cid = cluster_id(), G = num_clusters();
  const uint32_t J = C * NG;
  Tail* tl = reinterpret_cast<Tail*>(smem + (size_t)a.stages * 2 * a.stage_bytes);

  // This CTA's vocabulary range (copied by bulk copies) and this group's slice.
  const int cs0 = (int)rank * (int)NG * a.slice;
  const int clen = max(0, min((int)NG * a.slice, a.V - cs0));
  const int ctma = a.use_tma ? ((clen * (int)sizeof(TIn)) & ~15) / (int)sizeof(TIn) : 0;
  const uint32_t tma_bytes = (uint32_t)ctma * (uint32_t)sizeof(TIn);
  const int jslice = (int)rank * (int)NG + grp;
  const int s0 = jslice * a.slice;
  const int len = max(0, min(a.slice, a.V - s0));
  const int tma_len = max(0, min(len, ctma - grp * a.slice));  // entries of the slice in smem
  const int64_t my_units = (int64_t)cid < a.units ? (a.units - 1 - cid) / G + 1 : 0;
  const int64_t nrows = my_units * a.R;
  const bool leader = rank == 0;
  const bool want_tv = a.tv_out != nullptr;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&tl->full[s], 1);
      tl->stage_cnt[s] = 0;
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(&tl->rbar[p], 1);
      mbar_init(&tl->cbar[p], 1);
      mbar_init(&tl->dbar[p], 1);
    }
    mbar_init(&tl->fbar, 1);
    for (int i = 0; i < kLogN; ++i) {
      mbar_init(&tl->logfull[i], 1);
      mbar_init(&tl->logempty[i], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  cluster_sync();  // every CTA's barriers exist before anyone sends to them

  if (warp == ncomp / 32) {
    if (leader) bookkeep<VERIFY>(a, tl, J, nrows, want_tv);
    cluster_sync();
    return;
  }

  GroupState* gs = &tl->gs[grp];
  const int barid = 1 + grp;
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
      bulk_load(stg, (const TIn*)a.zT + rowT * a.ld + cs0, tma_bytes, &tl->full[s], pol);
      if (hasD)
        bulk_load(stg + a.stage_bytes, (const TIn*)a.zD + rowD * a.ld + cs0, tma_bytes,
                  &tl->full[s], pol);
    }
  };
  if (tid == 0)
    for (int64_t it = 0; it < nrows && it < a.stages; ++it) issue(it);

  bool done = false;  // verify: sequence finished (identical in every group)
  int acc_len = 0;
  int emitted = -1;
  int uses = 0;   // candidate exchanges so far
  int duses = 0;  // fp64 exchanges so far
  int x_pref = (nrows > 0 && a.K > 0) ? a.draft[(int64_t)cid * a.K] : -1;

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
    const bool draws = (k == a.K) || VERIFY;  // rows that may draw a token need the argmax
    if (k == 0) {
      done = false;
      acc_len = 0;
      emitted = -1;
    }
    const int x = k < a.K ? x_pref : -1;
    const bool x_ok = k < a.K && x >= 0 && x < a.V;
    if (it + 1 < nrows) {  // prefetch the next row's draft token
      const int64_t un = cid + ((it + 1) / a.R) * G;
      const int kn = (int)((it + 1) % a.R);
      x_pref = kn < a.K ? a.draft[un * a.K + kn] : -1;
    }

    if (!mbar_wait(&tl->full[s], ph)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
    const TIn* stT =
        reinterpret_cast<const TIn*>(smem + (size_t)s * 2 * a.stage_bytes) + grp * a.slice;
    const TIn* stD = reinterpret_cast<const TIn*>(smem + (size_t)s * 2 * a.stage_bytes +
                                                  a.stage_bytes) + grp * a.slice;
    const TIn* gT = (const TIn*)a.zT + rowT * a.ld + s0;
    const TIn* gD = (const TIn*)a.zD + rowD * a.ld + s0;

    const float mt = load_slice<TIn, CPT>(xt, stT, gT, len, tma_len, gtid, gthr);
    float md = -INFINITY;
    if (hasD) md = load_slice<TIn, CPT>(xd, stD, gD, len, tma_len, gtid, gthr);
    const bool owner = x_ok && x >= s0 && x < s0 + len;
    if (owner) {
      const int le = x - s0;
      if (((le / EPC) % gthr) == gtid) {
        gs->zx[par][0] = le < tma_len ? Elem<TIn>::get(stT, le) : Elem<TIn>::get(gT, le);
        gs->zx[par][1] = le < tma_len ? Elem<TIn>::get(stD, le) : Elem<TIn>::get(gD, le);
      }
    }
    bar_sync_n(barid, gthr);  // (A0) this group is done with the stage
    if (gtid == 0) {
      // the last group to finish with the stage refills it
      __threadfence_block();
      if (atomicAdd(&tl->stage_cnt[s], 1) == (int)NG - 1) {
        tl->stage_cnt[s] = 0;
        if (it + a.stages < nrows) issue(it + a.stages);
      }
    }
    int amax = 0x7FFFFFFF;  // this thread's first entry equal to its max (global index)
    if (draws) {
#pragma unroll
      for (int i = EPT - 1; i >= 0; --i)
        if (xt[i] == mt) amax = s0 + (gtid + (i / EPC) * gthr) * EPC + (i % EPC);
    }
    const float mwT = warp_max(mt);
    const float mwD = hasD ? warp_max(md) : -INFINITY;
    if (draws) {  // warp argmax: lowest index among lanes holding the warp max
      int ai = (mt == mwT) ? amax : 0x7FFFFFFF;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ai = min(ai, __shfl_xor_sync(0xffffffffu, ai, o));
      amax = ai;
    }
    const float mwTs = mwT == -INFINITY ? 0.f : mwT;
    const float mwDs = mwD == -INFINITY ? 0.f : mwD;
    float sT = exp_slice<EPT>(xt, mwTs, a.cT);
    float sD = 0.f;
    if (hasD) sD = exp_slice<EPT>(xd, mwDs, a.cT);
    sT = warp_sum(sT);
    if (hasD) sD = warp_sum(sD);
    if (lane == 0) {
      gs->wpart[gwarp] = make_float4(mwT, sT, mwD, sD);
      gs->wargv[gwarp] = mwT;
      gs->wargi[gwarp] = amax;
    }
    bar_sync_n(barid, gthr);  // (A) warp partials are visible
    if (gwarp == 0) {
      const float4 wp =
          lane < gnw ? gs->wpart[lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      Msg m;
      m.mT = warp_max(wp.x);
      m.mD = warp_max(wp.z);
      m.sT = warp_sum(part_term(wp.x, wp.y, m.mT, a.cT));
      m.sD = warp_sum(part_term(wp.z, wp.w, m.mD, a.cT));
      const float tvp = (lane < gnw && it > 0) ? gs->tvw[lane] : 0.f;
      m.tvprev = warp_sum(tvp);
      int ai = 0x7FFFFFFF;
      if (draws) {
        if (lane < gnw && gs->wargv[lane] == m.mT) ai = gs->wargi[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ai = min(ai, __shfl_xor_sync(0xffffffffu, ai, o));
      }
      m.aux = ai;
      m.zxT = owner ? gs->zx[par][0] : 0.f;
      m.zxD = owner ? gs->zx[par][1] : 0.f;
      if (grp == 0 && lane == 0) mbar_arrive_expect_tx(&tl->rbar[par], J * (uint32_t)sizeof(Msg));
      send_row_msg(tl, par, jslice, C, lane, m);
    }
    if (!mbar_wait(&tl->rbar[par], (uint32_t)((it >> 1) & 1))) raise_err(a.dev_err, SD_DEV_TIMEOUT);

    // Rebuild the row's normalisers from the J messages (every warp, same order).
    const Msg* rv = tl->recv[par];
    const float pm1 = lane < (int)J ? rv[lane].mT : -INFINITY;
    const float ps1 = lane < (int)J ? rv[lane].sT : 0.f;
    const float pm2 = lane < (int)J ? rv[lane].mD : -INFINITY;
    const float ps2 = lane < (int)J ? rv[lane].sD : 0.f;
    const float MT = warp_max(pm1);
    const float ST = warp_sum(part_term(pm1, ps1, MT, a.cT));
    const float MD = hasD ? warp_max(pm2) : 0.f;
    const float SD = hasD ? warp_sum(part_term(pm2, ps2, MD, a.cT)) : 1.f;
    const bool badT = !(MT > -INFINITY && MT < INFINITY && ST > 0.f && ST < INFINITY);
    const bool badD = hasD && !(MD > -INFINITY && MD < INFINITY && SD > 0.f && SD < INFINITY);
    const bool bad = badT || badD;

    if (leader && grp == 0 && gwarp == 0) {  // hand the row to the bookkeeping warp
      const int slot = (int)(it % kLogN);
      if (it >= kLogN && !mbar_wait(&tl->logempty[slot], (uint32_t)(((it / kLogN) - 1) & 1)))
        raise_err(a.dev_err, SD_DEV_TIMEOUT);
      if (lane < (int)J) tl->log[slot].m[lane] = rv[lane];
      if (lane == 0) {
        tl->log[slot].unit = unit;
        tl->log[slot].k = k;
        tl->log[slot].x = x;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->logfull[slot]);
    }

    // Per-warp scales turning register exps into normalised probabilities.
    const float scT = (mwT > -INFINITY && !badT) ? ex2((mwT - MT) * a.cT) / ST : 0.f;
    const float scD = (hasD && mwD > -INFINITY && !badD) ? ex2((mwD - MD) * a.cT) / SD : 0.f;

    if (want_tv && hasD) {
      float tv = 0.f;
#pragma unroll
      for (int i = 0; i < EPT; ++i) tv += fabsf(__fmul_rn(xt[i], scT) - __fmul_rn(xd[i], scD));
      tv = warp_sum(tv);
      if (lane == 0) gs->tvw[gwarp] = tv;
    }

    // ---------------- verification: accept test (identical in every group, fp64) ----------------
    bool draw_residual = false;
    if (VERIFY && k < a.K && !done) {
      if (gwarp == 0) {
        const double lse64T = row_lse64(pm1, ps1, MT, lane < (int)J, a.tau64);
        const double lse64D = row_lse64(pm2, ps2, MD, lane < (int)J, a.tau64);
        if (lane == 0) {
          int acc = 0;
          if (!bad && x_ok) {
            const Msg& o = rv[x / a.slice];
            acc = accept_test((double)o.zxT, (double)o.zxD, lse64T, lse64D, a.tau64, a.seed,
                              a.round, (uint32_t)rowT);
          }
          gs->flag[0] = acc;
          gs->lse64[0] = lse64T;
          gs->lse64[1] = lse64D;
          if (leader && grp == 0 && !x_ok) raise_err(a.dev_err, SD_DEV_TOKEN_OOB);
          if (leader && grp == 0 && bad) raise_err(a.dev_err, SD_DEV_NONFINITE);
        }
      }
      bar_sync_n(barid, gthr);
      const bool accept = gs->flag[0] != 0;
      if (bad) {
        done = true;
        acc_len = k;
        emitted = -1;
      } else if (accept) {
        acc_len = k + 1;
      } else {
        draw_residual = true;
      }
    } else if (VERIFY && bad && leader && tid == 0 && (k < a.K || !done)) {
      raise_err(a.dev_err, SD_DEV_NONFINITE);
    }

    // ---------------- Gumbel-max draws: bonus token / residual token ----------------
    const bool draw_bonus = (k == a.K) && !badT && (!VERIFY || !done);
    if (draw_bonus || draw_residual) {
      // Reference entry: the row's argmax v* (first slice holding the row max).
      int vstar;
      {
        int cand = (lane < (int)J && pm1 == MT) ? rv[lane].aux : 0x7FFFFFFF;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, o));
        vstar = cand;
      }
      ScreenCtx cx;
      cx.s0 = s0;
      cx.len = len;
      cx.tid = gtid;
      cx.nthr = gthr;
      cx.gT = gT;
      cx.gD = gD;
      cx.tau64 = a.tau64;
      cx.mw_a = mwTs * a.inv_tau;
      cx.scT = scT;
      cx.scD = scD;
      cx.mwT = mwTs;
      cx.mwD = mwDs;
      cx.cT = a.cT;
      if (draw_residual) {
        cx.lseT = gs->lse64[0];
        cx.lseD = gs->lse64[1];
      }
      const uint32_t tag = draw_bonus ? SD_STREAM_BONUS : SD_STREAM_RESIDUAL;
      cx.rowid = draw_bonus ? (uint32_t)unit : (uint32_t)rowT;
      const Stream st(a.seed, a.round, tag);
      // Tref = fp32 score of v* minus its error bound: a lower bound on the winner.
      {
        const U4 w = st.at((uint32_t)(vstar >> 2), cx.rowid);
        const float g = gumbel_f32(uniform_f32(word_of(w, vstar & 3)));
        const float av = MT * a.inv_tau;
        const float margin = 4e-6f + 1e-6f * (fabsf(av) + 2.f * fabsf(g));
        cx.rho = (mwT > -INFINITY) ? ex2((mwT - MT) * a.cT + (margin - g) * kLog2e) : 0.f;
      }
      int mode = draw_bonus ? 0 : 1;
      for (int pass = 0; pass < 2; ++pass) {
        const int up = uses & 1;
        const uint32_t uph = (uint32_t)((uses >> 1) & 1);
        ++uses;
        Cand cd = cand_empty();
        if (!VERIFY)
          screen_bonus<CPT, EPC>(xt, cx, st, cd);
        else
          screen_global<TIn, CPT>(cx, st, mode, &cd);
        cd = warp_cand(cd);
        if (lane == 0) gs->wcand[gwarp] = cd;
        bar_sync_n(barid, gthr);
        if (gwarp == 0) {
          Cand c2 = lane < gnw ? gs->wcand[lane] : cand_empty();
          c2 = warp_cand(c2);
          if (grp == 0 && lane == 0) mbar_arrive_expect_tx(&tl->cbar[up], J * (uint32_t)sizeof(Cand));
          if (lane < (int)C) {
            const uint32_t ra = peer_addr(&tl->crecv[up][jslice], (uint32_t)lane);
            const uint32_t rb = peer_addr(&tl->cbar[up], (uint32_t)lane);
            st_async_v4(ra, c2.s, c2.lo, c2.hi, c2.ohi, rb);
            st_async_v4(ra + 16, __int_as_float(c2.idx), 0.f, 0.f, 0.f, rb);
          }
        }
        if (!mbar_wait(&tl->cbar[up], uph)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
        Cand c3 = lane < (int)J ? tl->crecv[up][lane] : cand_empty();
        c3 = warp_cand(c3);
        const int decision = c3.idx == 0x7FFFFFFF ? 2 : (c3.ohi < c3.lo ? 0 : 1);
        int winner = c3.idx;
        if (decision == 2 && mode == 1) {  // all-zero residual: draw from p instead
          if (leader && tid == 0) raise_err(a.dev_err, SD_DEV_ZERO_RESIDUAL);
          mode = 0;
          continue;
        }
        if (decision == 1) {  // near-tie: exact fp64 re-score of every entry that can still win
          const int dp = duses & 1;
          const uint32_t dph = (uint32_t)((duses >> 1) & 1);
          ++duses;
          double s64 = -INFINITY;
          int i64 = 0x7FFFFFFF;
          rescore_exact<TIn, CPT>(cx, st, mode, c3.lo, &s64, &i64);
          warp_c64(s64, i64);
          if (lane == 0) {
            gs->wc64[gwarp].s = s64;
            gs->wc64[gwarp].idx = i64;
          }
          bar_sync_n(barid, gthr);
          if (gwarp == 0) {
            double ss = lane < gnw ? gs->wc64[lane].s : -INFINITY;
            int ii = lane < gnw ? gs->wc64[lane].idx : 0x7FFFFFFF;
            warp_c64(ss, ii);
            if (grp == 0 && lane == 0)
              mbar_arrive_expect_tx(&tl->dbar[dp], J * (uint32_t)sizeof(Cand64));
            if (lane < (int)C) {
              const uint32_t ra = peer_addr(&tl->drecv[dp][jslice], (uint32_t)lane);
              const uint32_t rb = peer_addr(&tl->dbar[dp], (uint32_t)lane);
              const unsigned long long bits = __double_as_longlong(ss);
              st_async_v4(ra, __uint_as_float((uint32_t)bits),
                          __uint_as_float((uint32_t)(bits >> 32)), __int_as_float(ii), 0.f, rb);
            }
          }
          if (!mbar_wait(&tl->dbar[dp], dph)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
          double ss = lane < (int)J ? tl->drecv[dp][lane].s : -INFINITY;
          int ii = lane < (int)J ? tl->drecv[dp][lane].idx : 0x7FFFFFFF;
          warp_c64(ss, ii);
          winner = ii;
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

    // ---------------- end of unit ----------------
    if (k == a.K && leader && tid == 0) {
      if (!VERIFY) {
        if (badT) {
          a.bonus_out[unit] = -1;
          if (a.tokens_out) a.tokens_out[unit * a.R + a.K] = -1;
        }
      } else {
        a.acc_len[unit] = acc_len;
        for (int jj = 0; jj < a.R; ++jj) {
          int tok = -1;
          if (jj < acc_len) tok = a.draft[unit * a.K + jj];
          else if (jj == acc_len) tok = emitted;
          a.out_tokens[unit * a.R + jj] = tok;
        }
      }
    }
  }

  // Last row's TV partials go to the leader, which hands them to its bookkeeping warp.
  if (want_tv && nrows > 0) {
    bar_sync_n(barid, gthr);
    if (gwarp == 0) {
      float tvp = lane < gnw ? gs->tvw[lane] : 0.f;
      tvp = warp_sum(tvp);
      if (leader && grp == 0 && lane == 0) mbar_arrive_expect_tx(&tl->fbar, J * 4u);
      if (lane == 0)
        st_async_b32(peer_addr(&tl->frecv[jslice], 0), __float_as_uint(tvp),
                     peer_addr(&tl->fbar, 0));
      if (leader && grp == 0) {
        if (!mbar_wait(&tl->fbar, 0)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
        const int slot = (int)(nrows % kLogN);
        if (nrows >= kLogN &&
            !mbar_wait(&tl->logempty[slot], (uint32_t)(((nrows / kLogN) - 1) & 1)))
          raise_err(a.dev_err, SD_DEV_TIMEOUT);
        if (lane < (int)J) tl->log[slot].m[lane].tvprev = tl->frecv[lane];
        __syncwarp();
        if (lane == 0) mbar_arrive(&tl->logfull[slot]);
      }
    }
  }
  cluster_sync();  // all messages into this CTA have landed; peers may exit
}

// ====================================================================== SMC-SD kernel
// Pipelined kernel for SMC-SD rounds: every row has a target and a draft half;
// the last row of each particle also draws the bonus token.  A cluster of C
// CTAs walks its particles' rows in order; CTA r owns vocabulary slice r.
//
// Warp roles of a CTA:
//   producers (one per 32 x 32 entries of the slice), row by row: move the
//     row's slices from the ring to registers, warp maxima, exps (one MUFU
//     exp2 per entry) and sums; the exps of both halves go to tensor memory
//     (TMEM, two row buffers per warp); post the (max, sum) partials.  In the
//     row after a particle's last row they also screen that row's bonus-token
//     candidates from its exps, still in TMEM.
//   consumers (four, one per TMEM lane quarter), one row behind: once the
//     row's messages are in, rebuild its normalisers, read the exps back from
//     TMEM and take the TV partial sum |p - q|; then hand the row buffer back.
//   communication: turns the producers' partials into one 32-byte message per
//     row for every CTA of the cluster (st.async into distributed shared
//     memory, completing on the receiver's mbarrier -- no cluster barrier on
//     the row path), sends each row's TV partial and bonus candidate to the
//     leader, and refills the ring with bulk async copies (no multicast).
//   bookkeeping (leader only): fp64 lse, log-probs, log-weights, TV and bonus
//     tokens (near-ties settled exactly in fp64).
// MUFU work (producers) and the exchange plus TV (consumers) overlap; every
// element is read from HBM once and exponentiated once.

constexpr int kRing = 8;     // message slots per CTA
constexpr int kLead = 2;     // rows a CTA's messages can run ahead of the leader's
constexpr int kMaxStages = 4;
constexpr uint32_t kTmemCols = 512;  // all of the SM's tensor memory (one CTA per SM)
constexpr int kConsumers = 4;        // phase-B warps, one per TMEM lane quarter
constexpr int kMaxThreadsSmc = 640;  // up to 14 producers + 4 consumers + 2 service warps
static_assert(kMaxThreadsSmc / 32 - kConsumers - 2 <= 16, "one lane per producer in each half-warp");
constexpr size_t kMinSmem = 120 * 1024;  // > half an SM's shared memory: one CTA per SM

struct alignas(16) BMsg {  // one slice's phase-B results for the leader
  float tv, s, lo, hi;
  float ohi;
  int idx;
  float pad0, pad1;
};

struct alignas(128) SmcTail {
  uint64_t full[kMaxStages];    // ring stages (target and draft slices of one row)
  uint64_t empty[kMaxStages];   // producers done reading a stage
  uint64_t afull[2];  // producers done with a row (exps in TMEM, partials posted)
  uint64_t bfull[2];  // consumers done with a row (TV partials, candidates posted)
  uint64_t tfree[2];  // consumers done reading a TMEM row buffer
  uint64_t sfin;      // producers posted the last row's bonus candidates
  uint64_t rbar[kRing], bbar[kRing], adone[kRing];
  int abort_flag;
  uint32_t tmem_base;
  Msg recv[kRing][kMaxCluster];
  BMsg brecv[kRing][kMaxCluster];
  float4 wpart[2][kMaxWarps];
  float wtv[2][kConsumers];
  Cand wcand[4][kMaxWarps];  // producers' bonus candidates, by row & 3
  // Raw logits of a row's draft token at its owner, by row & 3: producer warps
  // are not ordered among themselves, so the owner may post row it+2's value
  // before the slowest warp has finished row it (and so before the
  // communication warp has read it); row it+3 needs row it's TMEM buffer back,
  // which comes after that read.
  float zx[4][2];
};

// Wait sites, reported in bits 8..15 of the error word with SD_DEV_TIMEOUT.
enum WaitSite : uint32_t {
  kWsFull = 1u << 8, kWsRow = 1u << 10, kWsAfull = 1u << 11, kWsBfull = 1u << 12,
  kWsAdone = 1u << 13, kWsBook = 1u << 14, kWsBmsg = 1u << 15
};

// Bounded wait; after one expiry every later wait of the CTA returns at once
// (the outputs are then garbage, SD_DEV_TIMEOUT is set, nothing hangs).
__device__ __forceinline__ void swait(uint64_t* bar, uint32_t parity, SmcTail* tl, uint32_t* err,
                                      uint32_t site) {
  if (mbar_try_wait(bar, parity)) return;
  volatile int* ab = &tl->abort_flag;
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if ((i & 15u) == 0 && *ab) return;  // (a shared-memory read every 16 polls only)
    if (mbar_try_wait(bar, parity)) return;
  }
  *ab = 1;
  raise_err(err, SD_DEV_TIMEOUT | site);
}

// Paired warp reductions (two independent values per shuffle round).
// Warp maxima in one instruction each (redux.sync on f32, sm_100a): NaN inputs
// are dropped (as fmaxf does), or with .NaN make the result NaN.
__device__ __forceinline__ void warp_max2(float& a, float& b) {
  asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(a));
  asm volatile("redux.sync.max.f32 %0, %0, 0xffffffff;" : "+f"(b));
}
__device__ __forceinline__ void warp_max2_nan(float& a, float& b) {
  asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(a));
  asm volatile("redux.sync.max.NaN.f32 %0, %0, 0xffffffff;" : "+f"(b));
}
__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, a, o);
    const float y = __shfl_xor_sync(0xffffffffu, b, o);
    a += x;
    b += y;
  }
}
// fp64 lse of a row's target and draft halves from the C slice partials of its
// messages: half-warp 0 sums the target's, half-warp 1 the draft's, and both
// logs run at once.  Slice factors use MUFU exp2, the sums and logs are fp64.
struct Lse2 {
  double T, D;
};
__device__ __noinline__ Lse2 row_lse_pair(const Msg* e, uint32_t C, float MT, float MD,
                                          double inv_tau64, float cT) {
  const int lane = threadIdx.x & 31, h = lane >> 4, l = lane & 15;
  const bool has = l < (int)C;
  const float m = has ? (h ? e[l].mD : e[l].mT) : -INFINITY;
  const float s = has ? (h ? e[l].sD : e[l].sT) : 0.f;
  const float M = h ? MD : MT;
  double t = m > -INFINITY ? (double)s * (double)ex2((m - M) * cT) : 0.0;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  const double lse = (double)M * inv_tau64 + log(t);
  return Lse2{__shfl_sync(0xffffffffu, lse, 0), __shfl_sync(0xffffffffu, lse, 16)};
}

// Row normalisers from per-slice (max, sum) partials held one per lane.  A
// NaN partial max drops out of the max but makes the sum NaN.
struct Norm {
  float MT, ST, MD, SD;
  bool badT, badD;
};
__device__ __forceinline__ Norm row_norm(float pm1, float ps1, float pm2, float ps2, float cT) {
  Norm n;
  n.MT = pm1;
  n.MD = pm2;
  warp_max2(n.MT, n.MD);
  n.ST = part_term(pm1, ps1, n.MT, cT);
  n.SD = part_term(pm2, ps2, n.MD, cT);
  warp_sum2(n.ST, n.SD);
  n.badT = !(n.MT > -INFINITY && n.MT < INFINITY && n.ST > 0.f && n.ST < INFINITY);
  n.badD = !(n.MD > -INFINITY && n.MD < INFINITY && n.SD > 0.f && n.SD < INFINITY);
  return n;
}

// Exact fp64 bonus draw over a whole target row (a near-tie the fp32 screen
// could not settle; rare).  One warp.
template <typename TIn>
__device__ __noinline__ int exact_bonus_row(const TIn* row, int V, double tau64, float inv_tau,
                                            float lo_star, const Stream st, uint32_t rowid) {
  const int lane = threadIdx.x & 31;
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int q = lane; q * 4 < V; q += 32) {
    const U4 w = st.at((uint32_t)q, rowid);
    for (int j = 0; j < 4; ++j) {
      const int v = q * 4 + j;
      if (v >= V) break;
      const float z = Elem<TIn>::get(row, v);
      const float a32 = z * inv_tau;
      if (!(a32 + kGumbelMaxF + 1e-3f >= lo_star)) continue;
      const float g32 = gumbel_f32(uniform_f32(word_of(w, j)));
      const float hi = a32 + g32 + 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
      if (!(hi >= lo_star)) continue;
      const double s64 = (double)z / tau64 + gumbel_f64(uniform_f64(word_of(w, j)));
      c64_merge(best, bi, s64, v);
    }
  }
  warp_c64(best, bi);
  return bi == 0x7FFFFFFF ? -1 : bi;
}

// Candidate from one kept entry: a = z / tau in fp32, Gumbel in fp32, with
// bounds that contain the exact fp64 score.
__device__ __noinline__ Cand bonus_cand_a(float a32, float u, int v) {
  const float g32 = gumbel_f32(u);
  Cand cd;
  cd.s = a32 + g32;
  const float d = 4e-6f + 4.8e-7f * (fabsf(a32) + 2.f * fabsf(g32));
  cd.lo = cd.s - d;
  cd.hi = cd.s + d;
  cd.ohi = -INFINITY;
  cd.idx = v;
  cd.pad0 = cd.pad1 = cd.pad2 = 0;
  return cd;
}

// 16-byte chunks of a row slice: 8 bf16 or 4 fp32 entries.
template <typename TIn>
struct Chunk;
template <>
struct Chunk<uint16_t> {
  static constexpr int EPC = 8;
  using Acc = uint32_t;  // two bf16 maxima
  static constexpr uint32_t kAcc0 = 0xFF80FF80u;
  static __device__ __forceinline__ void max_acc(Acc& m, const uint4& v) {
    m = bmax2_nan(m, bmax2_nan(bmax2_nan(v.x, v.y), bmax2_nan(v.z, v.w)));
  }
  static __device__ __forceinline__ float acc_f32(Acc m) {
    return fmax_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
  }
  static __device__ __forceinline__ float elem(const uint4& v, int j) {  // j: compile-time
    const uint32_t w = (j >> 1) == 0 ? v.x : ((j >> 1) == 1 ? v.y : ((j >> 1) == 2 ? v.z : v.w));
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
  static __device__ __forceinline__ uint4 neg_inf() {
    return make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
  }
  static __device__ __noinline__ uint4 gather(const uint16_t* st, const uint16_t* g, int e0, int len,
                                              int tma_len) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t h[2];
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int e = e0 + 2 * j + b;
        h[b] = e < tma_len ? (uint32_t)st[e] : (e < len ? (uint32_t)g[e] : 0xFF80u);
      }
      w[j] = h[0] | (h[1] << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Chunk<float> {
  static constexpr int EPC = 4;
  using Acc = float;
  static constexpr float kAcc0 = -INFINITY;
  static __device__ __forceinline__ void max_acc(Acc& m, const uint4& v) {
    m = fmax_nan(m, fmax_nan(fmax_nan(__uint_as_float(v.x), __uint_as_float(v.y)),
                             fmax_nan(__uint_as_float(v.z), __uint_as_float(v.w))));
  }
  static __device__ __forceinline__ float acc_f32(Acc m) { return m; }
  static __device__ __forceinline__ float elem(const uint4& v, int j) {  // j: compile-time
    return __uint_as_float(j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w)));
  }
  static __device__ __forceinline__ uint4 neg_inf() {
    return make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);
  }
  static __device__ __noinline__ uint4 gather(const float* st, const float* g, int e0, int len,
                                              int tma_len) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + j;
      w[j] = e < tma_len ? __float_as_uint(st[e])
                         : (e < len ? __float_as_uint(g[e]) : 0xFF800000u);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// Chunk starting at slice entry e0: from the ring stage where the bulk copy
// covered it, else from HBM; entries past the slice read as -inf (a chunk
// wholly past it without a call: the last lanes of a CTA hold such chunks).
template <typename TIn>
__device__ __forceinline__ uint4 load_chunk(const TIn* st, const TIn* g, int e0, int len,
                                            int tma_len) {
  if (e0 + Chunk<TIn>::EPC <= tma_len) return *reinterpret_cast<const uint4*>(st + e0);
  if (e0 >= len) return Chunk<TIn>::neg_inf();
  return Chunk<TIn>::gather(st, g, e0, len, tma_len);
}

// Bonus-token screen over this thread's target entries of a particle's last
// row, from the exps held in TMEM (relative to the warp max), in two halves of
// sixteen entries (one loop body, kept small for the instruction cache): the
// four Philox blocks of a half are drawn together (independent, so they
// overlap); an entry whose y = e * rho = e^{a - Tref} proves it cannot win is
// dropped before any log; the few kept entries become candidates with fp32
// bounds, their logit over tau recovered as a = m/tau + ln(e) (m: the warp max
// the exp is relative to; the error is far inside the candidate bounds).
template <typename TIn>
__device__ __forceinline__ Cand bonus_screen(uint32_t tcolT, int s0, int len, int tid, int ncomp,
                                             float rho, float mw_a, const Stream bst,
                                             uint32_t rowid) {
  constexpr int EPC = Chunk<TIn>::EPC;
  Cand cd = cand_empty();
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    float e[16];
    __syncwarp();
    tmem_ld16(tcolT + 16u * (uint32_t)h, e);
    tmem_wait_ld();
    // One bound for the half: with y <= ymax = emax * rho, keep_bonus needs
    // u >= thr(ymax) (same fp32 steps, monotone), so a word whose top 23 bits
    // m = w >> 9 fall below mstar fails for every entry here;
    // u = (m + 1/2) 2^-23 >= thr  <=>  m >= thr 2^23 - 1/2 (exact in fp32).
    float emax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) emax = fmaxf(emax, e[i]);
    const float thr = (1.0f - (emax * rho) * 1.001f) - 2.4e-7f;
    const uint32_t mstar = thr > 0.f ? (uint32_t)ceilf(thr * 8388608.f - 0.5f) : 0u;
    U4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // entries 16h + 4q .. +3 of this thread: one Philox block
      const int i = 16 * h + 4 * q;
      const int eg = (tid + (i / EPC) * ncomp) * EPC + (i % EPC);
      w[q] = bst.at((uint32_t)((s0 + eg) >> 2), rowid);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 16 * h + 4 * q;
      const int eg = (tid + (i / EPC) * ncomp) * EPC + (i % EPC);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if ((word_of(w[q], j) >> 9) < mstar) continue;
        const float ej = e[4 * q + j];
        const float u = uniform_f32(word_of(w[q], j));
        if (keep_bonus(ej * rho, u) && eg + j < len && ej > 0.f)
          cd = cand_merge(cd, bonus_cand_a(mw_a + logf(ej), u, s0 + eg + j));
      }
    }
  }
  return cd;
}

template <typename TIn>
__device__ void smc_bookkeep(const ScoreArgs& a, SmcTail* tl, uint32_t C, uint32_t cid, uint32_t G,
                             int nrows, bool want_tv) {
  const int lane = threadIdx.x & 31;
  const Stream bst(a.seed, a.round, SD_STREAM_BONUS);
  const bool lane_tokens = a.K <= 32;
  double logw_acc = 0.0;
  bool unit_bad = false;
  bool prev_bad = false, prev_badT = false;
  int k = 0;
  int64_t unit = cid;
  // draft tokens of a particle, one per lane; prefetched one particle ahead
  auto fetch_tokens = [&](int64_t u) -> int {
    return (lane_tokens && lane < a.K && u < a.units) ? a.draft[u * a.K + lane] : -1;
  };
  auto fetch_prev = [&](int64_t u) -> double {
    return (a.logw_prev && u < a.units) ? a.logw_prev[u] : 0.0;
  };
  int xs = -1, xs_next = fetch_tokens(unit);
  double lwp = 0.0, lwp_next = fetch_prev(unit);
  for (int it = 0; it <= nrows; ++it) {
    bool bad_cur = false, badT_cur = false;
    if (it < nrows) {
      if (k == 0) {
        xs = xs_next;
        lwp = lwp_next;
        xs_next = fetch_tokens(unit + G);
        lwp_next = fetch_prev(unit + G);
        logw_acc = 0.0;
        unit_bad = false;
      }
      const int slot = it % kRing;
      const int64_t rowT = unit * a.R + k;
      swait(&tl->rbar[slot], (uint32_t)((it / kRing) & 1), tl, a.dev_err, kWsBook);
      const Msg* e = tl->recv[slot];
      const bool has = lane < (int)C;
      const Norm nm = row_norm(has ? e[lane].mT : -INFINITY, has ? e[lane].sT : 0.f,
                               has ? e[lane].mD : -INFINITY, has ? e[lane].sD : 0.f, a.cT);
      const Lse2 lse = row_lse_pair(e, C, nm.MT, nm.MD, a.inv_tau64, a.cT);
      const double lse64T = lse.T, lse64D = lse.D;
      bad_cur = nm.badT || nm.badD;
      badT_cur = nm.badT;
      int x = -1;
      float zxT = 0.f, zxD = 0.f;
      if (k < a.K) {
        x = lane_tokens ? __shfl_sync(0xffffffffu, xs, k) : a.draft[unit * a.K + k];
        if (x >= 0 && x < a.V) {
          const Msg& o = e[x / a.slice];
          zxT = o.zxT;
          zxD = o.zxD;
        }
      }
      if (lane == 0) {
        if (bad_cur) raise_err(a.dev_err, SD_DEV_NONFINITE);
        if (a.lse_out) {
          a.lse_out[rowT * 2 + 0] = nm.badT ? NAN : lse64T;
          a.lse_out[rowT * 2 + 1] = nm.badD ? NAN : lse64D;
        }
        if (k < a.K) {
          const bool x_ok = x >= 0 && x < a.V;
          double lp = NAN, lq = NAN;
          if (!x_ok) raise_err(a.dev_err, SD_DEV_TOKEN_OOB);
          if (x_ok && !bad_cur) {
            lp = (double)zxT * a.inv_tau64 - lse64T;
            lq = (double)zxD * a.inv_tau64 - lse64D;
          } else {
            unit_bad = true;
          }
          logw_acc += lp - lq;
          if (a.lp_out) {
            a.lp_out[(unit * a.K + k) * 2 + 0] = lp;
            a.lp_out[(unit * a.K + k) * 2 + 1] = lq;
          }
        } else {
          a.logw_out[unit] = unit_bad ? NAN : lwp + logw_acc;
        }
      }
      if (k == a.K && a.tokens_out) {
        if (lane_tokens) {
          if (lane < a.K) a.tokens_out[unit * a.R + lane] = xs;
        } else {
          for (int j = lane; j < a.K; j += 32) a.tokens_out[unit * a.R + j] = a.draft[unit * a.K + j];
        }
      }
    }
    if (it >= 1) {  // row it-1: TV partials and the bonus candidates
      const int p = it - 1;
      const int pslot = p % kRing;
      const int pk = k == 0 ? a.R - 1 : k - 1;
      const int64_t punit = k == 0 ? unit - G : unit;
      swait(&tl->bbar[pslot], (uint32_t)((p / kRing) & 1), tl, a.dev_err, kWsBmsg);
      const BMsg* bm = tl->brecv[pslot];
      const bool has = lane < (int)C;
      float tv = has ? bm[lane].tv : 0.f;
      Cand c = cand_empty();
      if (pk == a.K && has) {
        c.s = bm[lane].s;
        c.lo = bm[lane].lo;
        c.hi = bm[lane].hi;
        c.ohi = bm[lane].ohi;
        c.idx = bm[lane].idx;
      }
      // Both of row p's slots (row message and leader message) are read: the
      // CTAs may now run far enough ahead to refill them (the leader's
      // communication warp waits for this before each row message).
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->adone[pslot]);
      tv = warp_sum(tv);
      if (want_tv && lane == 0) a.tv_out[punit * a.R + pk] = prev_bad ? NAN : 0.5f * tv;
      if (pk == a.K) {
        c = warp_cand(c);
        int winner;
        if (prev_badT || c.idx == 0x7FFFFFFF) winner = -1;
        else if (c.ohi < c.lo) winner = c.idx;
        else
          winner = exact_bonus_row<TIn>((const TIn*)a.zT + (punit * a.R + pk) * a.ld, a.V, a.tau64,
                                        a.inv_tau, c.lo, bst, (uint32_t)punit);
        if (lane == 0) {
          a.bonus_out[punit] = winner;
          if (a.tokens_out) a.tokens_out[punit * a.R + a.K] = winner;
        }
      }
    }
    prev_bad = bad_cur;
    prev_badT = badT_cur;
    if (it < nrows && ++k == a.R) {
      k = 0;
      unit += G;
    }
  }
}

template <typename TIn>
__global__ void __launch_bounds__(kMaxThreadsSmc, 1) smc_kernel(const ScoreArgs a) {
  using CK = Chunk<TIn>;
  constexpr int EPC = CK::EPC;
  constexpr int CPT = kEPT / EPC;          // chunks per producer thread
  constexpr bool HOLD = sizeof(TIn) == 2;  // bf16: raw chunks stay in registers for pass 2
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // warps [0, nA): producers; [nA, nA + 4): consumers; then communication, bookkeeping
  const int nA = (int)(blockDim.x >> 5) - kConsumers - 2;
  const int ncomp = nA * 32;
  const int wComm = nA + kConsumers, wBook = wComm + 1;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const uint32_t cid = cluster_id(), G = num_clusters();
  const int nS = a.stages;
  const size_t sb = a.stage_bytes;  // one tensor's slice; a stage holds both
  SmcTail* tl = reinterpret_cast<SmcTail*>(smem + (size_t)nS * 2 * sb);

  const int s0 = (int)rank * a.slice;
  const int len = max(0, min(a.slice, a.V - s0));
  const int tma_len = a.use_tma ? ((len * (int)sizeof(TIn)) & ~15) / (int)sizeof(TIn) : 0;
  const uint32_t tma_bytes = (uint32_t)tma_len * (uint32_t)sizeof(TIn);
  const int64_t my_units = (int64_t)cid < a.units ? (a.units - 1 - cid) / G + 1 : 0;
  const int nrows = (int)(my_units * a.R);
  const bool leader = rank == 0;
  const bool want_tv = a.tv_out != nullptr;
  const float cT = a.cT;

  if (tid == 0) {
    for (int st = 0; st < nS; ++st) {
      mbar_init(&tl->full[st], 1);
      mbar_init(&tl->empty[st], (uint32_t)nA);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tl->afull[b], (uint32_t)nA);
      mbar_init(&tl->bfull[b], kConsumers);
      mbar_init(&tl->tfree[b], kConsumers);
    }
    mbar_init(&tl->sfin, (uint32_t)nA);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&tl->rbar[i], 1);
      mbar_init(&tl->bbar[i], 1);
      mbar_init(&tl->adone[i], 1);
    }
    tl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == wComm) {  // the communication warp owns the CTA's tensor memory
    tmem_alloc(&tl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  cluster_sync();

  if (warp == wBook) {  // ---------------- bookkeeping (leader only)
    if (leader) smc_bookkeep<TIn>(a, tl, C, cid, G, nrows, want_tv);
    cluster_sync();
    return;
  }

  if (warp == wComm) {  // ---------------- communication warp
    const uint64_t pol = policy_evict_first();
    // stage st <- row `it` of this cluster: unit cid + (it / R) * G, position it % R
    auto issue = [&](int it, int st) {
      const int64_t row = ((int64_t)cid + (int64_t)(it / a.R) * G) * a.R + (it % a.R);
      unsigned char* stg = smem + (size_t)st * 2 * sb;
      mbar_arrive_expect_tx(&tl->full[st], 2u * tma_bytes);
      if (tma_bytes) {
        bulk_load(stg, (const TIn*)a.zT + row * a.ld + s0, tma_bytes, &tl->full[st], pol);
        bulk_load(stg + sb, (const TIn*)a.zD + row * a.ld + s0, tma_bytes, &tl->full[st], pol);
      }
    };
    if (lane == 0)
      for (int i = 0; i < nS && i < nrows; ++i) issue(i, i);
    int k = 0, stage = 0;  // position and ring stage of row it
    for (int it = 0; it <= nrows; ++it) {
      if (it < nrows) {  // row it: refill its stage once read, then its message
        if (it + nS < nrows) {
          swait(&tl->empty[stage], (uint32_t)((it / nS) & 1), tl, a.dev_err, kWsAfull);
          if (lane == 0) issue(it + nS, stage);
        }
        swait(&tl->afull[it & 1], (uint32_t)((it >> 1) & 1), tl, a.dev_err, kWsAfull);
        const float4 wp =
            lane < nA ? tl->wpart[it & 1][lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        float mT = wp.x, mD = wp.z;
        warp_max2_nan(mT, mD);  // a warp's NaN max (NaN in its entries) must reach the sum
        float sumT = part_term(wp.x, wp.y, mT, cT), sumD = part_term(wp.z, wp.w, mD, cT);
        warp_sum2(sumT, sumD);
        float zxT = 0.f, zxD = 0.f;
        if (k < a.K) {
          zxT = tl->zx[it & 3][0];
          zxD = tl->zx[it & 3][1];
        }
        const int slot = it % kRing;
        // Once this message is out, the other CTAs can send rows up to it + kLead;
        // their slots must already have been read by the bookkeeping warp.
        if (leader && it + kLead >= kRing) {
          const int r = it + kLead - kRing;
          swait(&tl->adone[r % kRing], (uint32_t)((r / kRing) & 1), tl, a.dev_err, kWsAdone);
        }
        if (lane == 0) mbar_arrive_expect_tx(&tl->rbar[slot], C * (uint32_t)sizeof(Msg));
        if (lane < (int)C) {
          const uint32_t ra = peer_addr(&tl->recv[slot][rank], (uint32_t)lane);
          const uint32_t rb = peer_addr(&tl->rbar[slot], (uint32_t)lane);
          st_async_v4(ra, mT, sumT, mD, sumD, rb);
          st_async_v4(ra + 16, zxT, zxD, 0.f, 0.f, rb);
        }
        if (++stage == nS) stage = 0;
      }
      if (it >= 1) {  // row it-1: the consumers are done with it
        const int p = it - 1;
        swait(&tl->bfull[p & 1], (uint32_t)((p >> 1) & 1), tl, a.dev_err, kWsBfull);
        float tv = lane < kConsumers ? tl->wtv[p & 1][lane] : 0.f;
        tv = warp_sum(tv);
        const int pk = k == 0 ? a.R - 1 : k - 1;
        Cand cd = cand_empty();
        if (pk == a.K) {  // the producers screened it during the next row (the last: on its own)
          if (p == nrows - 1) swait(&tl->sfin, 0u, tl, a.dev_err, kWsBfull);
          if (lane < nA) cd = tl->wcand[p & 3][lane];
          cd = warp_cand(cd);
        }
        const int pslot = p % kRing;
        if (leader && lane == 0) mbar_arrive_expect_tx(&tl->bbar[pslot], C * (uint32_t)sizeof(BMsg));
        if (lane == 0) {
          const uint32_t ra = peer_addr(&tl->brecv[pslot][rank], 0);
          const uint32_t rb = peer_addr(&tl->bbar[pslot], 0);
          st_async_v4(ra, want_tv ? tv : 0.f, cd.s, cd.lo, cd.hi, rb);
          st_async_v4(ra + 16, cd.ohi, __int_as_float(cd.idx), 0.f, 0.f, rb);
        }
      }
      if (it < nrows && ++k == a.R) k = 0;
    }
    // Every bulk copy this warp issued has landed before the CTA may exit (they
    // all have, unless a wait gave up above).
    if (lane == 0)
      for (int st = 0; st < nS && st < nrows; ++st)
        mbar_wait(&tl->full[st], (uint32_t)(((nrows - 1 - st) / nS) & 1));
    cluster_sync();
    tmem_fence_after();
    tmem_dealloc(tl->tmem_base, kTmemCols);
    return;
  }

  if (warp >= nA) {  // ---------------- consumers
    // Quarter q of TMEM holds the rows of producers q, q + 4, ...: 128 columns
    // from 128 * (w / 4), two row buffers of 64 (32 target exps, 32 draft exps).
    const int q = warp & 3, cidx = warp - nA;
    const uint32_t tq = tl->tmem_base + ((32u * (uint32_t)q) << 16);
    for (int p = 0; p < nrows; ++p) {
      swait(&tl->afull[p & 1], (uint32_t)((p >> 1) & 1), tl, a.dev_err, kWsAfull);
      swait(&tl->rbar[p % kRing], (uint32_t)((p / kRing) & 1), tl, a.dev_err, kWsRow);
      __syncwarp();
      tmem_fence_after();
      const Msg* rv = tl->recv[p % kRing];
      const bool has = lane < (int)C;
      const Norm nm = row_norm(has ? rv[lane].mT : -INFINITY, has ? rv[lane].sT : 0.f,
                               has ? rv[lane].mD : -INFINITY, has ? rv[lane].sD : 0.f, cT);
      // Scale factors of all producers at once (one exp2 and one division per
      // lane instead of a chain per producer): lane w < 16 takes producer w's
      // target half, lane 16 + w its draft half; lanes < 16 also -scD / scT.
      const int wl = lane & 15;
      const bool hD = lane >= 16;
      const float4 wq =
          wl < nA ? tl->wpart[p & 1][wl] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
      const float mwl = hD ? wq.z : wq.x;
      const bool badl = hD ? nm.badD : nm.badT;
      const float scl = (!badl && mwl > -INFINITY)
                            ? ex2((mwl - (hD ? nm.MD : nm.MT)) * cT) * (1.f / (hD ? nm.SD : nm.ST))
                            : 0.f;
      const float sco = __shfl_xor_sync(0xffffffffu, scl, 16);
      const float nrl = scl > 0.f ? -(sco / scl) : 0.f;
      float tv = 0.f;
      for (int w = q; w < nA; w += 4) {
        const float scT = __shfl_sync(0xffffffffu, scl, w);
        const float scD = __shfl_sync(0xffffffffu, scl, w + 16);
        const float nr = __shfl_sync(0xffffffffu, nrl, w);
        const uint32_t tb = tq + 128u * (uint32_t)(w >> 2) + 64u * (uint32_t)(p & 1);
        if (scT > 0.f) {
          // sum |p - q| = scT * sum |eT - eD * (scD / scT)|: one fused op per entry,
          // exactly 0 for identical rows (ratio 1).
          const float2 nr2 = f2(nr);
          float eT[kEPT], eD[kEPT];
          tmem_ld32(tb, eT);
          tmem_ld32(tb + 32u, eD);
          tmem_wait_ld();
          float2 t2 = f2(0.f), u2 = f2(0.f);
#pragma unroll
          for (int j = 0; j < kEPT; j += 4) {
            const float2 d0 = __ffma2_rn(make_float2(eD[j], eD[j + 1]), nr2, make_float2(eT[j], eT[j + 1]));
            const float2 d1 = __ffma2_rn(make_float2(eD[j + 2], eD[j + 3]), nr2, make_float2(eT[j + 2], eT[j + 3]));
            t2 = __fadd2_rn(t2, make_float2(fabsf(d0.x), fabsf(d0.y)));
            u2 = __fadd2_rn(u2, make_float2(fabsf(d1.x), fabsf(d1.y)));
          }
          tv += scT * ((t2.x + t2.y) + (u2.x + u2.y));
        } else if (scD > 0.f) {  // no target mass in these entries (or a bad row): TV part = sum q
          float eD[kEPT];
          tmem_ld32(tb + 32u, eD);
          tmem_wait_ld();
          float sq = 0.f;
#pragma unroll
          for (int j = 0; j < kEPT; ++j) sq += eD[j];
          tv += scD * sq;
        }
      }
      // the row buffer goes back to the producers
      __syncwarp();
      tmem_fence_before();
      if (lane == 0) mbar_arrive(&tl->tfree[p & 1]);
      tv = warp_sum(tv);
      if (lane == 0) tl->wtv[p & 1][cidx] = tv;
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->bfull[p & 1]);
    }
    __syncwarp();
    tmem_fence_before();
    cluster_sync();
    return;
  }

  // ---------------- producers
  const uint32_t tcol = tl->tmem_base + ((32u * (uint32_t)(warp & 3)) << 16) + 128u * (uint32_t)(warp >> 2);
  int k = 0;           // position of row `it` within its particle
  int64_t unit = cid;  // particle of row `it`
  int stage = 0;
  uint32_t phase = 0;
  int x_next = (nrows > 0 && a.K > 0) ? a.draft[(int64_t)cid * a.K] : -1;
  float mwT_prev = -INFINITY;  // this warp's raw target max of the previous row

  // Bonus-token screen of row p (a particle's last row) over this warp's entries,
  // from its exps still in TMEM, once the row's messages give its max M.
  auto screen = [&](int p, int64_t punit) {
    swait(&tl->rbar[p % kRing], (uint32_t)((p / kRing) & 1), tl, a.dev_err, kWsRow);
    __syncwarp();
    const Msg* rv = tl->recv[p % kRing];
    const bool has = lane < (int)C;
    const Norm nm = row_norm(has ? rv[lane].mT : -INFINITY, has ? rv[lane].sT : 0.f,
                             has ? rv[lane].mD : -INFINITY, has ? rv[lane].sD : 0.f, cT);
    Cand cd = cand_empty();
    if (!nm.badT && mwT_prev > -INFINITY) {
      // Tref = M/tau + g_min - margin bounds the winning score from below
      const float margin = 1e-5f + 2e-7f * fabsf(nm.MT * a.inv_tau);
      const float rho = ex2((mwT_prev - nm.MT) * cT + (-kGumbelMinF + margin) * kLog2e);
      cd = bonus_screen<TIn>(tcol + 64u * (uint32_t)(p & 1), s0, len, tid, ncomp, rho,
                             mwT_prev * a.inv_tau, Stream(a.seed, a.round, SD_STREAM_BONUS),
                             (uint32_t)punit);
    }
    cd = warp_cand(cd);
    if (lane == 0) tl->wcand[p & 3][warp] = cd;
  };

  for (int it = 0; it < nrows; ++it) {
    const int x = k < a.K ? x_next : -1;
    {  // prefetch the draft token of row it+1
      int kn = k + 1;
      int64_t un = unit;
      if (kn == a.R) {
        kn = 0;
        un += G;
      }
      x_next = (it + 1 < nrows && kn < a.K) ? a.draft[un * a.K + kn] : -1;
    }
    swait(&tl->full[stage], phase, tl, a.dev_err, kWsFull);
    const int64_t row = unit * a.R + k;
    const TIn* stT = reinterpret_cast<const TIn*>(smem + (size_t)stage * 2 * sb);
    const TIn* stD = reinterpret_cast<const TIn*>(smem + (size_t)stage * 2 * sb + sb);
    const TIn* gT = (const TIn*)a.zT + row * a.ld + s0;
    const TIn* gD = (const TIn*)a.zD + row * a.ld + s0;
    // pass 1: maxima
    uint4 rT[HOLD ? CPT : 1], rD[HOLD ? CPT : 1];
    typename CK::Acc aT = CK::kAcc0, aD = CK::kAcc0;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int e0 = (tid + c * ncomp) * EPC;
      const uint4 vT = load_chunk<TIn>(stT, gT, e0, len, tma_len);
      const uint4 vD = load_chunk<TIn>(stD, gD, e0, len, tma_len);
      CK::max_acc(aT, vT);
      CK::max_acc(aD, vD);
      if (HOLD) {
        rT[HOLD ? c : 0] = vT;
        rD[HOLD ? c : 0] = vD;
      }
    }
    if (x >= s0 && x < s0 + len) {  // the owner of the draft token records its raw logits
      const int le = x - s0;
      if (((le / EPC) % ncomp) == tid) {
        tl->zx[it & 3][0] = le < tma_len ? Elem<TIn>::get(stT, le) : Elem<TIn>::get(gT, le);
        tl->zx[it & 3][1] = le < tma_len ? Elem<TIn>::get(stD, le) : Elem<TIn>::get(gD, le);
      }
    }
    if (HOLD) {  // the stage is in registers now: it can be refilled
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->empty[stage]);
    }
    float mwT = CK::acc_f32(aT), mwD = CK::acc_f32(aD);
    warp_max2_nan(mwT, mwD);
    const float mwTs = mwT == -INFINITY ? 0.f : mwT;
    const float mwDs = mwD == -INFINITY ? 0.f : mwD;
    // this warp's TMEM row buffer (it & 1) is free once the consumers are done with row it-2
    if (it >= 2) swait(&tl->tfree[it & 1], (uint32_t)(((it - 2) >> 1) & 1), tl, a.dev_err, kWsRow);
    __syncwarp();
    tmem_fence_after();
    // pass 2: e = 2^(z cT - m cT) for both halves, summed and parked in TMEM
    const float2 c2 = f2(cT), nT2 = f2(-mwTs * cT), nD2 = f2(-mwDs * cT);
    const uint32_t tb = tcol + 64u * (uint32_t)(it & 1);
    float2 accT = f2(0.f), accD = f2(0.f);
    float eT[8], eD[8];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      uint4 vT, vD;
      if (HOLD) {
        vT = rT[HOLD ? c : 0];
        vD = rD[HOLD ? c : 0];
      } else {
        const int e0 = (tid + c * ncomp) * EPC;
        vT = load_chunk<TIn>(stT, gT, e0, len, tma_len);
        vD = load_chunk<TIn>(stD, gD, e0, len, tma_len);
      }
#pragma unroll
      for (int j = 0; j < EPC; j += 2) {
        const int i = (c * EPC + j) & 7;
        const float2 tT = __ffma2_rn(make_float2(CK::elem(vT, j), CK::elem(vT, j + 1)), c2, nT2);
        const float2 tD = __ffma2_rn(make_float2(CK::elem(vD, j), CK::elem(vD, j + 1)), c2, nD2);
        eT[i] = ex2(tT.x);
        eT[i + 1] = ex2(tT.y);
        eD[i] = ex2(tD.x);
        eD[i + 1] = ex2(tD.y);
        accT = __fadd2_rn(accT, make_float2(eT[i], eT[i + 1]));
        accD = __fadd2_rn(accD, make_float2(eD[i], eD[i + 1]));
        if (i + 2 == 8) {  // eight entries done: park them (whole warp, converged)
          const uint32_t col = (uint32_t)((c * EPC + j + 2) - 8);
          __syncwarp();
          tmem_st8(tb + col, eT);
          tmem_st8(tb + 32u + col, eD);
        }
      }
    }
    if (!HOLD) {  // pass 2 re-read the stage
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->empty[stage]);
    }
    float sTw = accT.x + accT.y, sDw = accD.x + accD.y;
    warp_sum2(sTw, sDw);
    if (lane == 0) tl->wpart[it & 1][warp] = make_float4(mwT, sTw, mwD, sDw);
    if (k == 0 && it > 0) screen(it - 1, unit - G);  // the previous row ended a particle
    mwT_prev = mwT;
    __syncwarp();
    tmem_wait_st();
    tmem_fence_before();
    if (lane == 0) mbar_arrive(&tl->afull[it & 1]);
    if (++stage == nS) {
      stage = 0;
      phase ^= 1u;
    }
    if (++k == a.R) {
      k = 0;
      unit += G;
    }
  }
  if (nrows > 0) {  // the last row ends a particle too
    screen(nrows - 1, unit - G);
    __syncwarp();
    if (lane == 0) mbar_arrive(&tl->sfin);
  }
  __syncwarp();
  tmem_fence_before();
  cluster_sync();
}

// ------------------------------------------------------------------ host side
struct LaunchPlan {
  int C, groups, threads, stages, slice;
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

// Chooses (cluster size C, warp groups per CTA) for this vocabulary: each
// group holds its slice in 32 registers per thread per row, all groups plus the
// service warp fit in 512 threads, J = C * groups <= 32 slices, and at least two
// ring stages fit in shared memory.  Among the feasible choices it keeps the
// most SMs busy for this many units, then prefers more groups (more overlap).
// SMCSD_GROUPS=1..3 caps the number of groups.  Plans are cached per
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
  int max_groups = kMaxGroups;
  if (const char* env = getenv("SMCSD_GROUPS")) {
    const int g = atoi(env);
    if (g >= 1 && g <= kMaxGroups) max_groups = g;
  }
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t tail = sizeof(Tail) + 128;
  bool found = false;
  int64_t best_score = -1;
  for (int C = 1; C <= kMaxCluster; ++C) {
    for (int ng = max_groups; ng >= 1; --ng) {
      if (C * ng > kMaxSlices) continue;
      const int slice = (int)(((int64_t)(V + C * ng - 1) / (C * ng) + 7) / 8 * 8);
      const int gthr = std::max(32, (int)(((slice + kEPT - 1) / kEPT + 31) / 32 * 32));
      const int threads = ng * gthr + 32;  // + the service warp
      if (threads > kMaxThreads || gthr / 32 > kMaxWarps) continue;
      const uint32_t sb = (uint32_t)(((int64_t)slice * ng * esize + 127) / 128 * 128);
      int stages = 0;
      for (int st = 4; st >= 2; --st)
        if ((size_t)st * 2 * sb + tail <= (size_t)optin) {
          stages = st;
          break;
        }
      if (stages == 0) continue;
      const size_t smem = (size_t)stages * 2 * sb + tail;
      const int nc = max_active_clusters(fn, C, threads, smem);
      if (nc <= 0) continue;
      const int64_t score = (std::min<int64_t>(ukey, nc) * C) * 8 + ng;
      if (score > best_score) {
        best_score = score;
        best = LaunchPlan{C, ng, threads, stages, slice, sb, smem, nc};
        found = true;
      }
    }
  }
  if (found) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)best.smem);
    cache[key] = best;
  }
  return found;
}

// Launch plan of the SMC-SD kernel: producer warps covering the slice at 32
// entries per thread per row (at most 16, so that two TMEM row buffers per
// warp fit), four consumers and the two service warps; the deepest ring
// that fits, and at least kMinSmem of shared memory so that one CTA runs per
// SM (it takes all of the SM's tensor memory).  Among the cluster sizes it
// keeps the most SMs busy for this many particles.
static bool make_plan_smc(const void* fn, int V, int esize, int64_t units, LaunchPlan& best) {
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
  bool found = false;
  int64_t best_score = -1;
  for (int C = 1; C <= kMaxCluster; ++C) {
    const int slice = (int)(((int64_t)(V + C - 1) / C + 7) / 8 * 8);
    const int ncomp = std::max(32, (int)(((slice + kEPT - 1) / kEPT + 31) / 32 * 32));
    const int threads = ncomp + 32 * (kConsumers + 2);  // + consumers, communication, bookkeeping
    if (threads > kMaxThreadsSmc || ncomp / 32 > kMaxWarps) continue;
    const uint32_t sb = (uint32_t)(((int64_t)slice * esize + 127) / 128 * 128);
    int nS = 0;
    for (int st = kMaxStages; st >= 2; --st)
      if ((size_t)st * 2 * sb + sizeof(SmcTail) + 128 <= (size_t)optin) {
        nS = st;
        break;
      }
    if (nS == 0) continue;
    const size_t smem = std::max((size_t)nS * 2 * sb + sizeof(SmcTail) + 128, kMinSmem);
    const int nc = max_active_clusters(fn, C, threads, smem);
    if (nc <= 0) continue;
    const int64_t score = std::min<int64_t>(ukey, nc) * C * 8 + nS;
    if (score > best_score) {
      best_score = score;
      best = LaunchPlan{C, 1, threads, nS, slice, sb, smem, nc};
      found = true;
    }
  }
  if (found) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)best.smem);
    cache[key] = best;
  }
  return found;
}

template <typename TIn>
static sd_status launch_smc(ScoreArgs& a, cudaStream_t stream) {
  const void* fn = (const void*)smc_kernel<TIn>;
  LaunchPlan p;
  if (!make_plan_smc(fn, a.V, (int)sizeof(TIn), a.units, p)) return SD_ERR_UNSUPPORTED;
  a.slice = p.slice;
  a.groups = 1;
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
  void* args[] = {(void*)&a};
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  return SD_OK;
}

template <typename TIn, bool VERIFY>
static sd_status launch_score(ScoreArgs& a, cudaStream_t stream) {
  const void* fn = kernel_ptr<TIn, VERIFY>();
  LaunchPlan p;
  if (!make_plan(fn, a.V, (int)sizeof(TIn), a.units, p)) return SD_ERR_UNSUPPORTED;
  a.slice = p.slice;
  a.groups = p.groups;
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
  a.inv_tau64 = 1.0 / (double)tau;
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
  return dt == SD_BF16 ? launch_smc<uint16_t>(a, s) : launch_smc<float>(a, s);
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
