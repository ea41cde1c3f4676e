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
// Software-pipelined variant for SMC-SD rounds (every row has a target and a
// draft half, the last row of each particle draws the bonus token).
//
// Iteration r of a CTA:
//   1. move row r's slices from the ring to registers, per-thread and warp max;
//   2. wait for row r-1's messages (sent one iteration ago, so their latency is
//      hidden behind step 1), rebuild row r-1's normalisers, screen row r-1's
//      bonus candidates if it ends a particle;
//   3. one fused loop over this thread's entries: row r's exp2 (MUFU) and sums,
//      row r-1's TV from its target exps (shared-memory buffer) and draft exps
//      (registers) -- each slot is read and then overwritten in place;
//   4. one CTA barrier; warp 0 combines the warp partials and pushes row r's
//      message (carrying row r-1's TV partial) to every CTA of the cluster, and
//      row r-1's bonus candidate to the leader.
// Row r's exps thus stay on chip until its TV is taken one iteration later;
// the bookkeeping warp of the leader turns the messages into log-weights, TV
// and bonus tokens (deciding near-ties exactly in fp64).

constexpr int kRing = 4;  // message slots: the bookkeeping warp may lag two rows

struct alignas(128) SmcTail {
  uint64_t full[2];
  uint64_t rbar[kRing], cbar[kRing], bdone[kRing];
  uint64_t fbar, pad;
  Msg recv[kRing][kMaxCluster];
  Cand crecv[kRing][kMaxCluster];
  float frecv[kMaxCluster];
  float4 wpart[2][kMaxWarps];  // warp scratch, by iteration parity: warps may run one
  float tvw[2][kMaxWarps];     // iteration ahead of warp 0, which reads the previous one
  Cand wcand[2][kMaxWarps];
  float zx[2][2];
};

// Paired warp reductions (two independent values per shuffle round).
__device__ __forceinline__ void warp_max2(float& a, float& b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, a, o);
    const float y = __shfl_xor_sync(0xffffffffu, b, o);
    a = fmaxf(a, x);
    b = fmaxf(b, y);
  }
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
__device__ __forceinline__ void warp_sum3(float& a, float& b, float& c) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, a, o);
    const float y = __shfl_xor_sync(0xffffffffu, b, o);
    const float z = __shfl_xor_sync(0xffffffffu, c, o);
    a += x;
    b += y;
    c += z;
  }
}
// fp64 lse of a row from per-slice partials (one per lane, `has` marks valid
// lanes); the slice factors use MUFU exp2, the sum and the log are fp64.
__device__ __noinline__ double row_lse_fast(float m, float s, float M, bool has, double tau64,
                                            float cT) {
  const double t = (has && m > -INFINITY) ? (double)s * (double)ex2((m - M) * cT) : 0.0;
  return (double)M / tau64 + log(warp_sum_d(t));
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

template <typename TIn>
__device__ void smc_bookkeep(const ScoreArgs& a, SmcTail* tl, uint32_t C, uint32_t cid, uint32_t G,
                             int nrows, bool want_tv) {
  const int lane = threadIdx.x & 31;
  double logw_acc = 0.0;
  bool unit_bad = false;
  bool prev_bad = false;
  int cuse[kRing] = {0, 0, 0, 0};
  const Stream bst(a.seed, a.round, SD_STREAM_BONUS);
  int k = 0;
  int64_t unit = cid;
  int64_t prev_row = -1;
  for (int it = 0; it < nrows; ++it, prev_row = unit * a.R + k, (++k == a.R ? (k = 0, unit += G) : 0)) {
    const int slot = it % kRing;
    const int64_t rowT = unit * a.R + k;
    if (!mbar_wait(&tl->rbar[slot], (uint32_t)((it / kRing) & 1))) raise_err(a.dev_err, SD_DEV_TIMEOUT);
    const Msg* e = tl->recv[slot];
    const bool has = lane < (int)C;
    const float pm1 = has ? e[lane].mT : -INFINITY, ps1 = has ? e[lane].sT : 0.f;
    const float pm2 = has ? e[lane].mD : -INFINITY, ps2 = has ? e[lane].sD : 0.f;
    float tvsum = has ? e[lane].tvprev : 0.f;
    float MT = pm1, MD = pm2;
    warp_max2(MT, MD);
    float ST = part_term(pm1, ps1, MT, a.cT), SD = part_term(pm2, ps2, MD, a.cT);
    warp_sum3(ST, SD, tvsum);
    const bool badT = !(MT > -INFINITY && MT < INFINITY && ST > 0.f && ST < INFINITY);
    const bool badD = !(MD > -INFINITY && MD < INFINITY && SD > 0.f && SD < INFINITY);
    const bool bad = badT || badD;
    const double lse64T = row_lse_fast(pm1, ps1, MT, has, a.tau64, a.cT);
    const double lse64D = row_lse_fast(pm2, ps2, MD, has, a.tau64, a.cT);
    int x = -1;
    float zxT = 0.f, zxD = 0.f;
    if (k < a.K) {
      x = a.draft[unit * a.K + k];
      if (x >= 0 && x < a.V) {
        const Msg& o = e[x / a.slice];
        zxT = o.zxT;
        zxD = o.zxD;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tl->bdone[slot]);  // message slot no longer needed
    if (lane == 0) {
      if (k == 0) {
        logw_acc = 0.0;
        unit_bad = false;
      }
      if (it > 0 && want_tv) a.tv_out[prev_row] = prev_bad ? NAN : 0.5f * tvsum;
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
          lp = (double)zxT / a.tau64 - lse64T;
          lq = (double)zxD / a.tau64 - lse64D;
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
          for (int jj = 0; jj < a.K; ++jj) a.tokens_out[unit * a.R + jj] = a.draft[unit * a.K + jj];
      }
    }
    prev_bad = bad;
    if (k == a.K) {  // bonus token: merge the slices' candidates
      const uint32_t ph = (uint32_t)(cuse[slot] & 1);
      ++cuse[slot];
      if (!mbar_wait(&tl->cbar[slot], ph)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
      Cand c = has ? tl->crecv[slot][lane] : cand_empty();
      c = warp_cand(c);
      int winner;
      if (badT || c.idx == 0x7FFFFFFF) winner = -1;
      else if (c.ohi < c.lo) winner = c.idx;
      else
        winner = exact_bonus_row<TIn>((const TIn*)a.zT + rowT * a.ld, a.V, a.tau64, a.inv_tau, c.lo,
                                      bst, (uint32_t)unit);
      __syncwarp();
      if (lane == 0) {
        a.bonus_out[unit] = winner;
        if (a.tokens_out) a.tokens_out[unit * a.R + a.K] = winner;
      }
    }
  }
  if (want_tv && nrows > 0) {  // the last row's TV arrives on its own
    if (!mbar_wait(&tl->fbar, 0)) raise_err(a.dev_err, SD_DEV_TIMEOUT);
    float v = lane < (int)C ? tl->frecv[lane] : 0.f;
    v = warp_sum(v);
    if (lane == 0) a.tv_out[prev_row] = prev_bad ? NAN : 0.5f * v;
  }
}

// Fused per-thread pass: row r's exps (CUR) and row r-1's TV (PREV).
template <int CPT, int EPC, bool CUR, bool PREV>
__device__ __forceinline__ void fused_pass(float* xt, float* xd, float* dp, float4* tb, int tid,
                                           int nthr, float mwT, float mwD, float cT, float scT,
                                           float scD, float& sT, float& sD, float& tv) {
  constexpr int EPT = CPT * EPC;
  float2 aT = make_float2(0.f, 0.f), aD = make_float2(0.f, 0.f);
  float t0 = 0.f, t1 = 0.f;
  const float2 mT2 = make_float2(-mwT, -mwT), mD2 = make_float2(-mwD, -mwD);
  const float2 c2 = make_float2(cT, cT);
#pragma unroll
  for (int q = 0; q < EPT / 4; ++q) {
    float4& slot = tb[q * nthr + tid];
    float4 old = make_float4(0.f, 0.f, 0.f, 0.f);
    if (PREV) old = slot;
    float4 nw;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = q * 4 + h * 2;
      if (PREV) {  // separately rounded products: identical rows give exactly 0
        const float o0 = h == 0 ? old.x : old.z, o1 = h == 0 ? old.y : old.w;
        t0 += fabsf(__fmul_rn(o0, scT) - __fmul_rn(dp[i], scD));
        t1 += fabsf(__fmul_rn(o1, scT) - __fmul_rn(dp[i + 1], scD));
      }
      if (CUR) {
        const float2 at = __fmul2_rn(__fadd2_rn(make_float2(xt[i], xt[i + 1]), mT2), c2);
        const float2 ad = __fmul2_rn(__fadd2_rn(make_float2(xd[i], xd[i + 1]), mD2), c2);
        const float2 et = make_float2(ex2(at.x), ex2(at.y));
        const float2 ed = make_float2(ex2(ad.x), ex2(ad.y));
        aT = __fadd2_rn(aT, et);
        aD = __fadd2_rn(aD, ed);
        if (h == 0) {
          nw.x = et.x;
          nw.y = et.y;
        } else {
          nw.z = et.x;
          nw.w = et.y;
        }
        dp[i] = ed.x;
        dp[i + 1] = ed.y;
      }
    }
    if (CUR) slot = nw;
  }
  sT = aT.x + aT.y;
  sD = aD.x + aD.y;
  tv = t0 + t1;
  (void)EPC;
}

// Row normalisers from per-slice (max, sum) partials held one per lane.
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

template <typename TIn, int CPT>
__global__ void __launch_bounds__(kMaxThreads, 1) smc_kernel(const ScoreArgs a) {
  constexpr int EPC = 16 / (int)sizeof(TIn);
  constexpr int EPT = CPT * EPC;
  static_assert(EPT == kEPT, "entries per thread");
  extern __shared__ __align__(128) unsigned char smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // warps [0, nwarps): compute; warp nwarps: communication; warp nwarps+1: bookkeeping
  const int ncomp = blockDim.x - 64, nwarps = ncomp >> 5;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const uint32_t cid = cluster_id(), G = num_clusters();
  float4* tbuf = reinterpret_cast<float4*>(smem + (size_t)2 * 2 * a.stage_bytes);
  SmcTail* tl = reinterpret_cast<SmcTail*>(smem + (size_t)2 * 2 * a.stage_bytes +
                                           (size_t)ncomp * EPT * sizeof(float));

  const int s0 = (int)rank * a.slice;
  const int len = max(0, min(a.slice, a.V - s0));
  const int tma_len = a.use_tma ? ((len * (int)sizeof(TIn)) & ~15) / (int)sizeof(TIn) : 0;
  const uint32_t tma_bytes = (uint32_t)tma_len * (uint32_t)sizeof(TIn);
  const int64_t my_units = (int64_t)cid < a.units ? (a.units - 1 - cid) / G + 1 : 0;
  const int nrows = (int)(my_units * a.R);
  const bool leader = rank == 0;
  const bool want_tv = a.tv_out != nullptr;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) mbar_init(&tl->full[s], 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&tl->rbar[i], 1);
      mbar_init(&tl->cbar[i], 1);
      mbar_init(&tl->bdone[i], 1);
    }
    mbar_init(&tl->fbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  cluster_sync();

  if (warp == nwarps + 1) {  // ---------------- bookkeeping (leader only)
    if (leader) smc_bookkeep<TIn>(a, tl, C, cid, G, nrows, want_tv);
    cluster_sync();
    return;
  }

  const uint64_t pol = policy_evict_first();
  // stage (row & 1) <- row `it` of this cluster: unit cid + (it / R) * G, position it % R
  auto issue = [&](int it) {
    const int s = it & 1;
    const int64_t row = ((int64_t)cid + (int64_t)(it / a.R) * G) * a.R + (it % a.R);
    unsigned char* stg = smem + (size_t)s * 2 * a.stage_bytes;
    mbar_arrive_expect_tx(&tl->full[s], tma_bytes * 2u);
    if (tma_bytes) {
      bulk_load(stg, (const TIn*)a.zT + row * a.ld + s0, tma_bytes, &tl->full[s], pol);
      bulk_load(stg + a.stage_bytes, (const TIn*)a.zD + row * a.ld + s0, tma_bytes, &tl->full[s], pol);
    }
  };

  if (warp == nwarps) {  // ---------------- communication warp
    if (lane == 0)
      for (int it = 0; it < nrows && it < 2; ++it) issue(it);
    int k = 0;
    for (int it = 0; it <= nrows; ++it) {
      const bool cur = it < nrows;
      const int par = it & 1;
      bar_sync_n(1, ncomp + 32);  // compute warps have posted their partials of iteration `it`
      if (cur && lane == 0 && it + 2 < nrows) issue(it + 2);  // stage `par` is free again
      float tvp = lane < nwarps ? tl->tvw[par][lane] : 0.f;
      if (cur) {
        const float4 wp =
            lane < nwarps ? tl->wpart[par][lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        float mT = wp.x, mD = wp.z;
        warp_max2(mT, mD);
        float sT = part_term(wp.x, wp.y, mT, a.cT), sD = part_term(wp.z, wp.w, mD, a.cT);
        warp_sum3(sT, sD, tvp);
        const bool owner_known = k < a.K;
        float zxT = 0.f, zxD = 0.f;
        if (owner_known) {
          zxT = tl->zx[par][0];
          zxD = tl->zx[par][1];
        }
        const int slot = it % kRing;
        if (leader && it >= 2 &&
            !mbar_wait(&tl->bdone[(it - 2) % kRing], (uint32_t)(((it - 2) / kRing) & 1)))
          raise_err(a.dev_err, SD_DEV_TIMEOUT);
        if (lane == 0) mbar_arrive_expect_tx(&tl->rbar[slot], C * (uint32_t)sizeof(Msg));
        if (lane < (int)C) {
          const uint32_t ra = peer_addr(&tl->recv[slot][rank], (uint32_t)lane);
          const uint32_t rb = peer_addr(&tl->rbar[slot], (uint32_t)lane);
          st_async_v4(ra, mT, sT, mD, sD, rb);
          st_async_v4(ra + 16, zxT, zxD, want_tv ? tvp : 0.f, 0.f, rb);
        }
      } else {
        tvp = warp_sum(tvp);
        if (want_tv && nrows > 0) {  // final iteration: the last row's TV goes to the leader
          if (leader && lane == 0) mbar_arrive_expect_tx(&tl->fbar, C * 4u);
          if (lane == 0)
            st_async_b32(peer_addr(&tl->frecv[rank], 0), __float_as_uint(tvp), peer_addr(&tl->fbar, 0));
        }
      }
      if (it > 0 && ((it - 1) % a.R) == a.K) {  // row it-1's bonus candidate goes to the leader
        const int pslot = (it - 1) % kRing;
        Cand c2 = lane < nwarps ? tl->wcand[par][lane] : cand_empty();
        c2 = warp_cand(c2);
        if (leader && lane == 0) mbar_arrive_expect_tx(&tl->cbar[pslot], C * (uint32_t)sizeof(Cand));
        if (lane == 0) {
          const uint32_t ra = peer_addr(&tl->crecv[pslot][rank], 0);
          const uint32_t rb = peer_addr(&tl->cbar[pslot], 0);
          st_async_v4(ra, c2.s, c2.lo, c2.hi, c2.ohi, rb);
          st_async_v4(ra + 16, __int_as_float(c2.idx), 0.f, 0.f, 0.f, rb);
        }
      }
      if (++k == a.R) k = 0;
    }
    cluster_sync();
    return;
  }

  // ---------------- compute warps
  float xt[EPT], xd[EPT], dp[EPT];
  float mwT_p = 0.f, mwD_p = 0.f;  // previous row's warp maxima (safe forms)
  bool okT_p = false, okD_p = false;
  const float inv_tau = a.inv_tau;
  int k = 0;          // position of row `it` within its particle
  int64_t unit = cid; // particle of row `it`
  int x_next = (nrows > 0 && a.K > 0) ? a.draft[(int64_t)cid * a.K] : -1;

  for (int it = 0; it <= nrows; ++it) {
    const bool cur = it < nrows;
    const bool prev = it > 0;
    const int par = it & 1;
    const int x = (cur && k < a.K) ? x_next : -1;
    {  // prefetch the draft token of row it+1
      int kn = k + 1;
      int64_t un = unit;
      if (kn == a.R) {
        kn = 0;
        un += G;
      }
      x_next = (it + 1 < nrows && kn < a.K) ? a.draft[un * a.K + kn] : -1;
    }

    // ---- previous row: normalisers, bonus screen (only the pending draft exps are live)
    float scT = 0.f, scD = 0.f;
    if (prev) {
      const int pit = it - 1;
      const int pslot = pit % kRing;
      const int pk = k == 0 ? a.R - 1 : k - 1;
      const int64_t punit = k == 0 ? unit - G : unit;
      if (!mbar_wait(&tl->rbar[pslot], (uint32_t)((pit / kRing) & 1))) raise_err(a.dev_err, SD_DEV_TIMEOUT);
      const Msg* rv = tl->recv[pslot];
      const bool has = lane < (int)C;
      const Norm nm = row_norm(has ? rv[lane].mT : -INFINITY, has ? rv[lane].sT : 0.f,
                               has ? rv[lane].mD : -INFINITY, has ? rv[lane].sD : 0.f, a.cT);
      scT = (!nm.badT && okT_p) ? ex2((mwT_p - nm.MT) * a.cT) / nm.ST : 0.f;
      scD = (!nm.badD && okD_p) ? ex2((mwD_p - nm.MD) * a.cT) / nm.SD : 0.f;
      if (pk == a.K) {
        Cand cd = cand_empty();
        if (!nm.badT && okT_p) {
          // Tref = M/tau + g_min - margin: a lower bound on the winning score.
          const float margin = 1e-5f + 2e-7f * fabsf(nm.MT * inv_tau);
          const float rho = ex2((mwT_p - nm.MT) * a.cT + (-kGumbelMinF + margin) * kLog2e);
          const float mw_a = mwT_p * inv_tau;
          const Stream st(a.seed, a.round, SD_STREAM_BONUS);
#pragma unroll
          for (int q = 0; q < EPT / 4; ++q) {
            const int c = q / (EPC / 4);
            const int e0 = (tid + c * ncomp) * EPC + (q % (EPC / 4)) * 4;
            if (e0 >= len) continue;
            const float4 ev = tbuf[q * ncomp + tid];
            const float y0 = ev.x * rho, y1 = ev.y * rho, y2 = ev.z * rho, y3 = ev.w * rho;
            if (fmaxf(fmaxf(y0, y1), fmaxf(y2, y3)) < kYSkip) continue;
            const int v0 = s0 + e0;
            const U4 w = st.at((uint32_t)(v0 >> 2), (uint32_t)punit);
            const float u0 = uniform_f32(w.x), u1 = uniform_f32(w.y);
            const float u2 = uniform_f32(w.z), u3 = uniform_f32(w.w);
            const bool k0 = keep_bonus(y0, u0) && e0 + 0 < len;
            const bool k1 = keep_bonus(y1, u1) && e0 + 1 < len;
            const bool k2 = keep_bonus(y2, u2) && e0 + 2 < len;
            const bool k3 = keep_bonus(y3, u3) && e0 + 3 < len;
            if (k0 | k1 | k2 | k3) {
              if (k0) cd = cand_merge(cd, bonus_cand(ev.x, u0, mw_a, v0));
              if (k1) cd = cand_merge(cd, bonus_cand(ev.y, u1, mw_a, v0 + 1));
              if (k2) cd = cand_merge(cd, bonus_cand(ev.z, u2, mw_a, v0 + 2));
              if (k3) cd = cand_merge(cd, bonus_cand(ev.w, u3, mw_a, v0 + 3));
            }
          }
        }
        cd = warp_cand(cd);
        if (lane == 0) tl->wcand[par][warp] = cd;
      }
    }

    // ---- current row: ring -> registers, maxima
    float mwT = -INFINITY, mwD = -INFINITY;
    if (cur) {
      if (!mbar_wait(&tl->full[par], (uint32_t)((it >> 1) & 1))) raise_err(a.dev_err, SD_DEV_TIMEOUT);
      const int64_t row = unit * a.R + k;
      const TIn* stT = reinterpret_cast<const TIn*>(smem + (size_t)par * 2 * a.stage_bytes);
      const TIn* stD = reinterpret_cast<const TIn*>(smem + (size_t)par * 2 * a.stage_bytes + a.stage_bytes);
      const TIn* gT = (const TIn*)a.zT + row * a.ld + s0;
      const TIn* gD = (const TIn*)a.zD + row * a.ld + s0;
      mwT = load_slice<TIn, CPT>(xt, stT, gT, len, tma_len, tid, ncomp);
      mwD = load_slice<TIn, CPT>(xd, stD, gD, len, tma_len, tid, ncomp);
      if (x >= s0 && x < s0 + len) {
        const int le = x - s0;
        if (((le / EPC) % ncomp) == tid) {
          tl->zx[par][0] = le < tma_len ? Elem<TIn>::get(stT, le) : Elem<TIn>::get(gT, le);
          tl->zx[par][1] = le < tma_len ? Elem<TIn>::get(stD, le) : Elem<TIn>::get(gD, le);
        }
      }
      warp_max2(mwT, mwD);
    }
    const float mwTs = mwT == -INFINITY ? 0.f : mwT;
    const float mwDs = mwD == -INFINITY ? 0.f : mwD;

    // ---- fused pass: row r exps + row r-1 TV ----
    float sT = 0.f, sD = 0.f, tv = 0.f;
    if (cur && prev)
      fused_pass<CPT, EPC, true, true>(xt, xd, dp, tbuf, tid, ncomp, mwTs, mwDs, a.cT, scT, scD, sT,
                                       sD, tv);
    else if (cur)
      fused_pass<CPT, EPC, true, false>(xt, xd, dp, tbuf, tid, ncomp, mwTs, mwDs, a.cT, scT, scD,
                                        sT, sD, tv);
    else if (prev)
      fused_pass<CPT, EPC, false, true>(xt, xd, dp, tbuf, tid, ncomp, mwTs, mwDs, a.cT, scT, scD,
                                        sT, sD, tv);
    warp_sum3(sT, sD, tv);
    if (lane == 0) {
      tl->wpart[par][warp] = make_float4(mwT, sT, mwD, sD);
      tl->tvw[par][warp] = tv;
    }
    // (A) post this iteration's partials to the communication warp and move on
    asm volatile("bar.arrive 1, %0;" ::"r"(ncomp + 32) : "memory");
    mwT_p = mwTs;
    mwD_p = mwDs;
    okT_p = mwT > -INFINITY;
    okD_p = mwD > -INFINITY;
    if (cur && ++k == a.R) {
      k = 0;
      unit += G;
    }
  }
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

// Launch plan of the pipelined SMC-SD kernel: one warp group per CTA, two
// ring stages, plus the target-exps buffer (32 fp32 per compute thread).
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
    const int threads = ncomp + 64;  // + communication and bookkeeping warps
    if (threads > kMaxThreads || ncomp / 32 > kMaxWarps) continue;
    const uint32_t sb = (uint32_t)(((int64_t)slice * esize + 127) / 128 * 128);
    const size_t smem = (size_t)2 * 2 * sb + (size_t)ncomp * kEPT * 4 + sizeof(SmcTail) + 128;
    if (smem > (size_t)optin) continue;
    const int nc = max_active_clusters(fn, C, threads, smem);
    if (nc <= 0) continue;
    const int64_t score = std::min<int64_t>(ukey, nc) * C;
    if (score > best_score) {
      best_score = score;
      best = LaunchPlan{C, 1, threads, 2, slice, sb, smem, nc};
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
  const void* fn = (const void*)smc_kernel<TIn, (int)(kEPT * sizeof(TIn) / 16)>;
  LaunchPlan p;
  if (!make_plan_smc(fn, a.V, (int)sizeof(TIn), a.units, p)) return SD_ERR_UNSUPPORTED;
  a.slice = p.slice;
  a.groups = 1;
  a.stages = 2;
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, smc_kernel<TIn, (int)(kEPT * sizeof(TIn) / 16)>, a);
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
