// Standard speculative-decoding verification kernel (N = 1).
//
// What it computes (include/smcsd.h, sd_verify_reject): per sequence, K
// drafted tokens are checked in order against the target; the first rejection
// discards the rest and draws one token from the residual max(p - q, 0); if all
// K are accepted a bonus token is drawn from the target row K+1.  Sources:
// "Faster LLM Inference via Sequential Monte Carlo", section 1 (standard SD,
// rejection, KV rollback); METASD section 1 (background) and section 2 (TV
// block divergence reported per position).
//
// Design (B200, sm_100a): one thread-block cluster of C CTAs walks a
// sequence's rows in order; CTA r owns vocabulary slice r (split-V) of the
// target and draft rows; the slices stream HBM -> shared memory by bulk async
// copies; each thread keeps 32 entries of each row in registers; per row the
// CTAs exchange (max, sum) partials through distributed shared memory
// (st.async completing on the receivers' mbarriers), then take the fp64
// accept test, the TV from the register-held exps and, at the first
// rejection (or after K acceptances), an exact Gumbel-max draw: an fp32 screen
// with rigorous error bounds keeps only entries that can still win, and
// near-ties are re-scored in fp64.
#include <algorithm>
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>
#include <cuda_runtime.h>

#include "rows.cuh"

namespace smcsd {

constexpr int kMaxThreads = 512;
constexpr int kMaxGroups = 3;
constexpr int kMaxSlices = 32;  // cluster size x groups

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

// Bookkeeping warp of the leader CTA: fp64 lse, log-probs, log-weights, TV and
// per-particle outputs, fed row by row through a small shared-memory ring so
// that none of this sits on the compute warps' critical path.
__device__ void verify_bookkeep(const ScoreArgs& a, Tail* tl, uint32_t J, int64_t nrows, bool want_tv) {
  const int lane = threadIdx.x & 31;
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
    const int k = e.k;
    const bool hasD = k < a.K;
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
    const int64_t rowD = unit * a.K + k;
    prev_tv_idx = (want_tv && hasD) ? rowD : -1;
    prev_bad = bad;
    __syncwarp();
    if (lane == 0) mbar_arrive(&tl->logempty[slot]);
  }
}

template <typename TIn, int CPT>
__global__ void __launch_bounds__(kMaxThreads, 1) verify_kernel(const ScoreArgs a) {
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
    if (leader) verify_bookkeep(a, tl, J, nrows, want_tv);
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
    const bool hasD = k < a.K;
    const int64_t rowT = unit * a.R + k;
    const int64_t rowD = unit * a.K + k;
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
    const bool hasD = k < a.K;
    const int64_t rowT = unit * a.R + k;
    const int64_t rowD = unit * a.K + k;
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
#pragma unroll
    for (int i = EPT - 1; i >= 0; --i)
      if (xt[i] == mt) amax = s0 + (gtid + (i / EPC) * gthr) * EPC + (i % EPC);
    const float mwT = warp_max(mt);
    const float mwD = hasD ? warp_max(md) : -INFINITY;
    {  // warp argmax: lowest index among lanes holding the warp max
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
      if (lane < gnw && gs->wargv[lane] == m.mT) ai = gs->wargi[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ai = min(ai, __shfl_xor_sync(0xffffffffu, ai, o));
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
    if (k < a.K && !done) {
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
    } else if (bad && leader && tid == 0 && (k < a.K || !done)) {
      raise_err(a.dev_err, SD_DEV_NONFINITE);
    }

    // ---------------- Gumbel-max draws: bonus token / residual token ----------------
    const bool draw_bonus = (k == a.K) && !badT && !done;
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
        emitted = winner;
        done = true;
        if (draw_bonus) acc_len = a.K;
        break;
      }
    }

    // ---------------- end of unit ----------------
    if (k == a.K && leader && tid == 0) {
      a.acc_len[unit] = acc_len;
      for (int jj = 0; jj < a.R; ++jj) {
        int tok = -1;
        if (jj < acc_len) tok = a.draft[unit * a.K + jj];
        else if (jj == acc_len) tok = emitted;
        a.out_tokens[unit * a.R + jj] = tok;
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

template <typename TIn>
static sd_status launch_verify(ScoreArgs& a, cudaStream_t stream) {
  const void* fn = (const void*)verify_kernel<TIn, (int)(kEPT * sizeof(TIn) / 16)>;
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
  return launch_clusters(fn, p, nclusters, a, stream);
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
  ScoreArgs a = {};
  a.zT = zT;
  a.zD = zD;
  a.ld = ld;
  a.V = V;
  a.K = K;
  a.R = K + 1;
  a.units = B;
  fill_tau(a, tau);
  a.draft = draft_tokens;
  a.seed = seed;
  a.round = round;
  a.tv_out = tv_out;
  a.acc_len = accepted_len;
  a.out_tokens = out_tokens;
  a.dev_err = dev_err;
  cudaStream_t s = (cudaStream_t)stream;
  return dt == SD_BF16 ? launch_verify<uint16_t>(a, s) : launch_verify<float>(a, s);
}