#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <cuda_runtime.h>

#include "rows.cuh"

namespace smcsd {

// ====================================================================== SMC-SD kernel
// Pipelined kernel for SMC-SD rounds: every row has a target and a draft half;
// the last row of each particle also draws the bonus token.  A cluster of C
// CTAs walks its particles' rows in order; CTA r owns vocabulary slice r.
//
// Warp roles of a CTA:
//   producers (one per 32 x 32 entries of the slice), row by row: move the
//     row's slices from the ring to registers, warp maxima, exps (one MUFU
//     exp2 per entry) and sums; the exps of both halves go to tensor memory
//     (TMEM, two row buffers per warp); post the (max, sum) partials.
//     On a particle's last row they also park each lane's chunk sums of the
//     target exps for the bonus draw (a two-level Gumbel-max: the block by
//     log-mass plus block noise, then the entry inside it); fp32 rows post
//     their warp's best block candidate instead.
//   consumers (four, one per TMEM lane quarter), one row behind: once the
//     row's messages are in, rebuild its normalisers, read the exps back from
//     TMEM and take the TV partial sum |p - q|; then hand the row buffer back.
//   communication: turns the producers' partials into one 32-byte message per
//     row for every CTA of the cluster (st.async into distributed shared
//     memory, completing on the receiver's mbarrier -- no cluster barrier on
//     the row path), scores a last row's 128-entry blocks from the parked
//     sums once its message is out (off the producers' path), sends each
//     row's TV partial and bonus candidate to the leader, and refills the
//     ring with bulk async copies (no multicast).
//   bookkeeping (leader only): fp64 lse, log-probs, log-weights, TV and bonus
//     tokens: the block from the candidates (a near-tie in fp64 over the
//     row's blocks), then the entry inside it from its 128 logits.
// MUFU work (producers) and the exchange plus TV (consumers) overlap; every
// element is read from HBM once and exponentiated once.

constexpr int kRing = 8;     // message slots per CTA
constexpr int kLead = 2;     // rows a CTA's messages can run ahead of the leader's
constexpr int kMaxStages = 4;
constexpr int kBlk = 128;    // entries per block of the two-level bonus draw
constexpr uint32_t kTmemCols = 512;  // all of the SM's tensor memory (one CTA per SM)
constexpr int kConsumers = 4;        // phase-B warps, one per TMEM lane quarter
constexpr int kMaxThreadsSmc = 640;  // up to 14 producers + 4 consumers + 2 service warps
static_assert(kMaxThreadsSmc / 32 - kConsumers - 2 <= 16, "one lane per producer in each half-warp");
constexpr size_t kMinSmem = 120 * 1024;  // > half an SM's shared memory: one CTA per SM
// bf16 rows: producers park each lane's chunk sums of a particle's last row
// (by row & 3, [warp][chunk][lane]) for the communication warp's block scores.
constexpr int kBpartRows = 4;
constexpr size_t kBpartBytes = (size_t)kBpartRows * kMaxWarps * (kEPT / 8) * 32 * sizeof(float);

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
  uint64_t rbar[kRing], bbar[kRing], adone[kRing];
  int abort_flag;
  uint32_t tmem_base;
  Msg recv[kRing][kMaxCluster];
  BMsg brecv[kRing][kMaxCluster];
  float4 wpart[2][kMaxWarps];
  float wtv[2][kConsumers];
  Cand wcand[4][kMaxWarps];  // producers' best bonus blocks, by row & 3
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

// Bounded waits (common.cuh: bounded_wait, kWaitNs of polling).  After one
// expiry every later abortable wait of the CTA returns at once (outputs are
// then garbage, SD_DEV_TIMEOUT is set, nothing hangs).  The waits that order
// the bulk copies into the ring are not abortable: a stage is refilled only
// after every producer has seen its last copy land, so no copy can still be
// in flight into a CTA that finishes.
__device__ __forceinline__ void swait(uint64_t* bar, uint32_t parity, SmcTail* tl, uint32_t* err,
                                      uint32_t site, bool abortable = true) {
  bounded_wait(bar, parity, &tl->abort_flag, err, site, abortable);
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

// Exact steps of the bonus draw, a two-level Gumbel-max over blocks of kBlk
// entries (the block by its log-mass plus block noise, then the entry inside
// it by plain Gumbel-max).  One warp each; both are fallbacks for the rare
// rows whose fp32 bounds do not settle a step.
//
// The block over a whole target row: lambda_j = log sum exp(z/tau), in fp64.
template <typename TIn>
__device__ __noinline__ int exact_block_row(const TIn* row, int V, double tau64, const Stream st,
                                            uint32_t rowid) {
  const int lane = threadIdx.x & 31;
  const int nb = (V + kBlk - 1) / kBlk;
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int j = lane; j < nb; j += 32) {
    const int v0 = j * kBlk, v1 = min(v0 + kBlk, V);
    double m = -INFINITY;
    for (int v = v0; v < v1; ++v) m = fmax(m, (double)Elem<TIn>::get(row, v) / tau64);
    if (!(m > -INFINITY)) continue;
    double sum = 0.0;
    for (int v = v0; v < v1; ++v) sum += exp((double)Elem<TIn>::get(row, v) / tau64 - m);
    const U4 w = st.at((uint32_t)(j >> 2), rowid);
    c64_merge(best, bi, m + log(sum) + gumbel_f64(uniform_f64(word_of(w, j & 3))), j);
  }
  warp_c64(best, bi);
  return bi == 0x7FFFFFFF ? -1 : bi;
}

// The entry inside block j: argmax (z/tau + g_v), g from the entry stream at
// the global position v (four entries, one Philox block, per lane); fp32
// bounds first, fp64 if two entries come within them.
template <typename TIn>
__device__ __noinline__ int exact_in_block(const TIn* row, int V, int j, float inv_tau,
                                           double tau64, const Stream st, uint32_t rowid) {
  const int lane = threadIdx.x & 31;
  const int v0 = j * kBlk + 4 * lane;
  float z[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  U4 w = U4{0u, 0u, 0u, 0u};
  Cand cd = cand_empty();
  if (lane < kBlk / 4 && v0 < V) {
    w = st.at((uint32_t)(v0 >> 2), rowid);
#pragma unroll
    for (int t = 0; t < 4; ++t) z[t] = v0 + t < V ? Elem<TIn>::get(row, v0 + t) : -INFINITY;
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (z[t] > -INFINITY)
        cd = cand_merge(cd, bonus_cand_a(z[t] * inv_tau, uniform_f32(word_of(w, t)), v0 + t));
  }
  cd = warp_cand(cd);
  if (cd.idx == 0x7FFFFFFF) return -1;
  if (cd.ohi < cd.lo) return cd.idx;
  double best = -INFINITY;
  int bi = 0x7FFFFFFF;
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (z[t] > -INFINITY)
      c64_merge(best, bi, (double)z[t] / tau64 + gumbel_f64(uniform_f64(word_of(w, t))), v0 + t);
  warp_c64(best, bi);
  return bi == 0x7FFFFFFF ? -1 : bi;
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

template <typename TIn>
__device__ void smc_bookkeep(const ScoreArgs& a, SmcTail* tl, uint32_t C, uint32_t cid, uint32_t G,
                             int nrows, bool want_tv) {
  const int lane = threadIdx.x & 31;
  const Stream bst(a.seed, a.round, SD_STREAM_BONUS);
  const Stream blkst(a.seed, a.round, SD_STREAM_BONUS_BLOCK);
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
  // the weight carried in: the previous round's log-weight plus this round's
  // log-potential of the particle (either may be absent)
  auto fetch_prev = [&](int64_t u) -> double {
    if (u >= a.units) return 0.0;
    return (a.logw_prev ? a.logw_prev[u] : 0.0) + (a.log_potential ? a.log_potential[u] : 0.0);
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
        // the block from the candidates when their bounds settle it (else in
        // fp64 over the row), then the entry inside it from its 128 logits
        int winner = -1;
        if (!prev_badT && c.idx != 0x7FFFFFFF) {
          const TIn* brow = (const TIn*)a.zT + (punit * a.R + pk) * a.ld;
          const int jb = c.ohi < c.lo ? c.idx
                                      : exact_block_row<TIn>(brow, a.V, a.tau64, blkst, (uint32_t)punit);
          if (jb >= 0)
            winner = exact_in_block<TIn>(brow, a.V, jb, a.inv_tau, a.tau64, bst, (uint32_t)punit);
        }
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
  float* bpart = reinterpret_cast<float*>(smem + (size_t)nS * 2 * sb + sizeof(SmcTail));

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
    float mwT_row = -INFINITY;   // lane w: producer warp w's target maximum of row it
    Cand pend = cand_empty();    // bf16: bonus candidate of the last row whose message went out
    const Stream blkst(a.seed, a.round, SD_STREAM_BONUS_BLOCK);
    for (int it = 0; it <= nrows; ++it) {
      if (it < nrows) {  // row it: refill its stage once read, then its message
        if (it + nS < nrows) {
          swait(&tl->empty[stage], (uint32_t)((it / nS) & 1), tl, a.dev_err, kWsAfull, false);
          if (lane == 0) issue(it + nS, stage);
        }
        swait(&tl->afull[it & 1], (uint32_t)((it >> 1) & 1), tl, a.dev_err, kWsAfull);
        const float4 wp =
            lane < nA ? tl->wpart[it & 1][lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        mwT_row = wp.x;
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
        if (pk == a.K) {
          if (EPC == 8) {
            cd = pend;  // scored by this warp after the row's message
          } else {  // the producers posted its bonus blocks with the row
            if (lane < nA) cd = tl->wcand[p & 3][lane];
            cd = warp_cand(cd);
          }
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
      if (EPC == 8 && it < nrows && k == a.K) {
        // Row it's bonus blocks from the lanes' parked chunk sums: block (w, c, h)
        // is lanes 16h..16h+15 of warp w's chunk row c, local entries
        // 256 (c nA + w) + 128 h; lambda = ln(sum) + m_w / tau (the exps are
        // relative to the warp's maximum m_w) plus the block's noise, with fp32
        // error bounds.  A block whose exps all flushed to 0 lies > 80 nats below
        // its warp's best block and cannot win (block noise spans < 20).
        const float* bp = bpart + (size_t)(it & (kBpartRows - 1)) * kMaxWarps * CPT * 32;
        const int64_t unit = (int64_t)cid + (int64_t)(it / a.R) * G;
        const int nlb = 2 * CPT * nA;
        Cand cd = cand_empty();
        for (int lb0 = 0; lb0 < nlb; lb0 += 32) {  // warp-uniform trip count (shuffles)
          const int lb = lb0 + lane;
          const int c = lb / (2 * nA), w = (lb >> 1) % nA, h = lb & 1;
          const int local = 256 * (c * nA + w) + 128 * h;
          const float mw = __shfl_sync(0xffffffffu, mwT_row, w);
          if (lb < nlb && local < len) {
            const float4* q = reinterpret_cast<const float4*>(bp + (w * CPT + c) * 32 + 16 * h);
            const float4 q0 = q[0], q1 = q[1], q2 = q[2], q3 = q[3];
            const float sum = ((q0.x + q0.y) + (q0.z + q0.w)) + ((q1.x + q1.y) + (q1.z + q1.w)) +
                              ((q2.x + q2.y) + (q2.z + q2.w)) + ((q3.x + q3.y) + (q3.z + q3.w));
            if (sum > 0.f) {
              const float mws = mw == -INFINITY ? 0.f : mw;
              const int jb = (s0 + local) / kBlk;
              const U4 wr = blkst.at((uint32_t)(jb >> 2), (uint32_t)unit);
              const float g32 = gumbel_f32(uniform_f32(word_of(wr, jb & 3)));
              const float lam = logf(sum) + mws * a.inv_tau;
              const float sc = lam + g32;
              const float d = score_err(lam, g32) + 2e-5f + 2e-7f * fabsf(mws * cT);
              Cand e;
              e.s = sc;
              e.lo = sc - d;
              e.hi = sc + d;
              e.ohi = -INFINITY;
              e.idx = jb;
              e.aux = -1;
              e.pad1 = e.pad2 = 0;
              cd = cand_merge(cd, e);
            }
          }
        }
        pend = warp_cand(cd);
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
  const Stream blkst(a.seed, a.round, SD_STREAM_BONUS_BLOCK);
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
    swait(&tl->full[stage], phase, tl, a.dev_err, kWsFull, false);
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
    const bool brow = k == a.K;  // a particle's last row: the bonus draw's block sums too
    float bsum = 0.f;            // lane q < 8: the target exp sum of this warp's block q
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      float2 bacc = f2(0.f), dacc = f2(0.f);  // this chunk's sums (same order for both halves)
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
        bacc = __fadd2_rn(bacc, make_float2(eT[i], eT[i + 1]));
        dacc = __fadd2_rn(dacc, make_float2(eD[i], eD[i + 1]));
        if (i + 2 == 8) {  // eight entries done: park them (whole warp, converged)
          const uint32_t col = (uint32_t)((c * EPC + j + 2) - 8);
          __syncwarp();
          tmem_st8(tb + col, eT);
          tmem_st8(tb + 32u + col, eD);
        }
      }
      accT = __fadd2_rn(accT, bacc);
      accD = __fadd2_rn(accD, dacc);
      if (brow && EPC == 8) {  // bf16: the lane's chunk sum, scored by the communication warp
        bpart[(size_t)(it & (kBpartRows - 1)) * kMaxWarps * CPT * 32 + (warp * CPT + c) * 32 + lane] =
            bacc.x + bacc.y;
      } else if (brow) {  // fp32: a chunk row of the warp is one block
        float sb = bacc.x + bacc.y;
        if (EPC == 8) {
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) sb += __shfl_xor_sync(0xffffffffu, sb, o);
          const float t0 = __shfl_sync(0xffffffffu, sb, 0), t1 = __shfl_sync(0xffffffffu, sb, 16);
          if (lane == 2 * c) bsum = t0;
          if (lane == 2 * c + 1) bsum = t1;
        } else {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sb += __shfl_xor_sync(0xffffffffu, sb, o);
          if (lane == c) bsum = sb;
        }
      }
    }
    if (brow && EPC != 8) {
      // Block candidates of the bonus draw: lambda_j = ln(sum) + m/tau (the exps
      // are relative to the warp max m) plus the block's Gumbel noise, with fp32
      // error bounds.  A block whose exps all flushed to 0 lies > 80 nats below
      // this warp's best block and cannot win (block noise spans < 20).
      Cand cd = cand_empty();
      if (lane < 8 && bsum > 0.f) {
        const int local = EPC == 8 ? (32 * warp + 16 * (lane & 1) + (lane >> 1) * ncomp) * 8
                                   : (32 * warp + lane * ncomp) * 4;
        if (local < len) {
          const int jb = (s0 + local) / kBlk;
          const U4 w = blkst.at((uint32_t)(jb >> 2), (uint32_t)unit);
          const float g32 = gumbel_f32(uniform_f32(word_of(w, jb & 3)));
          const float lam = logf(bsum) + mwTs * a.inv_tau;
          const float sc = lam + g32;
          // ln(sum) error: exp arguments rounded in fp32 (|t| <= 130 before
          // flushing; the max term 2^-24 |m c| each), ex2.approx, the sum
          const float d = score_err(lam, g32) + 2e-5f + 2e-7f * fabsf(mwTs * cT);
          cd.s = sc;
          cd.lo = sc - d;
          cd.hi = sc + d;
          cd.idx = jb;
        }
      }
      cd = warp_cand(cd);
      if (lane == 0) tl->wcand[it & 3][warp] = cd;
    }
    if (!HOLD) {  // pass 2 re-read the stage
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->empty[stage]);
    }
    float sTw = accT.x + accT.y, sDw = accD.x + accD.y;
    warp_sum2(sTw, sDw);
    if (lane == 0) tl->wpart[it & 1][warp] = make_float4(mwT, sTw, mwD, sDw);
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
  __syncwarp();
  tmem_fence_before();
  cluster_sync();
}

// ------------------------------------------------------------------ host side

// ------------------------------------------------------------------ host side
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
    const int slice = (int)(((int64_t)(V + C - 1) / C + kBlk - 1) / kBlk * kBlk);  // whole blocks
    if (C > 1 && (int64_t)(C - 1) * slice >= V) continue;  // no empty slice
    const int ncomp = std::max(32, (int)(((slice + kEPT - 1) / kEPT + 31) / 32 * 32));
    const int threads = ncomp + 32 * (kConsumers + 2);  // + consumers, communication, bookkeeping
    if (threads > kMaxThreadsSmc || ncomp / 32 > kMaxWarps) continue;
    const uint32_t sb = (uint32_t)(((int64_t)slice * esize + 127) / 128 * 128);
    const size_t extra = esize == 2 ? kBpartBytes : 0;  // parked bonus chunk sums (bf16)
    int nS = 0;
    for (int st = kMaxStages; st >= 2; --st)
      if ((size_t)st * 2 * sb + sizeof(SmcTail) + extra + 128 <= (size_t)optin) {
        nS = st;
        break;
      }
    if (nS == 0) continue;
    const size_t smem = std::max((size_t)nS * 2 * sb + sizeof(SmcTail) + extra + 128, kMinSmem);
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
  return launch_clusters(fn, p, nclusters, a, stream);
}

}  // namespace smcsd

using namespace smcsd;

extern "C" sd_status smcsd_score(const void* zT, const void* zD, sd_dtype dt, int B, int N, int K,
                                 int V, int64_t ld, const int32_t* draft_tokens, float tau,
                                 uint64_t seed, uint64_t round, const double* logw_prev,
                                 const double* log_potential, double* logw_out,
                                 int32_t* bonus_out, float* tv_out,
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
  fill_tau(a, tau);
  a.draft = draft_tokens;
  a.seed = seed;
  a.round = round;
  a.logw_prev = logw_prev;
  a.log_potential = log_potential;
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

