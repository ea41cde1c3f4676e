// Logit n-gram store of stochastic n-gram drafting, on the GPU.
//
// STAND, Methodology item 1: for each observed n-gram the store keeps the
// next-token distribution reduced to its most likely (index, probability)
// pairs; a repeated n-gram merges the stored and the new distribution by a
// weighted average in which an unstored index has probability 0, and the
// result is cut back to the top entries, so each n-gram costs fixed memory.
// Drafting samples those rows (gumbel_topk_sparse, item 2).
//
// Three kernels:
//   observe  one CTA per observed row (persistent): the row's log-sum-exp and
//            each thread's largest logit in one HBM pass; the k-th largest of
//            those maxima is a lower bound T on the row's k-th largest logit,
//            so a second pass (from L2) gathers only entries >= T; their rank
//            order gives the top k, with probabilities exp(z/tau - lse);
//   update   (1) one CTA sorts the batch's (key, position) pairs in shared
//            memory (bitonic) and writes the order and the runs of equal keys
//            to a caller-provided workspace; (2) one warp per distinct key
//            finds or claims its slot (open addressing, linear probing, the
//            warp testing 32 slots per step), then merges the key's
//            observations in batch order: old entries on lanes 0..k-1, the
//            observation on lanes k..2k-1, partners found by __match_any_sync,
//            values (c * old + obs) / (c + 1) in fp64 with one rounding per
//            operation, and the new top k by a bitonic sort across the warp;
//   lookup   one warp per query probes the same way and copies the row out.
//
// Table layout in one caller-owned device buffer (capacity C, a power of two,
// k entries per row):  keys u64 [C] | counts i32 [C] | idx i32 [C][k] |
// prob f32 [C][k].  Key 0 marks an empty slot; a key packs the n-gram exactly:
// n << 60 | t0 << 40 | t1 << 20 | t2 (n <= 3 ids below 2^20).
#include <cuda_runtime.h>

#include "common.cuh"
#include "rowload.cuh"

namespace smcsd {

constexpr int kNgramMaxK = 16;
constexpr int kNgramMaxN = 3;
constexpr uint32_t kNgramMaxId = 1u << 20;
constexpr int kObsThreads = 512;
constexpr int kObsCap = 1024;          // candidates >= T gathered per row
constexpr int kSortThreads = 1024;
constexpr int kUpdateMax = 16384;      // observations per update call (one CTA sorts them)
__device__ constexpr uint64_t kBadKey = ~0ull;  // sorts last; never stored

// ------------------------------------------------------------------ keys and slots
__device__ __forceinline__ uint64_t pack_key(const int32_t* ctx, int n, bool& ok) {
  uint64_t key = (uint64_t)n << 60;
  ok = true;
  for (int i = 0; i < n; ++i) {
    const int32_t t = ctx[i];
    if (t < 0 || (uint32_t)t >= kNgramMaxId) ok = false;
    key |= (uint64_t)((uint32_t)t & (kNgramMaxId - 1)) << (40 - 20 * i);
  }
  return key;
}

// splitmix64's output mix (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", 2014): spreads the packed key over the slots.
__device__ __forceinline__ uint64_t mix64(uint64_t x) {
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  x ^= x >> 31;
  return x;
}

struct TableView {
  uint64_t* keys;
  int32_t* counts;
  int32_t* idx;
  float* prob;
  int64_t cap;  // power of two
  int k;
};

__host__ __device__ inline size_t table_bytes(int64_t cap, int k) {
  return (size_t)cap * (8 + 4 + 8 * (size_t)k);
}

__host__ __device__ inline TableView table_view(void* base, int64_t cap, int k) {
  TableView t;
  char* p = (char*)base;
  t.keys = (uint64_t*)p;
  t.counts = (int32_t*)(p + cap * 8);
  t.idx = (int32_t*)(p + cap * 12);
  t.prob = (float*)(p + cap * 12 + cap * 4 * (int64_t)k);
  t.cap = cap;
  t.k = k;
  return t;
}

// Warp-cooperative probe for `key` (uniform across the warp).  Returns the
// slot holding it, or claims the first empty slot in its probe sequence when
// `insert` is set; -1 when the key is absent (lookup) or the table is full.
// `fresh` tells whether this call claimed the slot.
__device__ __forceinline__ int64_t probe(const TableView& t, uint64_t key, bool insert,
                                         bool& fresh) {
  const int lane = threadIdx.x & 31;
  const uint64_t mask = (uint64_t)t.cap - 1;
  const uint64_t h = mix64(key);
  fresh = false;
  for (int64_t p = 0; p < t.cap;) {
    const uint64_t s = (h + (uint64_t)p + (uint64_t)lane) & mask;
    const bool live = p + lane < t.cap;
    const uint64_t kk = live ? *((volatile uint64_t*)&t.keys[s]) : kBadKey;
    const unsigned hit = __ballot_sync(0xffffffffu, kk == key);
    const unsigned hole = __ballot_sync(0xffffffffu, kk == 0);
    const unsigned first = hit | hole;
    if (!first) {
      p += 32;
      continue;
    }
    const int fl = __ffs(first) - 1;
    if (hit & (1u << fl)) return (int64_t)((h + (uint64_t)p + (uint64_t)fl) & mask);
    if (!insert) return -1;  // an empty slot ends the probe sequence
    uint64_t old = 0;
    if (lane == fl) old = atomicCAS((unsigned long long*)&t.keys[s], 0ull, (unsigned long long)key);
    old = __shfl_sync(0xffffffffu, old, fl);
    if (old == 0 || old == key) {
      fresh = old == 0;
      return (int64_t)((h + (uint64_t)p + (uint64_t)fl) & mask);
    }
    // another key took that slot first: look at this window again
  }
  return -1;
}

// ------------------------------------------------------------------ observe
constexpr int kObsUnroll = 4;  // chunks a thread keeps in flight in the first pass

struct ObsSmem {
  int ncand;
  int flag;
  float red_m[kObsThreads / 32], red_s[kObsThreads / 32];
  float cz[kObsCap];
  int ci[kObsCap];
  float kbuf[(kObsThreads / 32) * kNgramMaxK];
  float sel_z[kNgramMaxK];
  int sel_i[kNgramMaxK];
  float bz[kObsThreads / 32];
  int bi[kObsThreads / 32];
  double lse;
};

__device__ __forceinline__ void better(float& bz, int& bi, float oz, int oi) {
  if (oz > bz || (oz == bz && oi < bi)) {
    bz = oz;
    bi = oi;
  }
}

template <typename TIn>
__global__ void __launch_bounds__(kObsThreads, 2) ngram_observe_kernel(
    const TIn* __restrict__ z, int rows, int V, int64_t ld, const int32_t* __restrict__ row_ids,
    int U, int k, float cT, double tau64, int vec, int32_t* __restrict__ idx_out,
    float* __restrict__ prob_out, uint32_t* dev_err) {
  __shared__ ObsSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
  const int nw = nthr >> 5;
  const int nchunks = (V + 7) / 8;
  const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
  const bool vecok = vec != 0;

  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int r = row_ids ? row_ids[u] : u;
    if (r < 0 || r >= rows) {  // uniform across the CTA
      if (tid < k) {
        idx_out[(int64_t)u * k + tid] = -1;
        prob_out[(int64_t)u * k + tid] = NAN;
      }
      if (tid == 0) raise_err(dev_err, SD_DEV_TOKEN_OOB);
      continue;
    }
    const TIn* row = z + (int64_t)r * ld;
    if (tid == 0) {
      sm.ncand = 0;
      sm.flag = 0;
    }
    __syncthreads();
    // ---------------- pass 1 (HBM): log-sum-exp and per-thread maxima
    float m = -INFINITY, S = 0.f, zmax = -INFINITY;
    bool bad = false;
    for (int c0 = tid; c0 < nchunks; c0 += kObsUnroll * nthr) {
      Raw8<TIn> raw[kObsUnroll];
#pragma unroll
      for (int q = 0; q < kObsUnroll; ++q)
        if (c0 + q * nthr < nchunks) raw[q] = load8_raw<TIn>(row, (c0 + q * nthr) * 8, V, vecok, keep);
#pragma unroll
      for (int q = 0; q < kObsUnroll; ++q) {
        if (c0 + q * nthr >= nchunks) break;
        float zz[8];
        unpack8<TIn>(raw[q], zz);
        float cm = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) cm = fmax_nan(cm, zz[j]);
        bad |= cm != cm;
        zmax = fmaxf(zmax, cm);
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
    bad = bad || m == INFINITY || S != S;
    const float M = warp_max(m);
    float Sw = (m == -INFINITY) ? 0.f : S * ex2((m - M) * cT);
    Sw = warp_sum(Sw);
    if (lane == 0) {
      sm.red_m[warp] = M;
      sm.red_s[warp] = Sw;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&sm.flag, 1);
    __syncthreads();
    if (warp == 0) {
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
    // k distinct entries (the k best per-thread maxima) are >= T, so the row's
    // k-th largest entry is too
    const float T = cta_kth_largest(zmax, k, sm.kbuf);  // (syncs the CTA)
    const bool rowbad = (sm.flag & 1) != 0;

    // ---------------- pass 2 (L2): the entries >= T
    if (!rowbad) {
      for (int c = tid; c < nchunks; c += nthr) {
        float zz[8];
        load8<TIn>(row, c * 8, V, vecok, drop, zz);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (zz[j] >= T && zz[j] > -INFINITY) {
            const int pos = atomicAdd(&sm.ncand, 1);
            if (pos < kObsCap) {
              sm.cz[pos] = zz[j];
              sm.ci[pos] = c * 8 + j;
            }
          }
        }
      }
    }
    __syncthreads();
    const int n = sm.ncand;
    int nsel = 0;
    if (!rowbad && n <= kObsCap) {
      // rank of each candidate in (z descending, index ascending) order
      for (int i = tid; i < n; i += nthr) {
        const float zi = sm.cz[i];
        const int vi = sm.ci[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
          const float zj = sm.cz[j];
          rank += (zj > zi || (zj == zi && sm.ci[j] < vi)) ? 1 : 0;
        }
        if (rank < k) {
          sm.sel_z[rank] = zi;
          sm.sel_i[rank] = vi;
        }
      }
      nsel = n < k ? n : k;
    } else if (!rowbad) {
      // more than kObsCap entries tie at or above T: k rounds of a CTA
      // arg-max over the row, each after the previous winner in that order
      float pz = INFINITY;
      int pi = -1;
      for (int rr = 0; rr < k; ++rr) {
        float bz = -INFINITY;
        int bi = 0x7FFFFFFF;
        for (int v = tid; v < V; v += nthr) {
          const float zv = ld_elem<TIn>(row, v);
          const bool after = zv < pz || (zv == pz && v > pi);
          if (after && zv > -INFINITY) better(bz, bi, zv, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          better(bz, bi, __shfl_xor_sync(0xffffffffu, bz, o), __shfl_xor_sync(0xffffffffu, bi, o));
        if (lane == 0) {
          sm.bz[warp] = bz;
          sm.bi[warp] = bi;
        }
        __syncthreads();
        if (warp == 0) {
          bz = lane < nw ? sm.bz[lane] : -INFINITY;
          bi = lane < nw ? sm.bi[lane] : 0x7FFFFFFF;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
            better(bz, bi, __shfl_xor_sync(0xffffffffu, bz, o), __shfl_xor_sync(0xffffffffu, bi, o));
          if (lane == 0) {
            sm.sel_z[rr] = bz;
            sm.sel_i[rr] = bi;
          }
        }
        __syncthreads();
        pz = sm.sel_z[rr];
        pi = sm.sel_i[rr];
        if (pi == 0x7FFFFFFF) break;  // no finite entry left
        nsel = rr + 1;
      }
    }
    __syncthreads();
    if (tid < k) {
      int32_t vi = -1;
      float p = rowbad ? NAN : 0.f;
      if (tid < nsel) {
        vi = sm.sel_i[tid];
        p = (float)exp((double)sm.sel_z[tid] / tau64 - sm.lse);
      }
      idx_out[(int64_t)u * k + tid] = vi;
      prob_out[(int64_t)u * k + tid] = p;
    }
    if (rowbad && tid == 0) raise_err(dev_err, SD_DEV_NONFINITE);
    __syncthreads();
  }
}

// ------------------------------------------------------------------ update, step 1: order
// Workspace (int32): [0] number of distinct keys D, [1] number of valid
// observations W, [2, 2 + U) observation positions sorted by (key, position),
// [2 + U, 2 + U + D) the start of each run of equal keys.
__host__ __device__ inline size_t workspace_ints(int U) { return (size_t)2 * U + 2; }

__global__ void __launch_bounds__(kSortThreads) ngram_sort_kernel(const int32_t* __restrict__ ctx,
                                                                   int n, int U, int P2,
                                                                   int32_t* __restrict__ ws,
                                                                   uint32_t* dev_err) {
  extern __shared__ __align__(16) unsigned char sort_raw[];
  uint64_t* sk = reinterpret_cast<uint64_t*>(sort_raw);
  int32_t* sv = reinterpret_cast<int32_t*>(sort_raw + (size_t)P2 * 8);
  __shared__ int wtot[kSortThreads / 32];
  __shared__ int s_bad, s_total, s_valid;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
  const int nw = nthr >> 5;
  if (tid == 0) {
    s_bad = 0;
    s_valid = 0;
  }
  __syncthreads();
  for (int i = tid; i < P2; i += nthr) {
    uint64_t key = kBadKey;
    if (i < U) {
      bool ok;
      key = pack_key(ctx + (int64_t)i * n, n, ok);
      if (!ok) {
        key = kBadKey;
        s_bad = 1;
      }
    }
    sk[i] = key;
    sv[i] = i;
  }
  __syncthreads();
  if (tid == 0 && s_bad) raise_err(dev_err, SD_DEV_TOKEN_OOB);
  // bitonic sort, ascending in (key, position)
  for (int size = 2; size <= P2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < (P2 >> 1); t += nthr) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t ka = sk[lo], kb = sk[hi];
        const int va = sv[lo], vb = sv[hi];
        const bool gt = ka > kb || (ka == kb && va > vb);
        if (gt == up) {
          sk[lo] = kb;
          sk[hi] = ka;
          sv[lo] = vb;
          sv[hi] = va;
        }
      }
      __syncthreads();
    }
  }
  // positions, valid count and the runs of equal keys (invalid keys sort last)
  for (int i = tid; i < U; i += nthr) {
    ws[2 + i] = sv[i];
    if (sk[i] != kBadKey && (i + 1 == P2 || sk[i + 1] == kBadKey)) s_valid = i + 1;
  }
  int carry = 0;
  for (int base = 0; base < U; base += nthr) {
    const int i = base + tid;
    const bool head = i < U && sk[i] != kBadKey && (i == 0 || sk[i] != sk[i - 1]);
    const unsigned b = __ballot_sync(0xffffffffu, head);
    if (lane == 0) wtot[warp] = __popc(b);
    __syncthreads();
    if (warp == 0) {
      const int v = lane < nw ? wtot[lane] : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      if (lane < nw) wtot[lane] = inc - v;
      if (lane == 31) s_total = inc;
    }
    __syncthreads();
    if (head) ws[2 + U + carry + wtot[warp] + __popc(b & ((1u << lane) - 1))] = i;
    carry += s_total;
    __syncthreads();
  }
  if (tid == 0) {
    ws[0] = carry;
    ws[1] = s_valid;
  }
}

// ------------------------------------------------------------------ update, step 2: merge
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads) ngram_merge_kernel(
    TableView t, const int32_t* __restrict__ ctx, int n, const int32_t* __restrict__ idx,
    const float* __restrict__ prob, int U, const int32_t* __restrict__ ws, uint32_t* dev_err) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = t.k;
  const int D = min(max(ws[0], 0), U), W = min(max(ws[1], 0), U);
  const int32_t* perm = ws + 2;
  const int32_t* runs = ws + 2 + U;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  const bool is_old = lane < k;
  const bool is_obs = lane >= k && lane < 2 * k;
  const unsigned obs_mask = ((1u << k) - 1u) << k;  // 2k <= 32
  for (int d = blockIdx.x * (blockDim.x >> 5) + warp; d < D; d += nwarps) {
    const int q0 = runs[d];
    const int q1 = d + 1 < D ? runs[d + 1] : W;
    bool ok;
    const uint64_t key = pack_key(ctx + (int64_t)perm[q0] * n, n, ok);
    bool fresh;
    const int64_t slot = probe(t, key, true, fresh);
    if (slot < 0) {
      if (lane == 0) raise_err(dev_err, SD_DEV_TABLE_FULL);
      continue;
    }
    int oi = -1;
    float op = 0.f;
    int c = 0;
    if (!fresh) {
      c = t.counts[slot];
      if (is_old) {
        oi = t.idx[slot * k + lane];
        op = t.prob[slot * k + lane];
      }
    }
    // the next observation's row is loaded while this one merges
    int nxi = -1;
    float nxp = 0.f;
    if (is_obs) {
      const int u0 = perm[q0];
      nxi = idx[(int64_t)u0 * k + (lane - k)];
      nxp = prob[(int64_t)u0 * k + (lane - k)];
    }
    for (int q = q0; q < q1; ++q) {
      const int xi = nxi;
      const float xp = nxp;
      if (is_obs && q + 1 < q1) {
        const int un = perm[q + 1];
        nxi = idx[(int64_t)un * k + (lane - k)];
        nxp = prob[(int64_t)un * k + (lane - k)];
      }
      // one id per lane for matching; empty entries get ids no other lane has
      const int id = is_old ? (oi >= 0 ? oi : -2 - lane) : (is_obs && xi >= 0 ? xi : -2 - lane);
      const unsigned same = __match_any_sync(0xffffffffu, id) & ~(1u << lane);
      const bool bad_obs = is_obs && xi >= 0 && (!(xp >= 0.f && xp < INFINITY) || (same & obs_mask));
      if (__any_sync(0xffffffffu, bad_obs)) {
        if (lane == 0) raise_err(dev_err, SD_DEV_NONFINITE);
        continue;
      }
      // the observed probability of an old entry, read from its partner lane
      const unsigned partner = same & obs_mask;
      const int src = (is_old && partner) ? __ffs(partner) - 1 : lane;
      const float from_obs = __shfl_sync(0xffffffffu, xp, src);
      const double cd = (double)c;
      bool cand = false;
      int vid = -1;
      float val = 0.f;
      if (is_old && oi >= 0) {
        cand = true;
        vid = oi;
        const double num = __dadd_rn(__dmul_rn(cd, (double)op), partner ? (double)from_obs : 0.0);
        val = __double2float_rn(__ddiv_rn(num, cd + 1.0));
      } else if (is_obs && xi >= 0 && !(same & ((1u << k) - 1u))) {
        cand = true;
        vid = xi;
        const double num = __dadd_rn(__dmul_rn(cd, 0.0), (double)xp);
        val = __double2float_rn(__ddiv_rn(num, cd + 1.0));
      }
      // bitonic sort of the warp's lanes in (value descending, index
      // ascending) order, non-candidates last: lane r ends with rank r
      const int ncand = __popc(__ballot_sync(0xffffffffu, cand));
      float sv = cand ? val : -INFINITY;
      int si = cand ? vid : 0x7FFFFFFF;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, sv, stride);
          const int oi2 = __shfl_xor_sync(0xffffffffu, si, stride);
          const bool other_first = ov > sv || (ov == sv && oi2 < si);
          const bool lower = (lane & stride) == 0, up = (lane & size) == 0;
          if (lower == up ? other_first : !other_first && (ov != sv || oi2 != si)) {
            sv = ov;
            si = oi2;
          }
        }
      }
      if (is_old) {
        oi = lane < ncand ? si : -1;
        op = lane < ncand ? sv : 0.f;
      }
      ++c;
    }
    if (is_old) {
      t.idx[slot * k + lane] = oi;
      t.prob[slot * k + lane] = op;
    }
    if (lane == 0) t.counts[slot] = c;
  }
}

// ------------------------------------------------------------------ lookup
__global__ void __launch_bounds__(kMergeThreads) ngram_lookup_kernel(
    TableView t, const int32_t* __restrict__ ctx, int n, int Q, int32_t* __restrict__ idx_out,
    float* __restrict__ prob_out, int32_t* __restrict__ count_out, uint32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (q >= Q) return;
  const int k = t.k;
  bool ok;
  const uint64_t key = pack_key(ctx + q * n, n, ok);
  int64_t slot = -1;
  if (ok) {
    bool fresh;
    slot = probe(t, key, false, fresh);
  } else if (lane == 0) {
    raise_err(dev_err, SD_DEV_TOKEN_OOB);
  }
  if (lane < k) {
    idx_out[q * k + lane] = slot >= 0 ? t.idx[slot * k + lane] : -1;
    prob_out[q * k + lane] = slot >= 0 ? t.prob[slot * k + lane] : 0.f;
  }
  if (lane == 0 && count_out) count_out[q] = slot >= 0 ? t.counts[slot] : 0;
}

}  // namespace smcsd

using namespace smcsd;

namespace {
bool pow2_capacity(int64_t cap) { return cap >= 32 && cap <= ((int64_t)1 << 40) && (cap & (cap - 1)) == 0; }
}  // namespace

extern "C" size_t ngram_table_bytes(int64_t capacity, int k) {
  if (!pow2_capacity(capacity) || k < 1 || k > kNgramMaxK) return 0;
  return table_bytes(capacity, k);
}

extern "C" size_t ngram_workspace_bytes(int U) {
  if (U < 0 || U > kUpdateMax) return 0;
  return workspace_ints(U) * sizeof(int32_t);
}

extern "C" sd_status ngram_table_clear(void* table, int64_t capacity, int k, void* stream) {
  if (!table || !pow2_capacity(capacity) || k < 1 || k > kNgramMaxK) return SD_ERR_INVALID_ARG;
  if (cudaMemsetAsync(table, 0, table_bytes(capacity, k), (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  return SD_OK;
}

extern "C" sd_status ngram_observe_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld,
                                        const int32_t* row_ids, int U, int k, float tau,
                                        int32_t* idx_out, float* prob_out, uint32_t* dev_err,
                                        void* stream) {
  if (rows < 0 || U < 0 || V < 1 || ld < V || k < 1 || k > kNgramMaxK || !(tau > 0.f && tau < INFINITY))
    return SD_ERR_INVALID_ARG;
  if (dt != SD_F32 && dt != SD_BF16) return SD_ERR_INVALID_ARG;
  if (!row_ids && U > rows) return SD_ERR_INVALID_ARG;
  if (U == 0) return SD_OK;
  if (!z || !idx_out || !prob_out) return SD_ERR_INVALID_ARG;
  const int esize = dt == SD_BF16 ? 2 : 4;
  const int vec = ((uintptr_t)z % 16 == 0) && ((ld * esize) % 16 == 0);
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const int grid = U < 2 * nsm ? U : 2 * nsm;  // persistent: two CTAs per SM take the rows in turn
  const float cT = (float)(1.4426950408889634 / (double)tau);
  cudaStream_t s = (cudaStream_t)stream;
  if (dt == SD_BF16)
    ngram_observe_kernel<uint16_t><<<grid, kObsThreads, 0, s>>>(
        (const uint16_t*)z, rows, V, ld, row_ids, U, k, cT, (double)tau, vec, idx_out, prob_out,
        dev_err);
  else
    ngram_observe_kernel<float><<<grid, kObsThreads, 0, s>>>(
        (const float*)z, rows, V, ld, row_ids, U, k, cT, (double)tau, vec, idx_out, prob_out,
        dev_err);
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

extern "C" sd_status ngram_store_update(void* table, int64_t capacity, int k, const int32_t* ctx,
                                        int n, const int32_t* idx, const float* prob, int U,
                                        void* workspace, size_t workspace_bytes,
                                        uint32_t* dev_err, void* stream) {
  if (!table || !pow2_capacity(capacity) || k < 1 || k > kNgramMaxK || n < 1 || n > kNgramMaxN ||
      U < 0)
    return SD_ERR_INVALID_ARG;
  if (U > kUpdateMax) return SD_ERR_UNSUPPORTED;
  if (U == 0) return SD_OK;
  if (!ctx || !idx || !prob || !workspace || workspace_bytes < workspace_ints(U) * sizeof(int32_t) ||
      (uintptr_t)workspace % 4 != 0 || (uintptr_t)table % 16 != 0)
    return SD_ERR_INVALID_ARG;
  int P2 = 1;
  while (P2 < U) P2 <<= 1;
  const size_t smem = (size_t)P2 * 12;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaFuncSetAttribute(ngram_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  int32_t* ws = (int32_t*)workspace;
  ngram_sort_kernel<<<1, kSortThreads, smem, s>>>(ctx, n, U, P2, ws, dev_err);
  // the merge reads what the sort writes: launch it only behind a sort that launched
  if (cudaGetLastError() != cudaSuccess) return SD_ERR_CUDA;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  const int wpb = kMergeThreads / 32;
  int grid = (U + wpb - 1) / wpb;
  if (grid > 8 * nsm) grid = 8 * nsm;
  ngram_merge_kernel<<<grid, kMergeThreads, 0, s>>>(table_view(table, capacity, k), ctx, n, idx,
                                                    prob, U, ws, dev_err);
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

extern "C" sd_status ngram_store_lookup(const void* table, int64_t capacity, int k,
                                        const int32_t* ctx, int n, int Q, int32_t* idx_out,
                                        float* prob_out, int32_t* count_out, uint32_t* dev_err,
                                        void* stream) {
  if (!table || !pow2_capacity(capacity) || k < 1 || k > kNgramMaxK || n < 1 || n > kNgramMaxN ||
      Q < 0 || (uintptr_t)table % 16 != 0)
    return SD_ERR_INVALID_ARG;
  if (Q == 0) return SD_OK;
  if (!ctx || !idx_out || !prob_out) return SD_ERR_INVALID_ARG;
  const int64_t threads = (int64_t)Q * 32;
  const int grid = (int)((threads + kMergeThreads - 1) / kMergeThreads);
  ngram_lookup_kernel<<<grid, kMergeThreads, 0, (cudaStream_t)stream>>>(
      table_view(const_cast<void*>(table), capacity, k), ctx, n, Q, idx_out, prob_out, count_out,
      dev_err);
  return cudaGetLastError() == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

// ------------------------------------------------------------------ update without a workspace
// The workspace of ngram_store_update taken from a fixed device array of this
// library instead of the caller, for callers that must not allocate.  It holds
// room for kUpdateMax observations; the sort writes every entry the merge
// reads, so nothing in it must start at zero.  All calls share the one array:
// calls that overlap on the GPU race on it.
static __device__ __align__(256) int32_t g_ngram_scratch[2 * kUpdateMax + 2];

extern "C" sd_status ngram_store_update_noalloc(void* table, int64_t capacity, int k,
                                                const int32_t* ctx, int n, const int32_t* idx,
                                                const float* prob, int U, uint32_t* dev_err,
                                                void* stream) {
  if (U > kUpdateMax) return SD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_ngram_scratch) != cudaSuccess) {
    cudaGetLastError();
    return SD_ERR_CUDA;
  }
  return ngram_store_update(table, capacity, k, ctx, n, idx, prob, U, scratch,
                            sizeof(g_ngram_scratch), dev_err, stream);
}
