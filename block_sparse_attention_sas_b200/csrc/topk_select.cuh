// Top-K building blocks shared by the gate/Top-K kernels and the fused
// select-and-decode kernel: composite keys (score, then the lower block
// index on ties), block-wide sorts and selections, and the selection of one
// row by a thread-block cluster.
#pragma once

#include <math.h>
#include <stdint.h>

#include "sas_common.cuh"

namespace sas {
namespace {

// Order-preserving map fp32 -> uint32 (larger float -> larger key); -0.0 is
// folded onto +0.0 so that the two compare equal, as fp32 values do.
__device__ __forceinline__ uint32_t fkey(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score a key of fkey() came from (-0.0 comes back as +0.0).
__device__ __forceinline__ float fkey_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ uint64_t ckey(float f, int i) {
  return ((uint64_t)fkey(f) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
}
__device__ __forceinline__ int ckey_index(uint64_t c) {
  return (int)(0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFu));
}

__device__ __forceinline__ float ckey_score(uint64_t c) { return fkey_value((uint32_t)(c >> 32)); }

// Sorts the block's E * blockDim.x keys (a power of two) in descending
// order with a bitonic network; thread t holds the keys at indices
// e * blockDim.x + t in v[e]. Stages whose partners are less than 32 apart
// exchange through warp shuffles (no barrier); the wider ones go through
// sm (E * blockDim.x keys). On return the sorted keys are in sm.
template <int E>
__device__ void block_sort_desc(uint64_t (&v)[E], uint64_t* sm) {
  const int bd = blockDim.x, tid = threadIdx.x, n = E * bd;
  bool in_smem = false;
  for (int k = 2; k <= n; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        if (!in_smem) {
          __syncthreads();  // every thread has read sm into registers
#pragma unroll
          for (int e = 0; e < E; ++e) sm[e * bd + tid] = v[e];
          __syncthreads();
          in_smem = true;
        }
        for (int i = tid; i < n; i += bd) {
          const int p = i ^ j;
          if (p > i) {
            const uint64_t a = sm[i], b = sm[p];
            if (((i & k) == 0) ? (a < b) : (a > b)) {
              sm[i] = b;
              sm[p] = a;
            }
          }
        }
        __syncthreads();
      } else {
        if (in_smem) {
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = sm[e * bd + tid];
          in_smem = false;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = e * bd + tid;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], j);
          // the lower index of a pair keeps the larger key in a descending run
          const bool keep_max = ((i & j) == 0) == ((i & k) == 0);
          v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
      }
    }
  if (!in_smem) {
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) sm[e * bd + tid] = v[e];
  }
  __syncthreads();
}

// Sorts one warp's 32 * EW keys in descending order in registers (lane l
// holds indices e * 32 + l in w[e]); every lane of the warp calls it.
template <int EW>
__device__ __forceinline__ void warp_sort_desc(uint64_t (&w)[EW]) {
  const int lane = threadIdx.x & 31;
  constexpr int n = 32 * EW;
#pragma unroll
  for (int k = 2; k <= n; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int e = 0; e < EW; ++e) {
          const int pe = e ^ (j >> 5);
          if (pe > e) {
            const bool desc = ((e * 32 + lane) & k) == 0;
            const uint64_t a = w[e], b = w[pe];
            if (desc ? (a < b) : (a > b)) {
              w[e] = b;
              w[pe] = a;
            }
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < EW; ++e) {
          const int i = e * 32 + lane;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, w[e], j);
          const bool keep_max = ((i & j) == 0) == ((i & k) == 0);
          w[e] = keep_max ? (w[e] > o ? w[e] : o) : (w[e] < o ? w[e] : o);
        }
      }
    }
}

template <int EW>
__device__ __forceinline__ void warp_sort_cand(const uint64_t* cand, int m, uint64_t* out, int k) {
  const int lane = threadIdx.x & 31;
  uint64_t w[EW];
#pragma unroll
  for (int e = 0; e < EW; ++e) w[e] = e * 32 + lane < m ? cand[e * 32 + lane] : 0ull;
  warp_sort_desc<EW>(w);
#pragma unroll
  for (int e = 0; e < EW; ++e)
    if (e * 32 + lane < k) out[e * 32 + lane] = w[e];
}

constexpr int kBins = 4096;     // histogram over the top 12 bits of a key
constexpr int kCandCap = 256;   // candidates sorted by one warp

struct TopkScratch {
  int hist[kBins];
  uint64_t cand[kCandCap];
  int warp_tot[32];
  int ncand, bin, above;
};

// Leaves the k largest of the block's keys (v[e], E per thread; 0 = empty),
// in descending order, in sm[0, k). Radix filter: a histogram over the top
// 12 bits of the keys finds the bin b holding the k-th largest; every key in
// a bin above b is in, and the rest come from bin b, so the keys in bins >= b
// are the candidates. Up to 256 candidates are sorted by one warp; past that
// (heavy ties) the block sorts all its keys. 1 <= k; every thread calls it.
template <int E>
__device__ void block_topk(uint64_t (&v)[E], int k, TopkScratch& ts, uint64_t* sm) {
  const int tid = threadIdx.x, bd = blockDim.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < kBins; i += bd) ts.hist[i] = 0;
  if (tid == 0) {
    ts.ncand = 0;
    ts.bin = 0;  // always overwritten: the block holds at least k keys
    ts.above = 0;
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (v[e] != 0ull) atomicAdd(&ts.hist[(int)(v[e] >> 52)], 1);
  __syncthreads();
  // Suffix counts: thread t owns bins [t W, t W + W).
  const int W = kBins / bd, b0 = tid * W;
  int local = 0;
  for (int x = 0; x < W; ++x) local += ts.hist[b0 + x];
  int suf = local;  // over this warp's lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += y;
  }
  if (lane == 0) ts.warp_tot[w] = suf;
  __syncthreads();
  int running = suf - local;
  for (int x = w + 1; x < (bd >> 5); ++x) running += ts.warp_tot[x];
  for (int x = W - 1; x >= 0; --x) {
    const int h = ts.hist[b0 + x];
    if (running < k && running + h >= k) {
      ts.bin = b0 + x;
      ts.above = running;
    }
    running += h;
  }
  __syncthreads();
  const int b = ts.bin, m = ts.above + ts.hist[b];
  if (m <= kCandCap) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (v[e] != 0ull && (int)(v[e] >> 52) >= b) ts.cand[atomicAdd(&ts.ncand, 1)] = v[e];
    __syncthreads();
    if (w == 0) {
      if (m <= 32) warp_sort_cand<1>(ts.cand, m, sm, k);
      else if (m <= 64) warp_sort_cand<2>(ts.cand, m, sm, k);
      else if (m <= 128) warp_sort_cand<4>(ts.cand, m, sm, k);
      else warp_sort_cand<8>(ts.cand, m, sm, k);
    }
    __syncthreads();
  } else {
    block_sort_desc<E>(v, sm);
  }
}

// Gate of a score under phi with the row's log-sum-exp (softmax), with the
// fast exponential (about 2 ulp here, far inside the gates' tolerance).
__device__ __forceinline__ float fast_gate(float sc, float lse, int phi) {
  if (phi == SAS_PHI_SIGMOID) return 1.f / (1.f + __expf(-sc));
  if (phi == SAS_PHI_RAW) return __expf(sc);
  return __expf(sc - lse);
}

// ---------------------------------------------------------------------------
// Selection of one row (up to 16 x 512 entries) by a thread-block cluster of
// CS CTAs of NT threads, CTA r holding a chunk of the row, E entries per
// thread, without sorting the row:
//  1. each CTA's (max, min, sum of exp) are read by every CTA of the cluster
//     through distributed shared memory (one round trip, lane x reading rank
//     x); every CTA forms the row's max M and LSE alike;
//  2. each CTA histograms its chunk over 64 buckets of (M - s) in steps of
//     1/8, or of (M - min) / 63 when the row's scores span less than 63/8
//     (bucket 63: everything further down, never counted: its count is the
//     rest of the row) and adds the histogram into every CTA's copy of
//     the row's histogram (remote reductions, no round trip); after a
//     cluster barrier each CTA finds b*, the bucket holding the k-th largest
//     score, in its own copy. When that is bucket 63, a second histogram
//     spreads [min, M - 63/8] over 64 buckets the same way;
//  3. every score in a bucket up to b* is a candidate -- a superset of the
//     top k, usually a few more than k. Each warp reserves room in rank 0's
//     list with one remote atomic and stores its candidates there; rank 0
//     then places each by its rank among them under the composite order,
//     which is its rank in the row.
// More than 1024 candidates (mass ties, known from the histogram) switch the
// cluster to an exact path: each CTA selects its chunk's best k and stores
// them in rank 0's list at rank * k.
// ---------------------------------------------------------------------------
constexpr int kSelMaxCta = 16;   // rows up to 16 chunks
constexpr int kSelCand = 1024;   // candidates rank 0 places by rank
constexpr int kSelNB = 64;       // buckets per histogram level
constexpr float kSelStep = 8.f;  // level-1 buckets per unit of score below the max (at least)

struct SelShared {
  float part[3];                     // this chunk's max, min, sum of exp (relative to its max)
  int hist[kSelNB];                  // this chunk's histogram
  unsigned int row_hist[2][kSelNB];  // the row's, levels 1 and 2 (the cluster adds into it)
  unsigned int nlist;                // rank 0: keys in its list
  uint64_t best[512];                // the exact path: this chunk's best, sorted
  float red[2][8];
  int wsum[8];
  float M, Mn, lse;
  int bstar, before, upto;
  TopkScratch ts;  // the exact path
};

// The cluster barrier of a selection (a CTA barrier for a one-CTA row).
__device__ __forceinline__ void sel_sync(int CS) {
  if (CS > 1)
    cluster_sync_all();
  else
    __syncthreads();
}

// Finds, in the row histogram h, the bucket holding the target-th entry in
// bucket order (warp 0; lane l sums buckets 2l and 2l + 1). `rest` >= 0
// gives the last bucket the count `rest` minus the other buckets' total (a
// bucket no CTA counts). Returns the bucket; *before / *upto = entries in
// the buckets before it / up to and including it. Every thread calls it;
// the result is the same in every CTA.
__device__ int sel_find_bucket(const unsigned int* h, int target, int rest, SelShared& sh,
                               int* before, int* upto) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int c0 = (int)h[2 * lane];
    int c1 = (rest >= 0 && lane == 31) ? 0 : (int)h[2 * lane + 1];
    int inc = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const int tot = __shfl_sync(0xffffffffu, inc, 31);
    if (rest >= 0 && lane == 31) {  // the uncounted bucket takes the rest
      c1 = rest - tot;
      inc = rest;
    }
    const int ex = inc - c0 - c1;  // entries before bucket 2 lane
    if (ex < target && ex + c0 >= target) {
      sh.bstar = 2 * lane;
      sh.before = ex;
      sh.upto = ex + c0;
    } else if (ex + c0 < target && inc >= target) {
      sh.bstar = 2 * lane + 1;
      sh.before = ex + c0;
      sh.upto = inc;
    }
  }
  __syncthreads();
  *before = sh.before;
  *upto = sh.upto;
  return sh.bstar;  // rewritten only after a later barrier
}

// Adds this CTA's histogram (sh.hist) into the row histogram `dst` of every
// CTA of the cluster (thread t: bucket t % 64 into ranks t / 64, t / 64 +
// NT / 64, ...), then clears sh.hist.
template <int NT>
__device__ __forceinline__ void sel_push_hist(SelShared& sh, unsigned int* dst, int CS) {
  const int tid = threadIdx.x, bkt = tid & (kSelNB - 1);
  __syncthreads();  // the local histogram is complete
  const unsigned int v = (unsigned int)sh.hist[bkt];
  if (v)
    for (int x = tid / kSelNB; x < CS; x += NT / kSelNB)
      dsmem_red_add_u32(dsmem_addr(&dst[bkt], (uint32_t)x), v);
  __syncthreads();  // read before cleared
  if (tid < kSelNB) sh.hist[tid] = 0;
}

// The selection of one row by the cluster. Thread tid of rank r holds
// f[e] = row[lo + tid + NT e] where ok[e] (entries of its chunk [lo, lo +
// chunk) below n); n = the row's valid entries, 1 <= kk = min(K, n) <= 256.
// Every thread of every CTA calls it. On return every CTA has passed the
// last cluster barrier of the selection, sh.M / sh.lse hold the row's max
// and log-sum-exp, and rank 0's `list` holds the returned number of keys
// (0 = an empty slot) whose kk largest are the row's Top-K. `list` needs
// max(1024, CS * kk) keys at rank 0.
template <int NT, int E>
__device__ int cluster_select(const float (&f)[E], const bool (&ok)[E], int lo, int chunk, int n,
                              int kk, int CS, SelShared& sh, uint64_t* list) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (ok[e]) {
      mx = fmaxf(mx, f[e]);
      mn = fminf(mn, f[e]);
    }
  mx = warp_max(mx);
  mn = -warp_max(-mn);
  if (lane == 0) {
    sh.red[0][warp] = mx;
    sh.red[1][warp] = mn;
  }
  if (tid < kSelNB) {
    sh.hist[tid] = 0;
    sh.row_hist[0][tid] = 0u;
    sh.row_hist[1][tid] = 0u;
  }
  if (tid == 0) sh.nlist = 0u;
  __syncthreads();
  float cm = -INFINITY, cmn = INFINITY;
#pragma unroll
  for (int x = 0; x < NW; ++x) {
    cm = fmaxf(cm, sh.red[0][x]);
    cmn = fminf(cmn, sh.red[1][x]);
  }
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (ok[e]) sum += __expf(f[e] - cm);
  sum = warp_sum(sum);
  if (lane == 0) sh.wsum[warp] = __float_as_int(sum);
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
#pragma unroll
    for (int x = 0; x < NW; ++x) t += __int_as_float(sh.wsum[x]);
    sh.part[0] = cm;
    sh.part[1] = cmn;
    sh.part[2] = t;
  }
  // (1) the partials are written and every CTA's row histograms and list
  // counter are cleared before anyone adds into them
  sel_sync(CS);

  if (warp == 0) {
    float pm = -INFINITY, pmn = INFINITY, ps = 0.f;
    if (lane < CS) {
      pm = dsmem_ld_f32(dsmem_addr(&sh.part[0], (uint32_t)lane));
      pmn = dsmem_ld_f32(dsmem_addr(&sh.part[1], (uint32_t)lane));
      ps = dsmem_ld_f32(dsmem_addr(&sh.part[2], (uint32_t)lane));
    }
    const float M = warp_max(pm);
    const float Mn = -warp_max(-pmn);
    const float S = warp_sum(ps > 0.f ? ps * __expf(pm - M) : 0.f);
    if (lane == 0) {
      sh.M = M;
      sh.Mn = Mn;
      sh.lse = M + __logf(S);
    }
  }
  __syncthreads();
  const float M = sh.M, Mn = sh.Mn;

  // ---- level 1: 1/8-wide buckets below the max (finer when the row's
  // scores span less: 63 buckets then cover the span); the last is never
  // counted. The width comes from M and Mn, so it is the same in every CTA.
  const float span = M - Mn;
  const float step = (span > 0.f && span < (float)(kSelNB - 1) / kSelStep)
                         ? (float)(kSelNB - 1) / span
                         : kSelStep;
  auto b1_of = [&](float x) -> int {
    return (int)fminf((M - x) * step, (float)(kSelNB - 1));
  };
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (ok[e]) {
      const int bb = b1_of(f[e]);
      if (bb < kSelNB - 1) atomicAdd(&sh.hist[bb], 1);
    }
  sel_push_hist<NT>(sh, sh.row_hist[0], CS);
  sel_sync(CS);  // (2) the row histogram is complete in every CTA
  int before, upto;
  const int b1 = sel_find_bucket(sh.row_hist[0], kk, n, sh, &before, &upto);

  // ---- level 2 (rare: the k-th score lies 63/8 or more below the max):
  // 64 buckets spread over [Mn, M - 63/8]
  const float top2 = M - (float)(kSelNB - 1) / step;
  const float inv2 = top2 > Mn ? (float)(kSelNB - 1) / (top2 - Mn) : 0.f;
  auto b2_of = [&](float x) -> int {
    return (int)fminf(fmaxf((top2 - x) * inv2, 0.f), (float)(kSelNB - 1));
  };
  int b2 = kSelNB - 1;
  int ncand = upto;
  if (b1 == kSelNB - 1) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (ok[e] && b1_of(f[e]) == kSelNB - 1) atomicAdd(&sh.hist[b2_of(f[e])], 1);
    sel_push_hist<NT>(sh, sh.row_hist[1], CS);
    sel_sync(CS);  // (2b)
    int before2, upto2;
    b2 = sel_find_bucket(sh.row_hist[1], kk - before, -1, sh, &before2, &upto2);
    ncand = before + upto2;
  }

  const uint32_t list0 = dsmem_addr(list, 0u), nlist0 = dsmem_addr(&sh.nlist, 0u);
  const bool exact = ncand > kSelCand;
  if (!exact) {
    // ---- this chunk's candidates into rank 0's list
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int bb = ok[e] ? b1_of(f[e]) : kSelNB;
      const bool take = bb < b1 || (bb == b1 && (b1 < kSelNB - 1 || b2_of(f[e]) <= b2));
      const uint32_t mask = __ballot_sync(0xffffffffu, take);
      if (mask == 0u) continue;
      uint32_t slot = 0u;
      if (lane == 0) slot = dsmem_atom_add_u32(nlist0, (uint32_t)__popc(mask));
      slot = __shfl_sync(0xffffffffu, slot, 0) + (uint32_t)__popc(mask & ((1u << lane) - 1u));
      if (take) dsmem_st_u64(list0 + 8u * slot, ckey(f[e], lo + tid + NT * e));
    }
  } else {
    // ---- exact path (mass ties): each chunk's best kk into rank 0's list,
    // at rank * kk (empty slots 0)
    const int len = max(0, min(n - lo, chunk));
    const int kc = min(kk, len);
    uint64_t v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = ok[e] ? ckey(f[e], lo + tid + NT * e) : 0ull;
    if (kc > 0) block_topk<E>(v, kc, sh.ts, sh.best);  // the best kc, sorted, in sh.best
    for (int p = tid; p < kk; p += NT)
      dsmem_st_u64(list0 + 8u * (uint32_t)(rank * kk + p), p < kc ? sh.best[p] : 0ull);
  }
  sel_sync(CS);  // (3) rank 0 holds the list; the selection touches no other CTA's memory after this
  return rank == 0 ? (exact ? CS * kk : (int)sh.nlist) : 0;
}

// Places keys[0, m) by rank (keys equal to 0 are empty slots): emit(rank,
// key) for the kk best. Short lists: a group of tpc threads per key splits
// the comparisons; long lists: four keys per thread, one pass over the list.
template <int NT, typename Emit>
__device__ __forceinline__ void place_by_rank(const uint64_t* keys, int m, int kk, Emit&& emit) {
  const int tid = threadIdx.x;
  if (m <= NT) {
    int tpc = 1;
    while (tpc < 8 && 2 * tpc * m <= NT) tpc *= 2;
    const int p = tid / tpc, part = tid % tpc;
    const uint64_t mine = p < m ? keys[p] : 0ull;
    int rk = 0;
    // Eight loads in flight, then eight comparisons (0 past the list: never
    // above a key that is placed).
    for (int q0 = part; q0 < m; q0 += 8 * tpc) {
      uint64_t y[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int q = q0 + u * tpc;
        y[u] = q < m ? keys[q] : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) rk += y[u] > mine;
    }
    for (int o = 1; o < tpc; o <<= 1) rk += __shfl_xor_sync(0xffffffffu, rk, o);
    if (part == 0 && mine != 0ull && rk < kk) emit(rk, mine);
    return;
  }
  for (int p0 = tid; p0 < m; p0 += 4 * NT) {
    uint64_t mine[4];
    int rk[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u * NT;
      mine[u] = p < m ? keys[p] : 0ull;
      rk[u] = 0;
    }
    for (int q = 0; q < m; ++q) {
      const uint64_t y = keys[q];
#pragma unroll
      for (int u = 0; u < 4; ++u) rk[u] += y > mine[u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (mine[u] != 0ull && rk[u] < kk) emit(rk[u], mine[u]);
  }
}

}  // namespace
}  // namespace sas
