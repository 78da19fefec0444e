// Gate softmax (Eq. 6) and deterministic Top-K block selection (Eq. 3).
//
// Per row of scores: log g_m = s_m - LSE(s over the valid history), gates
// g_m = exp(log g_m); then the k = min(K, n) largest scores, ordered by
// descending score with ties to the lower block index, padded with -1
// (picx.dev SAS summary, Theoretical Foundation Eq. 3 and Gradient Analysis
// Eq. 6; reproduction README, Core equations).
//
// Selection without sorting the row: scores map to order-preserving 32-bit
// keys; a most-significant-digit radix select (four passes over 8-bit
// digits, each a 256-bin histogram of the keys that share the prefix found
// so far) finds tau, the k-th largest key. Every key > tau is taken, plus the
// lowest-indexed (k - #{key > tau}) keys equal to tau, found by an ordered
// ballot scan. The k survivors are placed by rank (a survivor's rank is the
// number of survivors that beat it), which sorts them exactly.
//
// Two layouts of the same algorithm: one warp per row for short rows (the
// training case, one row per query block), one CTA per row for long rows
// (decode over thousands of history blocks).
//
// Gate activations (phi of Eq. 4): softmax over the valid history (Eq. 6,
// the method's own), and the two ablation variants the evolve.pub review
// (Summary) names: an elementwise sigmoid g = 1 / (1 + e^-s) and raw logits
// (log g = s, stored as g = e^s). Top-K is over the scores for every phi:
// each is increasing, so the selection is the same.
#include <mutex>

#include "sas_common.cuh"
#include "sas_internal.h"
#include "topk_select.cuh"

namespace sas {
namespace {

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Adds one per element to hist[bin] for the lanes with `valid`; lanes that
// hold the same bin are combined first, so each bin takes one atomic per warp.
__device__ __forceinline__ void warp_hist_add(int* hist, uint32_t bin, bool valid) {
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t key = valid ? bin : (0x10000u + lane);
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  if (valid && (__ffs(peers) - 1) == (int)lane) atomicAdd(&hist[bin], __popc(peers));
}

// Given a 256-bin histogram (the warp reads it), finds the digit holding the
// k-th largest element: returns the digit and sets `above` to the count of
// elements in bins above it. Every lane returns the same values.
__device__ __forceinline__ uint32_t warp_pick_digit(const int* hist, int k, int& above) {
  const int lane = threadIdx.x & 31;
  int h[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = hist[lane * 8 + i];
    sum += h[i];
  }
  int suf = sum;  // inclusive suffix sum over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, suf >= k);
  const int L = 31 - __clz(hit);  // highest lane whose suffix reaches k
  int ab = suf - sum, dig = 0;    // elements in lanes above L
  if (lane == L) {
    for (int i = 7; i >= 0; --i) {
      if (ab + h[i] >= k) {
        dig = L * 8 + i;
        break;
      }
      ab += h[i];
    }
  }
  above = __shfl_sync(0xffffffffu, ab, L);
  return (uint32_t)__shfl_sync(0xffffffffu, dig, L);
}

// Gate of one valid entry from its score (lse: the row's log-sum-exp, used by
// the softmax only).
__device__ __forceinline__ float gate_of(float sc, float lse, int phi) {
  if (phi == SAS_PHI_SIGMOID) return 1.f / (1.f + expf(-sc));
  if (phi == SAS_PHI_RAW) return expf(sc);
  return expf(sc - lse);
}

constexpr int kWarpRowsPerCta = 8;
constexpr int kWarpCap = 512;   // longest row handled by one warp
constexpr int kMaxK = 256;
constexpr int kArgmaxMaxK = 64;  // largest K taken by rounds of warp argmax

// Small K: the k largest of a row of n <= 32 E entries by k rounds of warp
// argmax. Each lane holds E composite keys, the score's order-preserving key
// above the complement of the index, so the larger composite is the higher
// score and, among equal scores, the lower index; no two entries share one,
// and round t yields the entry of rank t. Empty slots hold 0, below every
// composite of a valid entry (whose low word is at least ~511).
template <int E>
__device__ __forceinline__ void warp_argmax_topk(const float* v, int n, int k, int lane,
                                                 int32_t* out) {
  uint64_t key[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane + 32 * e;
    key[e] = i < n ? ((uint64_t)fkey(v[i]) << 32) | (uint64_t)(~(uint32_t)i) : 0ull;
  }
  for (int t = 0; t < k; ++t) {
    uint64_t m = key[0];
#pragma unroll
    for (int e = 1; e < E; ++e) m = key[e] > m ? key[e] : m;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, m, off);
      m = o > m ? o : m;
    }
    if (lane == 0) out[t] = (int32_t)(~(uint32_t)m);
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (key[e] == m) key[e] = 0ull;
  }
}

// ---------------------------------------------------------------------------
// One warp per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * kWarpRowsPerCta)
gate_topk_warp_kernel(const float* __restrict__ scores, int total_rows, int rows, int C,
                      int causal, int K, int phi, float* __restrict__ gates,
                      int32_t* __restrict__ idx) {
  __shared__ float s_val[kWarpRowsPerCta][kWarpCap];
  __shared__ uint32_t s_selkey[kWarpRowsPerCta][kMaxK];
  __shared__ int32_t s_selidx[kWarpRowsPerCta][kMaxK];
  __shared__ int s_hist[kWarpRowsPerCta][256];

  grid_launch_dependents();  // a dependent decode may start its prologue
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarpRowsPerCta + w;
  if (row >= total_rows) return;
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  const float* s = scores + row * (long long)C;
  float* g = gates + row * (long long)C;
  int32_t* out = idx + row * (long long)K;
  float* v = s_val[w];

  // ---- gates: max, sum, exp (Eq. 6)
  float mx = -INFINITY;
  for (int i = lane; i < n; i += 32) {
    const float f = s[i];
    v[i] = f;
    mx = fmaxf(mx, f);
  }
  mx = warp_max(mx);
  float sum = 0.f;
  for (int i = lane; i < n; i += 32) sum += expf(v[i] - mx);
  sum = warp_sum(sum);
  const float lse = mx + logf(sum);
  for (int i = lane; i < C; i += 32) g[i] = (i < n) ? gate_of(v[i], lse, phi) : 0.f;

  const int k = min(K, n);
  if (k > 0 && K <= kArgmaxMaxK) {
    __syncwarp();  // the row's scores in v are visible to every lane
    if (n <= 256)
      warp_argmax_topk<8>(v, n, k, lane, out);
    else
      warp_argmax_topk<16>(v, n, k, lane, out);
  } else if (k > 0) {
    // ---- tau = k-th largest key: radix select, four 8-bit digits
    int* hist = s_hist[w];
    uint32_t tau = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0;
      __syncwarp();
      for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const uint32_t key = (i < n) ? fkey(v[i]) : 0u;
        warp_hist_add(hist, (key >> shift) & 255u, i < n && (key & mask) == tau);
      }
      __syncwarp();
      int above;
      const uint32_t dig = warp_pick_digit(hist, krem, above);
      krem -= above;
      tau |= dig << shift;
      mask |= 255u << shift;
      __syncwarp();
    }
    const int need_eq = krem;

    // ---- ordered compaction of the survivors (index order)
    int run_eq = 0, run_sel = 0;
    const uint32_t lt = lanemask_lt();
    for (int base = 0; base < n && run_sel < k; base += 32) {
      const int i = base + lane;
      const uint32_t key = (i < n) ? fkey(v[i]) : 0u;
      const bool is_gt = (i < n) && key > tau;
      const bool is_eq = (i < n) && key == tau;
      const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = is_gt || (is_eq && run_eq + __popc(eqm & lt) < need_eq);
      const uint32_t selm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int p = run_sel + __popc(selm & lt);
        s_selkey[w][p] = key;
        s_selidx[w][p] = i;
      }
      run_eq += __popc(eqm);
      run_sel += __popc(selm);
    }
    __syncwarp();
    // ---- place by rank: descending key, then ascending index
    for (int p = lane; p < k; p += 32) {
      const uint32_t kp = s_selkey[w][p];
      int rank = 0;
      for (int q = 0; q < k; ++q) {
        const uint32_t kq = s_selkey[w][q];
        rank += (kq > kp) || (kq == kp && q < p);
      }
      out[rank] = s_selidx[w][p];
    }
  }
  for (int p = k + lane; p < K; p += 32) out[p] = -1;
}

// ---------------------------------------------------------------------------
// Long rows: a block per chunk of the row sorts the chunk, then a block per
// row merges the chunks' candidates.
// ---------------------------------------------------------------------------
// A row's k largest scores are among the k largest of each chunk, so each
// chunk passes on its top min(K, chunk) entries; the merge picks the row's k
// from those. Entries are compared by a composite 64-bit key: the score's
// order-preserving key above the complement of the block index. Larger
// composites are higher scores and, among equal scores, lower indices, and
// no two entries of a row share one, so a descending sort is the Top-K order
// with its tie rule. The gate softmax combines the chunks' (max, sum of exp)
// pairs. The chunk results travel through the row's own gates, which the
// merge reads first and then overwrites with the final gates (no workspace).
constexpr int kMaxChunk = 8192;       // longest chunk (64 KB of keys)
constexpr int kMaxCandidates = 8192;  // chunks x per-chunk candidates

// Block reductions for any multiple of 32 threads up to 1024 (red: 32 floats).
__device__ __forceinline__ float block_max(float x, float* red) {
  x = warp_max(x);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  return warp_max(lane < (int)(blockDim.x >> 5) ? red[lane] : -INFINITY);
}
__device__ __forceinline__ float block_sum(float x, float* red) {
  x = warp_sum(x);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  return warp_sum(lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f);
}

// Static shared memory of the chunk and merge kernels (scratch + reduction),
// counted against the 48 KB a launch gets without opting in.
constexpr size_t kStaticSmem = sizeof(TopkScratch) + 32 * sizeof(float) + 64;

// Writes g = exp(s - lse) for i < n and 0 past n, over [0, C) of one row
// (float4 accesses when both rows are 16-byte aligned).
__device__ __forceinline__ void write_gates(const float* srow, float* grow, int C, int n, float lse,
                                            int phi) {
  const int tid = threadIdx.x, bd = blockDim.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(srow) | reinterpret_cast<uintptr_t>(grow)) & 15) == 0;
  int i0 = 0;
  if (vec) {
    const int C4 = C >> 2;
    for (int q = tid; q < C4; q += bd) {
      const float4 x = reinterpret_cast<const float4*>(srow)[q];
      const int i = q * 4;
      float4 g;
      g.x = i < n ? gate_of(x.x, lse, phi) : 0.f;
      g.y = i + 1 < n ? gate_of(x.y, lse, phi) : 0.f;
      g.z = i + 2 < n ? gate_of(x.z, lse, phi) : 0.f;
      g.w = i + 3 < n ? gate_of(x.w, lse, phi) : 0.f;
      reinterpret_cast<float4*>(grow)[q] = g;
    }
    i0 = C4 * 4;
  }
  for (int i = i0 + tid; i < C; i += bd) grow[i] = i < n ? gate_of(srow[i], lse, phi) : 0.f;
}

// One block per (row, chunk of Lc = E * blockDim.x entries). FINAL (the row
// is one chunk): writes the row's idx and gates. Otherwise writes the
// chunk's max and sum of exp to gates[2c], gates[2c + 1] of its row, and its
// kc best composites, as pairs of 32-bit words, after the 2 * chunks floats
// of those pairs.
template <bool FINAL, int E>
__global__ void __launch_bounds__(1024)
gate_topk_chunk_kernel(const float* __restrict__ scores, int rows, int C, int causal, int K,
                       int chunks, int kc, int phi, float* __restrict__ gates,
                       int32_t* __restrict__ idx) {
  extern __shared__ uint64_t s_key[];  // E * blockDim.x keys
  __shared__ float red[32];
  __shared__ TopkScratch ts;
  const int tid = threadIdx.x, bd = blockDim.x, Lc = E * bd;
  const long long row = blockIdx.x / chunks;
  const int c = (int)(blockIdx.x % chunks);
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  const int lo = c * Lc, len = max(0, min(n - lo, Lc));
  const float* srow = scores + row * (long long)C;

  uint64_t v[E];
  float f[E];
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = e * bd + tid;
    const bool ok = i < len;
    f[e] = ok ? srow[lo + i] : -INFINITY;
    v[e] = ok ? ckey(f[e], lo + i) : 0ull;  // 0 is below every entry's composite
    mx = fmaxf(mx, f[e]);
  }
  mx = block_max(mx, red);
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e * bd + tid < len) sum += expf(f[e] - mx);
  sum = block_sum(sum, red);
  // The chunk's best min(K or kc, len) keys, sorted, in s_key.
  const int kk = min(FINAL ? K : kc, len);
  if (kk > 0) block_topk<E>(v, kk, ts, s_key);

  float* grow = gates + row * (long long)C;
  if (FINAL) {
    int32_t* out = idx + row * (long long)K;
    for (int p = tid; p < K; p += bd) out[p] = p < kk ? ckey_index(s_key[p]) : -1;
    write_gates(srow, grow, C, n, mx + logf(sum), phi);
  } else {
    if (tid == 0) {
      grow[2 * c] = mx;
      grow[2 * c + 1] = sum;
    }
    uint32_t* cand = reinterpret_cast<uint32_t*>(grow + 2 * chunks) + 2LL * c * kc;
    for (int p = tid; p < kc; p += bd) {
      const uint64_t key = p < kk ? s_key[p] : 0ull;
      cand[2 * p] = (uint32_t)(key & 0xFFFFFFFFu);
      cand[2 * p + 1] = (uint32_t)(key >> 32);
    }
  }
}

// One block per row: combines the chunks' softmax partials into the row's
// LSE, sorts the chunks' candidates (E * blockDim.x >= chunks * kc keys), and
// writes the row's idx and gates.
template <int E>
__global__ void __launch_bounds__(1024)
gate_topk_merge_kernel(const float* __restrict__ scores, int rows, int C, int causal, int K,
                       int chunks, int kc, int phi, float* __restrict__ gates,
                       int32_t* __restrict__ idx) {
  extern __shared__ uint64_t s_key[];  // E * blockDim.x keys
  __shared__ float red[32];
  __shared__ TopkScratch ts;
  const long long row = blockIdx.x;
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  float* grow = gates + row * (long long)C;
  const uint32_t* cand = reinterpret_cast<const uint32_t*>(grow + 2 * chunks);
  const int tid = threadIdx.x, bd = blockDim.x, nc = chunks * kc;

  uint64_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = e * bd + tid;
    v[e] = i < nc ? (((uint64_t)cand[2 * i + 1] << 32) | cand[2 * i]) : 0ull;
  }
  float m = -INFINITY;
  for (int c = tid; c < chunks; c += bd) m = fmaxf(m, grow[2 * c]);
  m = block_max(m, red);
  float acc = 0.f;
  for (int c = tid; c < chunks; c += bd) {
    const float sc = grow[2 * c + 1];
    if (sc > 0.f) acc += sc * expf(grow[2 * c] - m);  // empty chunks hold (-inf, 0)
  }
  acc = block_sum(acc, red);  // its barriers also order every scratch read before the writes below
  const float lse = m + logf(acc);
  const int k = min(K, n);
  if (k > 0) block_topk<E>(v, k, ts, s_key);
  int32_t* out = idx + row * (long long)K;
  for (int p = tid; p < K; p += bd) out[p] = p < k ? ckey_index(s_key[p]) : -1;
  write_gates(scores + row * (long long)C, grow, C, n, lse, phi);
}

// ---------------------------------------------------------------------------
// Decode-sized rows (513 .. 8192 entries): a thread-block cluster of CS CTAs
// per row, CTA r holding the 512 entries [512 r, 512 r + 512), two per
// thread, selects the row with cluster_select (bucket histograms exchanged
// over distributed shared memory; candidates placed by rank at rank 0). The
// gates are written last, so that no cluster barrier waits for those stores.
// ---------------------------------------------------------------------------
constexpr int kCbThreads = 256;
constexpr int kCbChunk = 512;  // entries per CTA

__global__ void __launch_bounds__(kCbThreads)
gate_topk_cbucket_kernel(const float* __restrict__ scores, int rows, int C, int causal, int K,
                         int CS, int phi, float* __restrict__ gates, int32_t* __restrict__ idx) {
  // rank 0's list: the candidates, or CS chunks' best kk on the exact path
  extern __shared__ uint64_t s_list[];
  __shared__ SelShared sh;
  grid_launch_dependents();  // a dependent decode may start its prologue
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank();
  const long long row = blockIdx.x / CS;
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  const int kk = min(K, n);  // the same in every CTA of the cluster
  const int lo = (int)rank * kCbChunk;
  const float* srow = scores + row * (long long)C;
  float* grow = gates + row * (long long)C;
  int32_t* out = idx + row * (long long)K;
  if (kk == 0) {  // an empty history (the whole cluster): gates 0, no selection
    for (int e = 0; e < 2; ++e) {
      const int i = lo + tid + kCbThreads * e;
      if (i < C) grow[i] = 0.f;
    }
    if (rank == 0)
      for (int p = tid; p < K; p += kCbThreads) out[p] = -1;
    return;
  }
  float f[2];
  bool ok[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int i = lo + tid + kCbThreads * e;
    ok[e] = i < n;
    f[e] = ok[e] ? srow[i] : -INFINITY;
  }
  const int m = cluster_select<kCbThreads, 2>(f, ok, lo, kCbChunk, n, kk, CS, sh, s_list);
  if (rank == 0) {
    place_by_rank<kCbThreads>(s_list, m, kk,
                              [&](int rk, uint64_t key) { out[rk] = ckey_index(key); });
    for (int p = kk + tid; p < K; p += kCbThreads) out[p] = -1;
  }
  // The gates go last, so that no cluster barrier waits for these stores.
  const float lse = sh.lse;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int i = lo + tid + kCbThreads * e;
    if (i < C) grow[i] = i < n ? fast_gate(f[e], lse, phi) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Long rows in one launch: a thread-block cluster of CS CTAs per row, CTA r
// taking the chunk [r Lc, (r + 1) Lc). Each chunk forms its softmax partial
// (max, sum of exp) and its best min(K, Lc) composites in shared memory; after
// a cluster barrier every CTA reads the CS partials through distributed shared
// memory (in rank order, so all form the same LSE) and writes its chunk's
// gates from the scores it still holds, while rank 0 gathers the candidates
// and selects the row's Top-K. A second barrier keeps every chunk's shared
// memory alive until those reads are done. No workspace, no second launch.
// ---------------------------------------------------------------------------
constexpr int kClThreads = 512;
constexpr int kClMaxCta = 16;

template <int EM>
__device__ void cluster_merge_topk(const uint64_t* cand_local, const int* cnt_local, int CS, int kc,
                                   int k, TopkScratch& ts, uint64_t* sm, int32_t* out, int K) {
  const int tid = threadIdx.x, bd = blockDim.x;
  uint64_t v[EM];
#pragma unroll
  for (int e = 0; e < EM; ++e) {
    const int i = e * bd + tid;
    const int r = i / kc, p = i - r * kc;
    uint64_t key = 0ull;
    if (r < CS) {
      const int cnt = (int)dsmem_ld_u32(dsmem_addr(cnt_local, (uint32_t)r));
      if (p < cnt) key = dsmem_ld_u64(dsmem_addr(cand_local + p, (uint32_t)r));
    }
    v[e] = key;
  }
  // Every CTA of the cluster may now leave once it is done with its gates:
  // this barrier pairs with the one the other ranks pass after their reads.
  cluster_sync_all();
  block_topk<EM>(v, k, ts, sm);
  for (int p = tid; p < K; p += bd) out[p] = p < k ? ckey_index(sm[p]) : -1;
}

template <int E>
__global__ void __launch_bounds__(kClThreads)
gate_topk_cluster_kernel(const float* __restrict__ scores, int rows, int C, int causal, int K,
                         int CS, int phi, float* __restrict__ gates, int32_t* __restrict__ idx) {
  extern __shared__ uint64_t s_key[];  // max(E, merge width) * blockDim.x keys
  __shared__ float red[32];
  __shared__ TopkScratch ts;
  __shared__ float s_part[2];  // this chunk's (max, sum of exp)
  __shared__ int s_cnt;        // its candidate count
  __shared__ float s_lse;
  grid_launch_dependents();  // a dependent decode may start its prologue
  const int tid = threadIdx.x, bd = blockDim.x, Lc = E * bd;
  const uint32_t rank = cluster_rank();
  const long long row = blockIdx.x / CS;
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  const int lo = (int)rank * Lc, len = max(0, min(n - lo, Lc));
  const int kc = min(K, Lc);
  const float* srow = scores + row * (long long)C;

  uint64_t v[E];
  float f[E];
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = e * bd + tid;
    const bool ok = i < len;
    f[e] = ok ? srow[lo + i] : -INFINITY;
    v[e] = ok ? ckey(f[e], lo + i) : 0ull;
    mx = fmaxf(mx, f[e]);
  }
  mx = block_max(mx, red);
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e * bd + tid < len) sum += expf(f[e] - mx);
  sum = block_sum(sum, red);
  const int kk = min(kc, len);
  if (kk > 0) block_topk<E>(v, kk, ts, s_key);
  if (tid == 0) {
    s_part[0] = mx;
    s_part[1] = sum;
    s_cnt = kk;
  }
  cluster_sync_all();

  // The row's LSE from the CS partials, combined in rank order by warp 0.
  if (tid < 32) {
    float pm = -INFINITY, ps = 0.f;
    if (tid < CS) {
      pm = dsmem_ld_f32(dsmem_addr(&s_part[0], (uint32_t)tid));
      ps = dsmem_ld_f32(dsmem_addr(&s_part[1], (uint32_t)tid));
    }
    const float M = warp_max(pm);
    const float t = warp_sum(ps > 0.f ? ps * expf(pm - M) : 0.f);
    if (tid == 0) s_lse = M + logf(t);
  }
  const int k = min(K, n);
  if (rank == 0) {
    // Gathers the candidates (registers), passes the second barrier, selects.
    const int nc = CS * kc;
    int32_t* out = idx + row * (long long)K;
    if (nc <= bd) cluster_merge_topk<1>(s_key, &s_cnt, CS, kc, max(k, 1), ts, s_key, out, k > 0 ? K : 0);
    else if (nc <= 2 * bd) cluster_merge_topk<2>(s_key, &s_cnt, CS, kc, max(k, 1), ts, s_key, out, k > 0 ? K : 0);
    else if (nc <= 4 * bd) cluster_merge_topk<4>(s_key, &s_cnt, CS, kc, max(k, 1), ts, s_key, out, k > 0 ? K : 0);
    else cluster_merge_topk<8>(s_key, &s_cnt, CS, kc, max(k, 1), ts, s_key, out, k > 0 ? K : 0);
    if (k == 0)
      for (int p = tid; p < K; p += bd) out[p] = -1;
  } else {
    cluster_sync_all();
  }
  __syncthreads();
  const float lse = s_lse;
  float* grow = gates + row * (long long)C;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int gi = lo + e * bd + tid;
    if (gi < C) grow[gi] = gi < n ? gate_of(f[e], lse, phi) : 0.f;
  }
}

int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// The bucket-selection cluster kernel for rows of up to 16 * 512 entries,
// when the device holds such a cluster; false leaves the row to other paths.
bool launch_cbucket_topk(const float* scores, long long total, int rows, int C, int causal, int K,
                         int phi, float* gates, int32_t* idx, cudaStream_t stream) {
  if (C > kSelMaxCta * kCbChunk || total * kSelMaxCta > 0x7fffffffLL) return false;
  const int CS = (C + kCbChunk - 1) / kCbChunk;
  if (CS < 2) return false;
  // rank 0's gather buffer: the bucket path's candidates, or the exact path's CS * K
  const size_t smem = (size_t)max(kSelCand, CS * K) * sizeof(uint64_t);
  auto kern = gate_topk_cbucket_kernel;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(total * CS));
  cfg.blockDim = dim3(kCbThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static std::mutex mu;
  static signed char fits[kSelMaxCta + 1] = {};
  {
    std::lock_guard<std::mutex> lk(mu);
    if (fits[CS] == 0) {
      bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(kSelMaxCta * 256 * sizeof(uint64_t))) == cudaSuccess;
      if (ok && CS > 8)
        ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
             cudaSuccess;
      int nclusters = 0;
      if (ok) ok = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess;
      fits[CS] = (ok && nclusters > 0) ? 1 : -1;
      (void)cudaGetLastError();
    }
    if (fits[CS] < 0) return false;
  }
  if (cudaLaunchKernelEx(&cfg, kern, scores, rows, C, causal, K, CS, phi, gates, idx) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  note_launches(1);
  return true;
}

// Launches the cluster kernel when the row fits (C <= 16 chunks of 4096) and
// the device can hold such a cluster; returns false (nothing launched) to
// leave the row to the two-launch path.
bool launch_cluster_topk(const float* scores, long long total, int rows, int C, int causal, int K,
                         int phi, float* gates, int32_t* idx, cudaStream_t stream) {
  if (C > kClMaxCta * 4096 || total * kClMaxCta > 0x7fffffffLL) return false;
  int Lc = kClThreads;
  while ((C + Lc - 1) / Lc > kClMaxCta) Lc <<= 1;
  const int CS = (C + Lc - 1) / Lc, E = Lc / kClThreads, kc = min(K, Lc);
  const int EM = pow2_at_least((CS * kc + kClThreads - 1) / kClThreads);
  const size_t smem = (size_t)max(E, EM) * kClThreads * sizeof(uint64_t);
  void (*kern)(const float*, int, int, int, int, int, int, float*, int32_t*) =
      E == 1 ? gate_topk_cluster_kernel<1> : E == 2 ? gate_topk_cluster_kernel<2>
             : E == 4 ? gate_topk_cluster_kernel<4> : gate_topk_cluster_kernel<8>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(total * CS));
  cfg.blockDim = dim3(kClThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Whether this (E, CS) fits on the device, asked once per process.
  static std::mutex mu;
  static signed char fits[4][kClMaxCta + 1] = {};
  const int ei = E == 1 ? 0 : E == 2 ? 1 : E == 4 ? 2 : 3;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (fits[ei][CS] == 0) {
      bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem) == cudaSuccess;
      if (ok && CS > 8)
        ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
             cudaSuccess;
      int nclusters = 0;
      if (ok) ok = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess;
      fits[ei][CS] = (ok && nclusters > 0) ? 1 : -1;
      (void)cudaGetLastError();  // a refused query leaves no sticky error behind
    }
    if (fits[ei][CS] < 0) return false;
  }
  if (cudaLaunchKernelEx(&cfg, kern, scores, rows, C, causal, K, CS, phi, gates, idx) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  note_launches(1);
  return true;
}

}  // namespace

cudaError_t launch_gate_topk(const float* scores, int B, int Hkv, int rows, int C, int causal,
                             int K, int phi, float* gates, int32_t* idx, cudaStream_t stream) {
  const long long total = (long long)B * Hkv * rows;
  if (total == 0) return cudaSuccess;
  const int maxlen = causal ? min(rows - 1, C) : C;
  if (maxlen <= kWarpCap) {
    const long long grid = (total + kWarpRowsPerCta - 1) / kWarpRowsPerCta;
    gate_topk_warp_kernel<<<(unsigned)grid, 32 * kWarpRowsPerCta, 0, stream>>>(
        scores, (int)total, rows, C, causal, K, phi, gates, idx);
    note_launches(1);
  } else if (launch_cbucket_topk(scores, total, rows, C, causal, K, phi, gates, idx, stream)) {
    // decode-sized rows: a cluster per row, bucket selection
  } else if (launch_cluster_topk(scores, total, rows, C, causal, K, phi, gates, idx, stream)) {
    // one launch: a cluster of chunk CTAs per row
  } else if (C <= 2048) {
    // One block per row sorts the whole row.
    const int Lp = pow2_at_least(C), threads = min(1024, Lp);
    const size_t smem = (size_t)Lp * sizeof(uint64_t);
    if (Lp / threads == 1)
      gate_topk_chunk_kernel<true, 1><<<(unsigned)total, threads, smem, stream>>>(
          scores, rows, C, causal, K, 1, min(K, Lp), phi, gates, idx);
    else
      gate_topk_chunk_kernel<true, 2><<<(unsigned)total, threads, smem, stream>>>(
          scores, rows, C, causal, K, 1, min(K, Lp), phi, gates, idx);
    note_launches(1);
  } else {
    // The shortest chunk (a power of two from 512) whose candidates fit the
    // merge (chunks * kc <= 8192) and whose partials fit the row's gates
    // (chunks * (2 + 2 kc) floats <= C). 8192 always qualifies for
    // 2048 < C <= 262144.
    int Lc = 512, chunks = 0, kc = 0;
    for (;; Lc <<= 1) {
      chunks = (C + Lc - 1) / Lc;
      kc = min(K, Lc);
      if (Lc == kMaxChunk ||
          ((long long)chunks * kc <= kMaxCandidates && (long long)chunks * (2 + 2 * kc) <= C))
        break;
    }
    if ((long long)chunks * kc > kMaxCandidates || (long long)chunks * (2 + 2 * kc) > C)
      return cudaErrorInvalidValue;  // beyond the documented C limit
    const int threads = min(1024, Lc), E = Lc / threads;
    cudaError_t e = cudaSuccess;
    const size_t smem = (size_t)Lc * sizeof(uint64_t);
    const unsigned grid = (unsigned)(total * chunks);
    auto chunk = [&](auto kern) {
      if (smem + kStaticSmem > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        kern<<<grid, threads, smem, stream>>>(scores, rows, C, causal, K, chunks, kc, phi, gates,
                                              idx);
    };
    switch (E) {
      case 1: chunk(gate_topk_chunk_kernel<false, 1>); break;
      case 2: chunk(gate_topk_chunk_kernel<false, 2>); break;
      case 4: chunk(gate_topk_chunk_kernel<false, 4>); break;
      default: chunk(gate_topk_chunk_kernel<false, 8>); break;
    }
    note_launches(1);
    if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
    const int Mp = pow2_at_least(chunks * kc);
    const int mthreads = min(1024, max(256, Mp)), ME = max(1, Mp / mthreads);
    const size_t msmem = (size_t)ME * mthreads * sizeof(uint64_t);
    auto merge = [&](auto kern) {
      if (msmem + kStaticSmem > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
      if (e == cudaSuccess)
        kern<<<(unsigned)total, mthreads, msmem, stream>>>(scores, rows, C, causal, K, chunks, kc,
                                                           phi, gates, idx);
    };
    switch (ME) {
      case 1: merge(gate_topk_merge_kernel<1>); break;
      case 2: merge(gate_topk_merge_kernel<2>); break;
      case 4: merge(gate_topk_merge_kernel<4>); break;
      default: merge(gate_topk_merge_kernel<8>); break;
    }
    note_launches(1);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace sas
