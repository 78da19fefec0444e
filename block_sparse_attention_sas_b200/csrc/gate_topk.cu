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
#include "sas_common.cuh"
#include "sas_internal.h"

namespace sas {
namespace {

// Order-preserving map fp32 -> uint32 (larger float -> larger key); -0.0 is
// folded onto +0.0 so that the two compare equal, as fp32 values do.
__device__ __forceinline__ uint32_t fkey(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

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

constexpr int kWarpRowsPerCta = 8;
constexpr int kWarpCap = 512;   // longest row handled by one warp
constexpr int kMaxK = 256;

// ---------------------------------------------------------------------------
// One warp per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * kWarpRowsPerCta)
gate_topk_warp_kernel(const float* __restrict__ scores, int total_rows, int rows, int C,
                      int causal, int K, float* __restrict__ gates, int32_t* __restrict__ idx) {
  __shared__ float s_val[kWarpRowsPerCta][kWarpCap];
  __shared__ uint32_t s_selkey[kWarpRowsPerCta][kMaxK];
  __shared__ int32_t s_selidx[kWarpRowsPerCta][kMaxK];
  __shared__ int s_hist[kWarpRowsPerCta][256];

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
  for (int i = lane; i < C; i += 32) g[i] = (i < n) ? expf(v[i] - lse) : 0.f;

  const int k = min(K, n);
  if (k > 0) {
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
// One CTA per row (long rows).
// ---------------------------------------------------------------------------
constexpr int kCtaThreads = 512;
constexpr int kCtaWarps = kCtaThreads / 32;

__device__ __forceinline__ float block_reduce_max(float x, float* red) {
  x = warp_max(x);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  float y = (lane < kCtaWarps) ? red[lane] : -INFINITY;
  return warp_max(y);
}
__device__ __forceinline__ float block_reduce_sum(float x, float* red) {
  x = warp_sum(x);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  float y = (lane < kCtaWarps) ? red[lane] : 0.f;
  return warp_sum(y);
}
// Dynamic shared memory: the row's values when n <= cap (else they are
// re-read from global memory, where the row stays L2-resident).
__global__ void __launch_bounds__(kCtaThreads)
gate_topk_cta_kernel(const float* __restrict__ scores, int rows, int C, int causal, int K,
                     int cap, float* __restrict__ gates, int32_t* __restrict__ idx) {
  extern __shared__ float s_dyn[];
  __shared__ float red_f[kCtaWarps];
  __shared__ int warp_cnt[kCtaWarps];
  __shared__ uint32_t s_selkey[kMaxK];
  __shared__ int32_t s_selidx[kMaxK];
  __shared__ int s_whist[kCtaWarps][256];
  __shared__ int s_hist[256];
  __shared__ int s_pick[2];

  const long long row = blockIdx.x;
  const int r = (int)(row % rows);
  const int n = causal ? min(r, C) : C;
  const float* s = scores + row * (long long)C;
  float* g = gates + row * (long long)C;
  int32_t* out = idx + row * (long long)K;
  const bool in_smem = n <= cap;
  const float* v = in_smem ? s_dyn : s;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;

  float mx = -INFINITY;
  for (int i = tid; i < n; i += kCtaThreads) {
    const float f = s[i];
    if (in_smem) s_dyn[i] = f;
    mx = fmaxf(mx, f);
  }
  mx = block_reduce_max(mx, red_f);  // includes a __syncthreads after the smem fill
  float sum = 0.f;
  for (int i = tid; i < n; i += kCtaThreads) sum += expf(v[i] - mx);
  sum = block_reduce_sum(sum, red_f);
  const float lse = mx + logf(sum);
  for (int i = tid; i < C; i += kCtaThreads) g[i] = (i < n) ? expf(v[i] - lse) : 0.f;

  const int k = min(K, n);
  if (k > 0) {
    // Radix select over four 8-bit digits: per-warp histograms, summed into
    // one, and warp 0 picks the digit.
    uint32_t tau = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < kCtaWarps * 256; i += kCtaThreads) (&s_whist[0][0])[i] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += kCtaThreads) {
        const int i = base + tid;
        const uint32_t key = (i < n) ? fkey(v[i]) : 0u;
        warp_hist_add(s_whist[w], (key >> shift) & 255u, i < n && (key & mask) == tau);
      }
      __syncthreads();
      for (int bin = tid; bin < 256; bin += kCtaThreads) {
        int t = 0;
#pragma unroll
        for (int x = 0; x < kCtaWarps; ++x) t += s_whist[x][bin];
        s_hist[bin] = t;
      }
      __syncthreads();
      if (w == 0) {
        int above;
        const uint32_t dig = warp_pick_digit(s_hist, krem, above);
        if (lane == 0) {
          s_pick[0] = (int)dig;
          s_pick[1] = above;
        }
      }
      __syncthreads();
      krem -= s_pick[1];
      tau |= (uint32_t)s_pick[0] << shift;
      mask |= 255u << shift;
    }
    const int need_eq = krem;

    // Each warp owns a contiguous, 32-aligned range of the row. Pass 1
    // counts its keys equal to tau; an exclusive scan over warps gives each
    // warp the number of equal keys before its range.
    const int chunk = ((n + kCtaWarps - 1) / kCtaWarps + 31) & ~31;
    const int lo = min(n, w * chunk), hi = min(n, lo + chunk);
    const uint32_t lt = lanemask_lt();
    int eq_here = 0;
    for (int i = lo + lane; i < hi; i += 32) eq_here += fkey(v[i]) == tau;
    eq_here = __reduce_add_sync(0xffffffffu, eq_here);
    __syncthreads();
    if (lane == 0) warp_cnt[w] = eq_here;
    __syncthreads();
    int eq_before = 0;
    for (int x = 0; x < w; ++x) eq_before += warp_cnt[x];
    // Pass 2: survivors per warp (no writes), then scan for output offsets.
    int sel_here = 0;
    {
      int run_eq = eq_before;
      for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const uint32_t key = (i < hi) ? fkey(v[i]) : 0u;
        const bool is_gt = (i < hi) && key > tau;
        const bool is_eq = (i < hi) && key == tau;
        const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
        const bool sel = is_gt || (is_eq && run_eq + __popc(eqm & lt) < need_eq);
        sel_here += __popc(__ballot_sync(0xffffffffu, sel));
        run_eq += __popc(eqm);
      }
    }
    __syncthreads();
    if (lane == 0) warp_cnt[w] = sel_here;
    __syncthreads();
    int sel_before = 0;
    for (int x = 0; x < w; ++x) sel_before += warp_cnt[x];
    // Pass 3: write survivors in index order.
    {
      int run_eq = eq_before, run_sel = sel_before;
      for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const uint32_t key = (i < hi) ? fkey(v[i]) : 0u;
        const bool is_gt = (i < hi) && key > tau;
        const bool is_eq = (i < hi) && key == tau;
        const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
        const bool sel = is_gt || (is_eq && run_eq + __popc(eqm & lt) < need_eq);
        const uint32_t selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const int p = run_sel + __popc(selm & lt);
          s_selkey[p] = key;
          s_selidx[p] = i;
        }
        run_eq += __popc(eqm);
        run_sel += __popc(selm);
      }
    }
    __syncthreads();
    for (int p = tid; p < k; p += kCtaThreads) {
      const uint32_t kp = s_selkey[p];
      int rank = 0;
      for (int q = 0; q < k; ++q) {
        const uint32_t kq = s_selkey[q];
        rank += (kq > kp) || (kq == kp && q < p);
      }
      out[rank] = s_selidx[p];
    }
  }
  for (int p = k + tid; p < K; p += kCtaThreads) out[p] = -1;
}

constexpr int kCtaSmemCap = 48 * 1024;  // floats kept in shared memory (192 KB)

}  // namespace

cudaError_t launch_gate_topk(const float* scores, int B, int Hkv, int rows, int C, int causal,
                             int K, float* gates, int32_t* idx, cudaStream_t stream) {
  const long long total = (long long)B * Hkv * rows;
  if (total == 0) return cudaSuccess;
  const int maxlen = causal ? min(rows - 1, C) : C;
  if (maxlen <= kWarpCap) {
    const long long grid = (total + kWarpRowsPerCta - 1) / kWarpRowsPerCta;
    gate_topk_warp_kernel<<<(unsigned)grid, 32 * kWarpRowsPerCta, 0, stream>>>(
        scores, (int)total, rows, C, causal, K, gates, idx);
    note_launches(1);
  } else {
    const int cap = min(maxlen, kCtaSmemCap);
    const size_t smem = (size_t)cap * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(gate_topk_cta_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gate_topk_cta_kernel<<<(unsigned)total, kCtaThreads, smem, stream>>>(scores, rows, C, causal,
                                                                          K, cap, gates, idx);
    note_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace sas
