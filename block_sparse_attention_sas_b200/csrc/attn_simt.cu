// Gated block-sparse causal attention on CUDA cores (fp32 FMA), forward and
// backward, for every supported (dtype, d, b). This is the exact-fp32 path
// (TF32 or bf16 tensor cores cannot meet an fp32 tolerance) and the path for
// shapes the tensor-core kernels do not cover.
//
// Forward (picx.dev SAS summary, Methodology Eq. 9; 1/sqrt(d) scale from the
// reproduction README, Core equations): one CTA per (query block j, row
// chunk, q head, batch) walks the selected history blocks of its KV head
// (bias log g_m) and then the current block (bias 0, causal), keeping an
// online softmax (running max, running sum) per row.
//
// Backward (chain rule through Eq. 9; Eq. 5 inner form for the gate
// gradient; Eq. 6 Jacobian for the scores):
//   csr:     per (batch, kv head), the query blocks that selected each key block
//   dq:      per (query block, q head): recompute P and dP = dO V^T; a
//            first sweep sums D_i = sum_t P_it dP_it exactly (using the
//            stored bf16 o for dO . o would carry its rounding into every
//            gradient), a second forms dS = P (dP - D), dq += scale dS K and
//            da(j,m) = sum of dS over the tile (one partial per q head and
//            row chunk); D goes to the workspace for the dk/dv pass
//   dkdv:    per key block: over the diagonal and every selecting query
//            block and head, dv += P^T dO, dk += scale dS^T Q
//   jacobian: dscores[j,k] = [k in I_j] da_k - g_k sum_{m in I_j} da_m
// Every sum has a fixed order, so results are deterministic.
#include <math.h>

#include "sas_common.cuh"
#include "sas_internal.h"

namespace sas {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int BS> struct Tiles {
  static constexpr int ROWS = BS < 64 ? BS : 64;  // query rows per CTA
  static constexpr int RC = BS / ROWS;             // row chunks per block
};

__device__ __forceinline__ long long idx_row(const AttnShape& s, int bi, int kvh, int j) {
  return ((long long)(bi * s.Hkv + kvh) * s.N + j);
}

// Block m of the iteration `it` for query block j: history slots first, then
// the current block. Returns false when the slot is empty or invalid.
__device__ __forceinline__ bool pick_block(const AttnShape& s, const int32_t* idx,
                                           const float* gates, int bi, int kvh, int j, int it,
                                           int nsel, int& m, float& bias, bool& cur,
                                           const DevCtx& ctx) {
  bias = 0.f;
  if (it == nsel) {
    m = j;
    cur = true;
    return true;
  }
  cur = false;
  if (s.dense) {
    m = it;
    return true;
  }
  m = idx[idx_row(s, bi, kvh, j) * s.K + it];
  if (m == -1) return false;
  if (m < -1 || m >= j) {
    if (threadIdx.x == 0) report(ctx, kDevErrBadIndex);
    return false;
  }
  if (gates) bias = logf(gates[idx_row(s, bi, kvh, j) * s.N + m]);
  return true;
}

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads)
fwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
           const int32_t* __restrict__ idx, const float* __restrict__ gates, AttnShape s,
           T* __restrict__ o, float* __restrict__ lse, DevCtx ctx) {
  constexpr int ROWS = Tiles<BS>::ROWS, RC = Tiles<BS>::RC;
  constexpr int DP = D + 1, BP = BS + 1;
  constexpr int NACC = ROWS * D / kThreads;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* Ks = Qs + ROWS * DP;
  float* Vs = Ks + BS * DP;
  float* Ps = Vs + BS * D;
  float* row_m = Ps + ROWS * BP;
  float* row_l = row_m + ROWS;
  float* row_a = row_l + ROWS;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x / RC, rc = blockIdx.x % RC;
  const int h = blockIdx.y, bi = blockIdx.z;
  const int G = s.Hq / s.Hkv, kvh = h / G;
  const int r0 = j * BS + rc * ROWS;
  if (r0 >= s.T) return;
  const long long qbase = (long long)(bi * s.Hq + h) * s.T * D;
  const long long kbase = (long long)(bi * s.Hkv + kvh) * s.T * D;

  for (int e = tid; e < ROWS * D; e += kThreads) {
    const int r = e / D, c = e % D, row = r0 + r;
    Qs[r * DP + c] = row < s.T ? ld_f(q + qbase + (long long)row * D + c) : 0.f;
  }
  for (int r = tid; r < ROWS; r += kThreads) {
    row_m[r] = -INFINITY;
    row_l[r] = 0.f;
  }
  float acc[NACC];
#pragma unroll
  for (int x = 0; x < NACC; ++x) acc[x] = 0.f;

  const int nsel = s.dense ? j : s.K;
  for (int it = 0; it <= nsel; ++it) {
    int m;
    float bias;
    bool cur;
    if (!pick_block(s, idx, gates, bi, kvh, j, it, nsel, m, bias, cur, ctx)) continue;
    // Outer gating: the logits carry no bias and the block's weights are
    // scaled by its gate w after the softmax.
    const float w = s.outer ? expf(bias) : 1.f;
    if (s.outer) bias = 0.f;
    __syncthreads();
    for (int e = tid; e < BS * D; e += kThreads) {
      const int t = e / D, c = e % D, key = m * BS + t;
      const bool ok = key < s.T;
      Ks[t * DP + c] = ok ? ld_f(k + kbase + (long long)key * D + c) : 0.f;
      Vs[t * D + c] = ok ? ld_f(v + kbase + (long long)key * D + c) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < ROWS * BS; e += kThreads) {
      const int r = e / BS, c = e % BS;
      float a = 0.f;
#pragma unroll 8
      for (int kk = 0; kk < D; ++kk) a = fmaf(Qs[r * DP + kk], Ks[c * DP + kk], a);
      float x = fmaf(a, s.scale, bias);
      const int qi = r0 + r, ki = m * BS + c;
      if (ki >= s.T || (cur && ki > qi)) x = -INFINITY;
      Ps[r * BP + c] = x;
    }
    __syncthreads();
    for (int r = warp; r < ROWS; r += kWarps) {
      float mx = -INFINITY;
      for (int c = lane; c < BS; c += 32) mx = fmaxf(mx, Ps[r * BP + c]);
      mx = warp_max(mx);
      const float mold = row_m[r];
      const float mnew = fmaxf(mold, mx);
      float sum = 0.f;
      for (int c = lane; c < BS; c += 32) {
        const float p = (mnew == -INFINITY) ? 0.f : expf(Ps[r * BP + c] - mnew);
        Ps[r * BP + c] = p * w;
        sum += p;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        const float alpha = (mnew == -INFINITY) ? 1.f : expf(mold - mnew);
        row_a[r] = alpha;
        row_l[r] = row_l[r] * alpha + sum;
        row_m[r] = mnew;
      }
    }
    __syncthreads();
#pragma unroll
    for (int x = 0; x < NACC; ++x) {
      const int e = tid + x * kThreads, r = e / D, c = e % D;
      float a = acc[x] * row_a[r];
#pragma unroll 8
      for (int t = 0; t < BS; ++t) a = fmaf(Ps[r * BP + t], Vs[t * D + c], a);
      acc[x] = a;
    }
  }
  __syncthreads();
#pragma unroll
  for (int x = 0; x < NACC; ++x) {
    const int e = tid + x * kThreads, r = e / D, c = e % D, row = r0 + r;
    if (row < s.T) st_f(o + qbase + (long long)row * D + c, acc[x] / row_l[r]);
  }
  for (int r = tid; r < ROWS; r += kThreads) {
    const int row = r0 + r;
    if (row < s.T) lse[(long long)(bi * s.Hq + h) * s.T + row] = row_m[r] + logf(row_l[r]);
  }
}

// ---------------------------------------------------------------------------
// Backward: reverse index. For (batch, kv head): list[off[m] .. off[m+1]) holds
// j*K + slot for every query block j whose slot selects key block m, in
// ascending j. One CTA per (batch, kv head).
// ---------------------------------------------------------------------------
constexpr int kCsrChunk = 16384;  // idx entries staged in shared memory at a time

// In-place exclusive prefix sum of a[0..n) in shared memory by the whole CTA
// (blockDim.x a multiple of 32, at most 1024); returns the total.
__device__ int block_exclusive_scan(int32_t* a, int n, int32_t* warp_tot) {
  const int nt = blockDim.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int per = (n + nt - 1) / nt;
  const int lo = min(n, t * per), hi = min(n, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += a[i];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int v = lane < nt / 32 ? warp_tot[lane] : 0;
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += x;
    }
    if (lane < nt / 32) warp_tot[lane] = vi - v;  // exclusive warp offsets
    if (lane == 31) warp_tot[32] = vi;            // total
  }
  __syncthreads();
  int run = warp_tot[w] + incl - sum;
  for (int i = lo; i < hi; ++i) {
    const int x = a[i];
    a[i] = run;
    run += x;
  }
  const int total = warp_tot[32];
  __syncthreads();
  return total;
}

// Reverse index of one (batch, KV head): for each key block m, the entries
// e = j*K + slot with idx[e] == m (m < j), in ascending order of e (so of j).
// The entries pass through shared memory in chunks (all threads load, many
// loads in flight); counts by shared-memory atomics and a block scan; then
// one warp walks the entries in order and places each at its key block's
// cursor (lanes holding the same block are ranked within the warp), so the
// lists come out sorted without a sort.
__global__ void __launch_bounds__(kThreads)
csr_kernel(const int32_t* __restrict__ idx, AttnShape s, int32_t* __restrict__ off_all,
           int32_t* __restrict__ list_all, DevCtx ctx) {
  extern __shared__ int32_t cnt[];  // N counts (then cursors), then a chunk of entries
  int32_t* stage = cnt + s.N;
  __shared__ int32_t warp_tot[33];
  const int bh = blockIdx.x;
  const int32_t* ix = idx + (long long)bh * s.N * s.K;
  int32_t* off = off_all + (long long)bh * (s.N + 1);
  int32_t* list = list_all + (long long)bh * s.N * s.K;
  const int total = s.N * s.K;
  const bool one_chunk = total <= kCsrChunk;
  auto load_chunk = [&](int c0, int nc) {
#pragma unroll 8
    for (int i = threadIdx.x; i < nc; i += blockDim.x) stage[i] = __ldg(ix + c0 + i);
  };
  for (int m = threadIdx.x; m < s.N; m += blockDim.x) cnt[m] = 0;
  for (int c0 = 0; c0 < total; c0 += kCsrChunk) {
    const int nc = min(kCsrChunk, total - c0);
    __syncthreads();
    load_chunk(c0, nc);
    __syncthreads();
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      const int e = c0 + i, m = stage[i];
      if (m >= 0 && m < e / s.K) atomicAdd(&cnt[m], 1);
    }
  }
  __syncthreads();
  const int n_all = block_exclusive_scan(cnt, s.N, warp_tot);
  for (int m = threadIdx.x; m < s.N; m += blockDim.x) off[m] = cnt[m];
  if (threadIdx.x == 0) off[s.N] = n_all;
  for (int c0 = 0; c0 < total; c0 += kCsrChunk) {
    const int nc = min(kCsrChunk, total - c0);
    if (!one_chunk) {
      __syncthreads();
      load_chunk(c0, nc);
      __syncthreads();
    }
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const uint32_t lt = (1u << lane) - 1u;
      for (int c = 0; c < nc; c += 32) {
        const int e = c0 + c + lane;
        const int m = c + lane < nc ? stage[c + lane] : -1;
        const bool valid = m >= 0 && m < e / s.K;
        const int key = valid ? m : -1 - lane;  // invalid lanes match nobody
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        int pos = 0;
        if (valid) pos = cnt[m] + __popc(peers & lt);
        __syncwarp();
        if (valid && (peers & lt) == 0) cnt[m] += __popc(peers);  // the group's leader
        __syncwarp();
        if (valid) list[pos] = e;
      }
    }
  }
}

// The same reverse index for N <= 1024 from a bitmap in shared memory: bit
// (m, j) is set when query block j selects key block m (rows of idx are
// distinct, so once at most). The entry e = j K + slot goes to position
// off[m] + (set bits of row m below j): the list of m in ascending j, the
// order the kernel above produces, with no ordered scan.
constexpr int kCsrBitmapMaxN = 1024;
__global__ void __launch_bounds__(1024)
csr_bitmap_kernel(const int32_t* __restrict__ idx, AttnShape s, int32_t* __restrict__ off_all,
                  int32_t* __restrict__ list_all) {
  extern __shared__ uint32_t bm[];  // [N][W] bit rows, then N counts
  __shared__ int32_t warp_tot[33];
  const int W = (s.N + 31) >> 5;
  int32_t* cnt = reinterpret_cast<int32_t*>(bm + (size_t)s.N * W);
  const int bh = blockIdx.x, tid = threadIdx.x, bd = blockDim.x;
  const int32_t* ix = idx + (long long)bh * s.N * s.K;
  int32_t* off = off_all + (long long)bh * (s.N + 1);
  int32_t* list = list_all + (long long)bh * s.N * s.K;
  const int total = s.N * s.K;
  for (int i = tid; i < s.N * W; i += bd) bm[i] = 0u;
  for (int m = tid; m < s.N; m += bd) cnt[m] = 0;
  __syncthreads();
  for (int e = tid; e < total; e += bd) {
    const int m = __ldg(ix + e), j = e / s.K;
    if (m >= 0 && m < j) {
      atomicOr(&bm[m * W + (j >> 5)], 1u << (j & 31));
      atomicAdd(&cnt[m], 1);
    }
  }
  __syncthreads();
  const int n_all = block_exclusive_scan(cnt, s.N, warp_tot);
  __syncthreads();
  for (int m = tid; m < s.N; m += bd) off[m] = cnt[m];
  if (tid == 0) off[s.N] = n_all;
  for (int e = tid; e < total; e += bd) {
    const int m = __ldg(ix + e), j = e / s.K;
    if (m >= 0 && m < j) {
      const uint32_t* row = bm + m * W;
      int r = __popc(row[j >> 5] & ((1u << (j & 31)) - 1u));
      for (int x = 0; x < (j >> 5); ++x) r += __popc(row[x]);
      list[cnt[m] + r] = e;
    }
  }
}

// ---------------------------------------------------------------------------
// Backward: dq and da (one CTA per query block row chunk and q head)
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads)
dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
          const float* __restrict__ lse, const T* __restrict__ dO, float* __restrict__ Dv,
          const int32_t* __restrict__ idx, const float* __restrict__ gates, AttnShape s,
          T* __restrict__ dq, float* __restrict__ da, DevCtx ctx) {
  constexpr int ROWS = Tiles<BS>::ROWS, RC = Tiles<BS>::RC;
  constexpr int DP = D + 1, BP = BS + 1;
  constexpr int NACC = ROWS * D / kThreads;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* dOs = Qs + ROWS * DP;
  float* Ks = dOs + ROWS * DP;
  float* Vs = Ks + BS * DP;
  float* Ps = Vs + BS * DP;
  float* dSs = Ps + ROWS * BP;
  float* lse_s = dSs + ROWS * BP;
  float* D_s = lse_s + ROWS;
  float* red = D_s + ROWS;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x / RC, rc = blockIdx.x % RC;
  const int h = blockIdx.y, bi = blockIdx.z;
  const int G = s.Hq / s.Hkv, kvh = h / G;
  const int r0 = j * BS + rc * ROWS;
  if (r0 >= s.T) return;
  const long long qrow0 = (long long)(bi * s.Hq + h) * s.T;
  const long long kbase = (long long)(bi * s.Hkv + kvh) * s.T * D;

  for (int e = tid; e < ROWS * D; e += kThreads) {
    const int r = e / D, c = e % D, row = r0 + r;
    const bool ok = row < s.T;
    Qs[r * DP + c] = ok ? ld_f(q + (qrow0 + row) * D + c) : 0.f;
    dOs[r * DP + c] = ok ? ld_f(dO + (qrow0 + row) * D + c) : 0.f;
  }
  for (int r = tid; r < ROWS; r += kThreads) {
    const int row = r0 + r;
    lse_s[r] = row < s.T ? lse[qrow0 + row] : 0.f;
    D_s[r] = 0.f;
  }
  float acc[NACC];
#pragma unroll
  for (int x = 0; x < NACC; ++x) acc[x] = 0.f;

  // Sweep 0 computes D_i = sum_t P_it dP_it exactly (the softmax Jacobian's
  // row term; equal to dO_i . o_i for the unrounded o). Sweep 1 forms dS.
  const int nsel = s.dense ? j : s.K;
  for (int sweep = 0; sweep < 2; ++sweep)
  for (int it = 0; it <= nsel; ++it) {
    int m;
    float bias;
    bool cur;
    if (!pick_block(s, idx, gates, bi, kvh, j, it, nsel, m, bias, cur, ctx)) continue;
    __syncthreads();
    for (int e = tid; e < BS * D; e += kThreads) {
      const int t = e / D, c = e % D, key = m * BS + t;
      const bool ok = key < s.T;
      Ks[t * DP + c] = ok ? ld_f(k + kbase + (long long)key * D + c) : 0.f;
      Vs[t * DP + c] = ok ? ld_f(v + kbase + (long long)key * D + c) : 0.f;
    }
    __syncthreads();
    if (sweep == 0) {
      for (int e = tid; e < ROWS * BS; e += kThreads) {
        const int r = e / BS, c = e % BS;
        float a = 0.f, b = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < D; ++kk) {
          a = fmaf(Qs[r * DP + kk], Ks[c * DP + kk], a);
          b = fmaf(dOs[r * DP + kk], Vs[c * DP + kk], b);
        }
        const int qi = r0 + r, ki = m * BS + c;
        float p = 0.f;
        if (qi < s.T && ki < s.T && !(cur && ki > qi)) p = expf(fmaf(a, s.scale, bias) - lse_s[r]);
        Ps[r * BP + c] = p * b;
      }
      __syncthreads();
      for (int r = warp; r < ROWS; r += kWarps) {
        float t = 0.f;
        for (int c = lane; c < BS; c += 32) t += Ps[r * BP + c];
        t = warp_sum(t);
        if (lane == 0) D_s[r] += t;
      }
      continue;
    }
    float dsum = 0.f;
    const float dinv = s.outer ? fminf(expf(-bias), 3.0e38f) : 1.f;
    for (int e = tid; e < ROWS * BS; e += kThreads) {
      const int r = e / BS, c = e % BS;
      float a = 0.f, b = 0.f;
#pragma unroll 8
      for (int kk = 0; kk < D; ++kk) {
        a = fmaf(Qs[r * DP + kk], Ks[c * DP + kk], a);
        b = fmaf(dOs[r * DP + kk], Vs[c * DP + kk], b);
      }
      const int qi = r0 + r, ki = m * BS + c;
      float p = 0.f;
      if (qi < s.T && ki < s.T && !(cur && ki > qi)) p = expf(fmaf(a, s.scale, bias) - lse_s[r]);
      // p is the gated weight (g p under outer gating). Inner: dS = p (dP - D);
      // outer: dS = p (dP - D / g) and da sums p dP (Eq. 5, outer form, times g).
      const float ds = p * (b - D_s[r] * dinv);
      Ps[r * BP + c] = p;
      dSs[r * BP + c] = ds;
      dsum += s.outer ? p * b : ds;
    }
    if (!cur && !s.dense && da != nullptr) {
      dsum = warp_sum(dsum);
      if (lane == 0) red[warp] = dsum;
    }
    __syncthreads();
    if (!cur && !s.dense && da != nullptr && tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kWarps; ++w) t += red[w];
      da[((qrow0 / s.T) * (long long)s.N * RC + (long long)j * RC + rc) * s.K + it] = t;
    }
#pragma unroll
    for (int x = 0; x < NACC; ++x) {
      const int e = tid + x * kThreads, r = e / D, c = e % D;
      float a = 0.f;
#pragma unroll 8
      for (int t = 0; t < BS; ++t) a = fmaf(dSs[r * BP + t], Ks[t * DP + c], a);
      acc[x] = fmaf(a, s.scale, acc[x]);
    }
  }
#pragma unroll
  for (int x = 0; x < NACC; ++x) {
    const int e = tid + x * kThreads, r = e / D, c = e % D, row = r0 + r;
    if (row < s.T) st_f(dq + (qrow0 + row) * D + c, acc[x]);
  }
  for (int r = tid; r < ROWS; r += kThreads) {
    const int row = r0 + r;
    if (row < s.T) Dv[qrow0 + row] = D_s[r];
  }
}

// ---------------------------------------------------------------------------
// Backward: dk and dv (one CTA per key block, all query blocks that attend it)
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads)
dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            const float* __restrict__ lse, const T* __restrict__ dO,
            const float* __restrict__ Dv, const float* __restrict__ gates,
            const int32_t* __restrict__ csr_off, const int32_t* __restrict__ csr_list,
            AttnShape s, T* __restrict__ dk, T* __restrict__ dv, DevCtx ctx) {
  constexpr int QR = Tiles<BS>::ROWS, RC = Tiles<BS>::RC;
  constexpr int DP = D + 1, BP = BS + 1;
  constexpr int NACC = BS * D / kThreads;
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + BS * DP;
  float* Qs = Vs + BS * DP;
  float* dOs = Qs + QR * DP;
  float* Ps = dOs + QR * DP;
  float* dSs = Ps + QR * BP;
  float* lse_s = dSs + QR * BP;
  float* D_s = lse_s + QR;

  const int tid = threadIdx.x;
  const int m = blockIdx.x, kvh = blockIdx.y, bi = blockIdx.z;
  const int G = s.Hq / s.Hkv;
  const long long kbase = (long long)(bi * s.Hkv + kvh) * s.T * D;
  for (int e = tid; e < BS * D; e += kThreads) {
    const int t = e / D, c = e % D, key = m * BS + t;
    const bool ok = key < s.T;
    Ks[t * DP + c] = ok ? ld_f(k + kbase + (long long)key * D + c) : 0.f;
    Vs[t * DP + c] = ok ? ld_f(v + kbase + (long long)key * D + c) : 0.f;
  }
  float adk[NACC], adv[NACC];
#pragma unroll
  for (int x = 0; x < NACC; ++x) adk[x] = adv[x] = 0.f;

  const int bh = bi * s.Hkv + kvh;
  int n_list;
  const int32_t* lst = nullptr;
  if (s.dense) {
    n_list = s.N - 1 - m;
  } else {
    const int lo = csr_off[(long long)bh * (s.N + 1) + m];
    n_list = csr_off[(long long)bh * (s.N + 1) + m + 1] - lo;
    lst = csr_list + (long long)bh * s.N * s.K + lo;
  }
  for (int it = -1; it < n_list; ++it) {
    int j;
    float bias = 0.f;
    const bool cur = it < 0;
    if (cur) {
      j = m;
    } else if (s.dense) {
      j = m + 1 + it;
    } else {
      j = lst[it] / s.K;
      if (gates) bias = logf(gates[((long long)bh * s.N + j) * s.N + m]);
    }
    const float dinv = s.outer ? fminf(expf(-bias), 3.0e38f) : 1.f;  // outer gating: dS = p (dP - D / g)
    for (int g = 0; g < G; ++g) {
      const int h = kvh * G + g;
      const long long qrow0 = (long long)(bi * s.Hq + h) * s.T;
      for (int qc = 0; qc < RC; ++qc) {
        const int r0 = j * BS + qc * QR;
        if (r0 >= s.T) break;
        __syncthreads();
        for (int e = tid; e < QR * D; e += kThreads) {
          const int r = e / D, c = e % D, row = r0 + r;
          const bool ok = row < s.T;
          Qs[r * DP + c] = ok ? ld_f(q + (qrow0 + row) * D + c) : 0.f;
          dOs[r * DP + c] = ok ? ld_f(dO + (qrow0 + row) * D + c) : 0.f;
        }
        for (int r = tid; r < QR; r += kThreads) {
          const int row = r0 + r;
          lse_s[r] = row < s.T ? lse[qrow0 + row] : 0.f;
          D_s[r] = row < s.T ? Dv[qrow0 + row] : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < QR * BS; e += kThreads) {
          const int r = e / BS, c = e % BS;
          float a = 0.f, b = 0.f;
#pragma unroll 8
          for (int kk = 0; kk < D; ++kk) {
            a = fmaf(Qs[r * DP + kk], Ks[c * DP + kk], a);
            b = fmaf(dOs[r * DP + kk], Vs[c * DP + kk], b);
          }
          const int qi = r0 + r, ki = m * BS + c;
          float p = 0.f;
          if (qi < s.T && ki < s.T && !(cur && ki > qi)) p = expf(fmaf(a, s.scale, bias) - lse_s[r]);
          Ps[r * BP + c] = p;
          dSs[r * BP + c] = p * (b - D_s[r] * dinv);
        }
        __syncthreads();
#pragma unroll
        for (int x = 0; x < NACC; ++x) {
          const int e = tid + x * kThreads, t = e / D, c = e % D;
          float a = adv[x], b = 0.f;
#pragma unroll 8
          for (int r = 0; r < QR; ++r) {
            a = fmaf(Ps[r * BP + t], dOs[r * DP + c], a);
            b = fmaf(dSs[r * BP + t], Qs[r * DP + c], b);
          }
          adv[x] = a;
          adk[x] = fmaf(b, s.scale, adk[x]);
        }
      }
    }
  }
#pragma unroll
  for (int x = 0; x < NACC; ++x) {
    const int e = tid + x * kThreads, t = e / D, c = e % D, key = m * BS + t;
    if (key < s.T) {
      st_f(dk + kbase + (long long)key * D + c, adk[x]);
      st_f(dv + kbase + (long long)key * D + c, adv[x]);
    }
  }
}

// ---------------------------------------------------------------------------
// Backward: gate Jacobian (Eq. 6 for the softmax gates; the sigmoid and
// raw-logit variants have diagonal Jacobians), one warp per score row
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
jacobian_kernel(const float* __restrict__ da, const int32_t* __restrict__ idx,
                const float* __restrict__ gates, AttnShape s, int RC, float* __restrict__ ds) {
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)s.B * s.Hkv * s.N;
  if (row >= rows) return;
  const int j = (int)(row % s.N);
  const long long bh = row / s.N;
  const int bi = (int)(bh / s.Hkv), kvh = (int)(bh % s.Hkv);
  const int G = s.Hq / s.Hkv;
  const int32_t* ix = idx + row * s.K;
  // da of each slot: sum over the group's heads and the row chunks.
  float tot = 0.f;
  for (int sl = lane; sl < s.K; sl += 32) {
    const int m = ix[sl];
    if (m < 0 || m >= j) continue;
    float a = 0.f;
    for (int g = 0; g < G; ++g)
      for (int rc = 0; rc < RC; ++rc)
        a += da[(((long long)(bi * s.Hq + kvh * G + g) * s.N + j) * RC + rc) * s.K + sl];
    tot += a;
  }
  tot = warp_sum(tot);
  float* out = ds + row * s.N;
  const float* g = gates + row * s.N;
  // softmax: d log g_m / d s_k = delta_mk - g_k (Eq. 6); sigmoid: delta_mk
  // (1 - g_k); raw logits: delta_mk. Only the softmax has the -g_k sum term.
  const bool softmax = s.phi == SAS_PHI_SOFTMAX;
  for (int kk = lane; kk < s.N; kk += 32) out[kk] = (kk < j && softmax) ? -g[kk] * tot : 0.f;
  __syncwarp();
  for (int sl = lane; sl < s.K; sl += 32) {
    const int m = ix[sl];
    if (m < 0 || m >= j) continue;
    float a = 0.f;
    for (int g2 = 0; g2 < G; ++g2)
      for (int rc = 0; rc < RC; ++rc)
        a += da[(((long long)(bi * s.Hq + kvh * G + g2) * s.N + j) * RC + rc) * s.K + sl];
    if (s.phi == SAS_PHI_SIGMOID) a *= 1.f - g[m];
    out[m] += a;
  }
}

size_t fwd_smem(int D, int BS) {
  const int ROWS = BS < 64 ? BS : 64;
  return sizeof(float) *
         ((size_t)ROWS * (D + 1) + (size_t)BS * (D + 1) + (size_t)BS * D + (size_t)ROWS * (BS + 1) +
          3 * ROWS);
}
size_t dq_smem(int D, int BS) {
  const int ROWS = BS < 64 ? BS : 64;
  return sizeof(float) * (2 * (size_t)ROWS * (D + 1) + 2 * (size_t)BS * (D + 1) +
                          2 * (size_t)ROWS * (BS + 1) + 2 * ROWS + kWarps);
}
size_t dkdv_smem(int D, int BS) {
  const int QR = BS < 64 ? BS : 64;
  return sizeof(float) * (2 * (size_t)BS * (D + 1) + 2 * (size_t)QR * (D + 1) +
                          2 * (size_t)QR * (BS + 1) + 2 * QR);
}

template <typename T, int D, int BS>
cudaError_t fwd_t(const AttnShape& s, const void* q, const void* k, const void* v,
                  const int32_t* idx, const float* gates, void* o, float* lse, const DevCtx& ctx,
                  cudaStream_t st) {
  const size_t smem = fwd_smem(D, BS);
  auto kern = fwd_kernel<T, D, BS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(s.N * Tiles<BS>::RC, s.Hq, s.B);
  kern<<<grid, kThreads, smem, st>>>((const T*)q, (const T*)k, (const T*)v, idx, gates, s, (T*)o,
                                     lse, ctx);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T, int D, int BS>
cudaError_t bwd_t(const AttnShape& s, const void* q, const void* k, const void* v, const void* o,
                  const float* lse, const void* dO, const int32_t* idx, const float* gates,
                  void* dq, void* dk, void* dv, float* dscores, void* ws, const DevCtx& ctx,
                  cudaStream_t st) {
  const BwdWorkspace L = bwd_workspace_layout(s, false);
  char* w = static_cast<char*>(ws);
  float* Dv = reinterpret_cast<float*>(w + L.off_D);
  float* da = reinterpret_cast<float*>(w + L.off_da);
  int32_t* coff = reinterpret_cast<int32_t*>(w + L.off_csr_off);
  int32_t* clist = reinterpret_cast<int32_t*>(w + L.off_csr_list);
  cudaError_t e;
  if (!s.dense) {
    if ((e = launch_bwd_csr(s, idx, coff, clist, ctx, st)) != cudaSuccess) return e;
  }
  {
    const size_t smem = dq_smem(D, BS);
    auto kern = dq_kernel<T, D, BS>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(s.N * Tiles<BS>::RC, s.Hq, s.B);
    kern<<<grid, kThreads, smem, st>>>((const T*)q, (const T*)k, (const T*)v, lse, (const T*)dO,
                                       Dv, idx, gates, s, (T*)dq, dscores ? da : nullptr, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t smem = dkdv_smem(D, BS);
    auto kern = dkdv_kernel<T, D, BS>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(s.N, s.Hkv, s.B);
    kern<<<grid, kThreads, smem, st>>>((const T*)q, (const T*)k, (const T*)v, lse, (const T*)dO,
                                       Dv, gates, coff, clist, s, (T*)dk, (T*)dv, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dscores) {
    const long long srows = (long long)s.B * s.Hkv * s.N;
    jacobian_kernel<<<(unsigned)((srows + kWarps - 1) / kWarps), kThreads, 0, st>>>(
        da, idx, gates, s, Tiles<BS>::RC, dscores);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t fwd_dispatch(const AttnShape& s, const void* q, const void* k, const void* v,
                         const int32_t* idx, const float* gates, void* o, float* lse,
                         const DevCtx& ctx, cudaStream_t st) {
#define SAS_FWD_CASE(DD, BB) \
  if (s.d == DD && s.b == BB) return fwd_t<T, DD, BB>(s, q, k, v, idx, gates, o, lse, ctx, st);
  SAS_FWD_CASE(64, 16) SAS_FWD_CASE(64, 32) SAS_FWD_CASE(64, 64)
  SAS_FWD_CASE(128, 16) SAS_FWD_CASE(128, 32) SAS_FWD_CASE(128, 64)
#undef SAS_FWD_CASE
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t bwd_dispatch(const AttnShape& s, const void* q, const void* k, const void* v,
                         const void* o, const float* lse, const void* dO, const int32_t* idx,
                         const float* gates, void* dq, void* dk, void* dv, float* dscores,
                         void* ws, const DevCtx& ctx, cudaStream_t st) {
#define SAS_BWD_CASE(DD, BB)                                                                    \
  if (s.d == DD && s.b == BB)                                                                   \
    return bwd_t<T, DD, BB>(s, q, k, v, o, lse, dO, idx, gates, dq, dk, dv, dscores, ws, ctx, \
                            st);
  SAS_BWD_CASE(64, 16) SAS_BWD_CASE(64, 32) SAS_BWD_CASE(64, 64)
  SAS_BWD_CASE(128, 16) SAS_BWD_CASE(128, 32) SAS_BWD_CASE(128, 64)
#undef SAS_BWD_CASE
  return cudaErrorInvalidValue;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

cudaError_t launch_bwd_csr(const AttnShape& s, const int32_t* idx, int32_t* off, int32_t* list,
                           const DevCtx& ctx, cudaStream_t st) {
  if (s.N <= kCsrBitmapMaxN) {
    const size_t W = ((size_t)s.N + 31) / 32;
    const size_t smem = sizeof(uint32_t) * ((size_t)s.N * W + s.N);
    cudaError_t e = cudaFuncSetAttribute(csr_bitmap_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    csr_bitmap_kernel<<<s.B * s.Hkv, 1024, smem, st>>>(idx, s, off, list);
    note_launches(1);
    return cudaGetLastError();
  }
  const size_t smem = sizeof(int32_t) * ((size_t)s.N + kCsrChunk);
  cudaError_t e =
      cudaFuncSetAttribute(csr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  csr_kernel<<<s.B * s.Hkv, kThreads, smem, st>>>(idx, s, off, list, ctx);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_jacobian(const AttnShape& s, const float* da, const int32_t* idx,
                                const float* gates, float* dscores, int RC, cudaStream_t st) {
  const long long srows = (long long)s.B * s.Hkv * s.N;
  jacobian_kernel<<<(unsigned)((srows + kWarps - 1) / kWarps), kThreads, 0, st>>>(
      da, idx, gates, s, RC, dscores);
  note_launches(1);
  return cudaGetLastError();
}

BwdWorkspace bwd_workspace_layout(const AttnShape& s, bool tc) {
  BwdWorkspace L;
  const int RC = tc ? 4 : (s.b < 64 ? 1 : s.b / 64);
  size_t off = 0;
  L.off_D = off;
  off = align256(off + sizeof(float) * (size_t)s.B * s.Hq * s.T);
  L.off_da = off;
  off = align256(off + sizeof(float) * (size_t)s.B * s.Hq * s.N * RC * (s.dense ? 0 : s.K));
  L.off_csr_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)s.B * s.Hkv * (s.N + 1));
  L.off_csr_list = off;
  off = align256(off + sizeof(int32_t) * (size_t)s.B * s.Hkv * s.N * (s.dense ? 0 : s.K));
  // Launch order of the key-outer dK/dV CTAs (most selected key blocks first).
  L.off_order = off;
  off = align256(off + sizeof(int32_t) * (size_t)s.B * s.Hkv * s.N);
  // dS tiles of every (query block, 128-row tile, slot) for the dq kernel:
  // [B][Hkv][N][G/2][K + 1][128][64] bf16 (slot K: the current block).
  L.off_ds = off;
  if (tc && !s.dense)  // the dense comparison recomputes dS for dq instead
    off = align256(off + sizeof(uint16_t) * (size_t)s.B * s.Hkv * s.N * (s.Hq / s.Hkv / 2) *
                             (s.K + 1) * 128 * 64);
  L.total = off;
  return L;
}

cudaError_t launch_attn_fwd_simt(sas_dtype_t dt, const AttnShape& s, const void* q, const void* k,
                                 const void* v, const int32_t* idx, const float* gates, void* o,
                                 float* lse, const DevCtx& ctx, cudaStream_t st) {
  if (dt == SAS_F32) return fwd_dispatch<float>(s, q, k, v, idx, gates, o, lse, ctx, st);
  return fwd_dispatch<__nv_bfloat16>(s, q, k, v, idx, gates, o, lse, ctx, st);
}

cudaError_t launch_attn_bwd_simt(sas_dtype_t dt, const AttnShape& s, const void* q, const void* k,
                                 const void* v, const void* o, const float* lse, const void* dO,
                                 const int32_t* idx, const float* gates, void* dq, void* dk,
                                 void* dv, float* dscores, void* ws, const DevCtx& ctx,
                                 cudaStream_t st) {
  if (dt == SAS_F32)
    return bwd_dispatch<float>(s, q, k, v, o, lse, dO, idx, gates, dq, dk, dv, dscores, ws, ctx,
                               st);
  return bwd_dispatch<__nv_bfloat16>(s, q, k, v, o, lse, dO, idx, gates, dq, dk, dv, dscores, ws,
                                     ctx, st);
}

}  // namespace sas
