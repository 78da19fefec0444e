// Block-selector scores from pooled block summaries.
//
// The evolve.pub review of SAS (Frequently asked questions) describes the
// selector as working from pooling-based block summaries and scoring history
// blocks per query block and KV-head group; no page gives its layers or
// weights. This library computes the weight-free form of that: a block's key
// summary is the mean of its keys, a query block's summary the mean of its
// rows over the G heads of the group, and
//   s[j, m] = scale * qbar_j . kbar_m   (m < j; 0 for m >= j),
// which is also the mean of the attention logits scale * q_i . k_t over every
// (row, head, key) pair of the two blocks. At decode the query summary is the
// mean of the group's G query heads of the single token.
//
// Memory-bound work (one read of q and k for the summaries), then a small
// fp32 product per (batch, KV head): plain CUDA-core kernels.
#include <math.h>

#include "sas_common.cuh"
#include "sas_internal.h"

namespace sas {
namespace {

// Mean over the rows of block m of `group` consecutive planes:
// x [planes_out * group][T][D] -> out [planes_out][N][D] fp32.
// One CTA per (output plane, block); thread c owns column c.
template <typename T, int D>
__global__ void __launch_bounds__(D)
pool_kernel(const T* __restrict__ x, int group, int rows, int pitch, int b, int N,
            float* __restrict__ out) {
  const int m = blockIdx.x, po = blockIdx.y, c = threadIdx.x;
  const int r0 = m * b, r1 = min(rows, r0 + b);
  float acc = 0.f;
  for (int g = 0; g < group; ++g) {
    const T* p = x + ((long long)(po * group + g) * pitch + r0) * D + c;
    for (int r = r0; r < r1; ++r, p += D) acc += ld_f(p);
  }
  const int cnt = (r1 - r0) * group;
  out[((long long)po * N + m) * D + c] = cnt > 0 ? acc / (float)cnt : 0.f;
}

// Training scores of one (batch, KV head): S = scale * Qbar Kbar^T on the
// causal lower triangle (m < j), 0 elsewhere. 32 x 32 output tiles, the d
// dimension staged through shared memory in chunks of 32.
constexpr int kTile = 32;
__global__ void __launch_bounds__(256)
scores_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int N, int d,
              float scale, float* __restrict__ s) {
  __shared__ float qs[kTile][kTile + 1], ks[kTile][kTile + 1];
  const int jt = blockIdx.y, mt = blockIdx.x, u = blockIdx.z;
  const int tx = threadIdx.x % kTile, ty = threadIdx.x / kTile;  // 32 x 8
  const float* qb = qbar + (long long)u * N * d;
  const float* kb = kbar + (long long)u * N * d;
  float* out = s + (long long)u * N * N;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (mt <= jt) {  // tiles above the diagonal hold no m < j
    for (int c0 = 0; c0 < d; c0 += kTile) {
      __syncthreads();
      for (int r = ty; r < kTile; r += 8) {
        const int j = jt * kTile + r, m = mt * kTile + r;
        qs[r][tx] = j < N ? qb[(long long)j * d + c0 + tx] : 0.f;
        ks[r][tx] = m < N ? kb[(long long)m * d + c0 + tx] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int c = 0; c < kTile; ++c) {
        const float kv = ks[tx][c];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = fmaf(qs[ty + 8 * i][c], kv, acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = jt * kTile + ty + 8 * i, m = mt * kTile + tx;
    if (j < N && m < N) out[(long long)j * N + m] = (m < j) ? acc[i] * scale : 0.f;
  }
}

// Decode scores of one (batch, KV head): qbar = the mean of the G query heads,
// s[m] = scale * qbar . kbar_m for m < C. A CTA takes 64 history blocks (8
// per warp), so the query mean is formed once per 64 blocks; a lane reads
// d / 32 consecutive columns of a block (one vector load when kbar is
// 16-byte aligned), and the eight blocks of a warp are in flight together.
template <typename T, int D, bool VEC>
__global__ void __launch_bounds__(256)
decode_scores_kernel(const T* __restrict__ q, const float* __restrict__ kbar, int G, int C,
                     float scale, float* __restrict__ s) {
  constexpr int W = D / 32;  // columns a lane
  __shared__ __align__(16) float qb[D];
  const int u = blockIdx.y;  // batch * Hkv + kvh
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = 0.f;
    for (int g = 0; g < G; ++g) a += ld_f(q + ((long long)u * G + g) * D + c);
    qb[c] = a / (float)G;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 64 + (threadIdx.x >> 5) * 8;
  float qv[W];
#pragma unroll
  for (int w = 0; w < W; ++w) qv[w] = qb[lane * W + w];
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + i;
    float kv[W];
    if (m < C) {
      const float* kr = kbar + ((long long)u * C + m) * D + lane * W;
      if (VEC && W == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(kr));
        kv[0] = v.x;
        kv[1 % W] = v.y;
        kv[2 % W] = v.z;
        kv[3 % W] = v.w;
      } else {
#pragma unroll
        for (int w = 0; w < W; ++w) kv[w] = __ldg(kr + w);
      }
    } else {
#pragma unroll
      for (int w = 0; w < W; ++w) kv[w] = 0.f;
    }
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) a = fmaf(qv[w], kv[w], a);
    acc[i] = a;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = warp_sum(acc[i]);
    if (lane == 0 && m0 + i < C) s[(long long)u * C + m0 + i] = a * scale;
  }
}

template <typename T>
cudaError_t pool(const T* x, int planes_out, int group, int rows, int pitch, int b, int N, int d,
                 float* out, cudaStream_t st) {
  if (N == 0 || planes_out == 0) return cudaSuccess;
  dim3 grid(N, planes_out);
  if (d == 128)
    pool_kernel<T, 128><<<grid, 128, 0, st>>>(x, group, rows, pitch, b, N, out);
  else
    pool_kernel<T, 64><<<grid, 64, 0, st>>>(x, group, rows, pitch, b, N, out);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_summaries(sas_dtype_t dt, const void* x, int planes_out, int group,
                                   int rows, int pitch, int b, int N, int d, float* out,
                                   cudaStream_t st) {
  if (dt == SAS_F32)
    return pool((const float*)x, planes_out, group, rows, pitch, b, N, d, out, st);
  return pool((const __nv_bfloat16*)x, planes_out, group, rows, pitch, b, N, d, out, st);
}

cudaError_t launch_selector_scores(const float* qbar, const float* kbar, int units, int N, int d,
                                   float scale, float* scores, cudaStream_t st) {
  if (units == 0 || N == 0) return cudaSuccess;
  dim3 grid((N + kTile - 1) / kTile, (N + kTile - 1) / kTile, units);
  scores_kernel<<<grid, 256, 0, st>>>(qbar, kbar, N, d, scale, scores);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_selector_scores_decode(sas_dtype_t dt, const void* q, const float* kbar,
                                          int units, int G, int C, int d, float scale,
                                          float* scores, cudaStream_t st) {
  if (units == 0 || C == 0) return cudaSuccess;
  dim3 grid((C + 63) / 64, units);
  const bool vec = (reinterpret_cast<uintptr_t>(kbar) & 15) == 0;
  auto go = [&](auto kern, const auto* qq) {
    kern<<<grid, 256, 0, st>>>(qq, kbar, G, C, scale, scores);
  };
  if (dt == SAS_F32) {
    const float* qq = (const float*)q;
    if (d == 128)
      vec ? go(decode_scores_kernel<float, 128, true>, qq)
          : go(decode_scores_kernel<float, 128, false>, qq);
    else
      go(decode_scores_kernel<float, 64, false>, qq);
  } else {
    const __nv_bfloat16* qq = (const __nv_bfloat16*)q;
    if (d == 128)
      vec ? go(decode_scores_kernel<__nv_bfloat16, 128, true>, qq)
          : go(decode_scores_kernel<__nv_bfloat16, 128, false>, qq);
    else
      go(decode_scores_kernel<__nv_bfloat16, 64, false>, qq);
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sas
