// One-token decode over a KV cache: the selected history blocks plus the
// current block (picx.dev SAS summary, Theoretical Foundation Eq. 2 with the
// gates dropped, Methodology Eq. 9 with them; evolve.pub review, Summary:
// hard selection kept at inference, gates dropped). Also the dense decode
// used as the comparison (every block).
//
// The work is a stream over the selected K/V rows (G query heads share each
// KV head), so it is bound by HBM bandwidth: per (batch, kv head) the
// (K+1)*b*d*2 elements of K and V are read once, with 16-byte loads.
//
// Layout of the work: the block list of a (batch, kv head) is cut into
// `splits` ranges of `bps` blocks, one CTA each. A CTA's four warps take
// 16-token chunks of its range round-robin and keep an online softmax per
// query head; the warps are merged in shared memory, and each CTA stores a
// partial (max, sum, unnormalised o) to the workspace. The last CTA of a
// (batch, kv head) to finish (counted with an atomic ticket) merges the
// partials by log-sum-exp, writes o, and resets the ticket to zero.
#include <math.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_internal.h"

namespace sas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kChunk = 16;  // tokens per warp work item
constexpr int kLPT = 8;     // lanes per token in the q.k phase
constexpr int kMaxSplits = 64;    // bounds the last CTA's merge

// Loads `n` consecutive elements (n*sizeof(T) a multiple of 4 bytes) as floats.
template <typename T, int n>
__device__ __forceinline__ void load_f(const T* p, float (&out)[n]);

template <>
__device__ __forceinline__ void load_f<__nv_bfloat16, 16>(const __nv_bfloat16* p, float (&out)[16]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    out[2 * i] = bf16lo(w[i]);
    out[2 * i + 1] = bf16hi(w[i]);
  }
}
template <>
__device__ __forceinline__ void load_f<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&out)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = bf16lo(w[i]);
    out[2 * i + 1] = bf16hi(w[i]);
  }
}
template <int n>
__device__ __forceinline__ void load_f_f32(const float* p, float (&out)[n]) {
  static_assert(n % 2 == 0, "");
  if constexpr (n % 4 == 0) {
#pragma unroll
    for (int i = 0; i < n / 4; ++i) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(p) + i);
      out[4 * i] = a.x;
      out[4 * i + 1] = a.y;
      out[4 * i + 2] = a.z;
      out[4 * i + 3] = a.w;
    }
  } else {
    const float2 a = __ldg(reinterpret_cast<const float2*>(p));
    out[0] = a.x;
    out[1] = a.y;
  }
}
template <> __device__ __forceinline__ void load_f<float, 16>(const float* p, float (&o)[16]) { load_f_f32<16>(p, o); }
template <> __device__ __forceinline__ void load_f<float, 8>(const float* p, float (&o)[8]) { load_f_f32<8>(p, o); }

// Block held by slot `sl` of a (batch, kv head): sparse -> idx entries then the
// current block; dense -> blocks 0..C in order. Returns -1 for an empty slot.
__device__ __forceinline__ int slot_block(const DecodeShape& s, const int32_t* ix, int sl,
                                          const DevCtx& ctx) {
  if (s.dense) return sl;
  if (sl == s.K) return s.C;
  const int m = ix[sl];
  if (m == -1) return -1;
  if (m < -1 || m >= s.C) {
    report(ctx, kDevErrBadIndex);
    return -1;
  }
  return m;
}

// Shared-memory element loads (vectorised; the stage buffers are 16-byte aligned).
template <typename T, int n>
__device__ __forceinline__ void lds_f(const T* p, float (&out)[n]) {
  if constexpr (sizeof(T) == 2) {
    static_assert(n % 2 == 0, "");
    if constexpr (n % 8 == 0) {
#pragma unroll
      for (int i = 0; i < n / 8; ++i) {
        const uint4 a = reinterpret_cast<const uint4*>(p)[i];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          out[8 * i + 2 * j] = bf16lo(w[j]);
          out[8 * i + 2 * j + 1] = bf16hi(w[j]);
        }
      }
    } else if constexpr (n == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(p);
      out[0] = bf16lo(a.x); out[1] = bf16hi(a.x); out[2] = bf16lo(a.y); out[3] = bf16hi(a.y);
    } else {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(p);
      out[0] = bf16lo(a); out[1] = bf16hi(a);
    }
  } else {
    if constexpr (n % 4 == 0) {
#pragma unroll
      for (int i = 0; i < n / 4; ++i) {
        const float4 a = reinterpret_cast<const float4*>(p)[i];
        out[4 * i] = a.x; out[4 * i + 1] = a.y; out[4 * i + 2] = a.z; out[4 * i + 3] = a.w;
      }
    } else {
      const float2 a = *reinterpret_cast<const float2*>(p);
      out[0] = a.x; out[1] = a.y;
    }
  }
}

constexpr int kMaxStages = 4;

// One CTA per (split, kv head, batch). Thread 0 streams the split's K/V blocks
// into a ring of shared-memory stages with bulk async copies (one mbarrier per
// stage, waits bounded by the context's limit); the four warps compute each
// staged block from shared memory (warp w takes the block's 16-token chunks
// w, w+4, ...) while later blocks are in flight.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
              const int32_t* __restrict__ idx, const float* __restrict__ gates, DecodeShape s,
              int nst, T* __restrict__ o, float* __restrict__ ws_ml, float* __restrict__ ws_o,
              uint32_t* __restrict__ ws_cnt, DevCtx ctx) {
  constexpr int VPL = D / kLPT;   // q.k dims per lane
  constexpr int TPP = 32 / kLPT;  // tokens per pass
  constexpr int DPL = D / 32;     // output dims per lane
  extern __shared__ __align__(128) unsigned char stage_mem[];
  __shared__ uint64_t full_bar[kMaxStages];
  __shared__ float s_x[kWarps][G][kChunk];
  __shared__ float s_p[kWarps][kChunk][G];
  __shared__ float s_m[kWarps][G], s_l[kWarps][G];
  __shared__ float s_o[kWarps][G][D];
  __shared__ float s_w[G * kMaxSplits];
  __shared__ float s_L[G];
  __shared__ int s_last, s_abort;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, bi = blockIdx.z;
  const int unit = bi * s.Hkv + kvh;
  const int nslots = s.dense ? s.C + 1 : s.K + 1;
  const int sl0 = split * s.bps, sl1 = min(nslots, sl0 + s.bps);
  const int ns = sl1 - sl0;
  const int cpb = s.b / kChunk;  // chunks per block
  const long long cache0 = (long long)unit * s.Lcap * D;
  const int32_t* ix = s.dense ? nullptr : idx + (long long)unit * s.K;
  const size_t stage_elems = (size_t)2 * s.b * D;  // K block then V block

  // Block of slot i of this split and its number of valid rows (0: skip).
  auto slot_rows = [&](int i, int& m) -> int {
    m = slot_block(s, ix, sl0 + i, ctx);
    if (m < 0) return 0;
    return min(s.b, s.L - m * s.b);
  };
  auto issue = [&](int i) -> bool {
    int m;
    const int rows = slot_rows(i, m);
    if (rows <= 0) return false;
    const int st = i % nst;
    T* kst = reinterpret_cast<T*>(stage_mem) + st * stage_elems;
    const uint32_t bytes = (uint32_t)(rows * D * sizeof(T));
    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
    bulk_g2s(kst, kc + cache0 + (long long)m * s.b * D, bytes, &full_bar[st]);
    bulk_g2s(kst + (size_t)s.b * D, vc + cache0 + (long long)m * s.b * D, bytes, &full_bar[st]);
    return true;
  };

  if (tid == 0) {
    for (int st = 0; st < nst; ++st) mbar_init(&full_bar[st], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  // Stage bookkeeping, identical in every thread: the parity each stage's
  // next completion will have, and (thread 0) which stages hold a copy in flight.
  uint32_t phase_bits = 0, pending = 0;
  if (tid == 0)
    for (int i = 0; i < min(nst, ns); ++i)
      if (issue(i)) pending |= 1u << (i % nst);

  // q for this lane's q.k dims, all G heads (scaled once).
  float qr[G][VPL];
  const int dseg = (lane % kLPT) * VPL;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    load_f<T, VPL>(q + ((long long)bi * s.Hq + kvh * G + g) * D + dseg, qr[g]);
#pragma unroll
    for (int i = 0; i < VPL; ++i) qr[g][i] *= s.scale;
  }
  float m_run[G], l_run[G], acc[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[g][i] = 0.f;
  }

  for (int i = 0; i < ns; ++i) {
    int m;
    const int rows = slot_rows(i, m);  // the same in every thread
    const int st = i % nst;
    if (rows > 0) {
      const bool ready = mbar_wait(ctx, &full_bar[st], (phase_bits >> st) & 1u);
      phase_bits ^= 1u << st;
      if (tid == 0) pending &= ~(1u << st);
      if (!__all_sync(0xffffffffu, ready)) {
        if (lane == 0) s_abort = 1;
      } else {
        const T* ks = reinterpret_cast<const T*>(stage_mem) + st * stage_elems;
        const T* vs = ks + (size_t)s.b * D;
        const float bias = (!s.dense && s.use_gates && sl0 + i < s.K)
                               ? logf(gates[(long long)unit * s.C + m]) : 0.f;
        for (int c = w; c < cpb; c += kWarps) {
          const int t0 = c * kChunk;
          if (t0 >= rows) break;
          const int nt = min(kChunk, rows - t0);
          // ---- logits: kLPT lanes per token, TPP tokens per pass
#pragma unroll
          for (int pass = 0; pass < kChunk / TPP; ++pass) {
            const int tt = pass * TPP + lane / kLPT;
            float dot[G];
#pragma unroll
            for (int g = 0; g < G; ++g) dot[g] = 0.f;
            if (tt < nt) {
              float kf[VPL];
              lds_f<T, VPL>(ks + (size_t)(t0 + tt) * D + dseg, kf);
#pragma unroll
              for (int g = 0; g < G; ++g)
#pragma unroll
                for (int x = 0; x < VPL; ++x) dot[g] = fmaf(qr[g][x], kf[x], dot[g]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
              for (int off = kLPT / 2; off > 0; off >>= 1)
                dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], off);
            }
            if ((lane % kLPT) == 0) {
#pragma unroll
              for (int g = 0; g < G; ++g) s_x[w][g][tt] = (tt < nt) ? dot[g] + bias : -INFINITY;
            }
          }
          __syncwarp();
          // ---- online softmax: lane t < kChunk owns token t
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float x = (lane < kChunk) ? s_x[w][g][lane] : -INFINITY;
            const float mx = warp_max(x);
            const float mnew = fmaxf(m_run[g], mx);
            const float p = (mnew == -INFINITY) ? 0.f : expf(x - mnew);
            const float alpha = (mnew == -INFINITY) ? 1.f : expf(m_run[g] - mnew);
            l_run[g] = l_run[g] * alpha + warp_sum(p);
            m_run[g] = mnew;
            if (lane < kChunk) s_p[w][lane][g] = p;
#pragma unroll
            for (int x2 = 0; x2 < DPL; ++x2) acc[g][x2] *= alpha;
          }
          __syncwarp();
          // ---- o += p v: lane owns DPL consecutive dims
#pragma unroll 4
          for (int t = 0; t < nt; ++t) {
            float vf[DPL];
            lds_f<T, DPL>(vs + (size_t)(t0 + t) * D + lane * DPL, vf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float p = s_p[w][t][g];
#pragma unroll
              for (int x2 = 0; x2 < DPL; ++x2) acc[g][x2] = fmaf(p, vf[x2], acc[g][x2]);
            }
          }
          __syncwarp();
        }
      }
    }
    __syncthreads();  // stage st is free; s_abort is visible
    if (s_abort) break;
    if (tid == 0 && i + nst < ns && issue(i + nst)) pending |= 1u << st;
  }
  if (s_abort) {
    // A copy never arrived: stop, let the copies still in flight land (bounded
    // waits), and leave without a partial; the error word reports it.
    if (tid == 0)
      for (int st = 0; st < nst; ++st)
        if (pending & (1u << st)) (void)mbar_wait(ctx, &full_bar[st], (phase_bits >> st) & 1u);
    return;
  }

  // ---- merge the warps of this CTA
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      s_m[w][g] = m_run[g];
      s_l[w][g] = l_run[g];
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) s_o[w][g][lane * DPL + i] = acc[g][i];
  }
  __syncthreads();
  const long long hbase = (long long)bi * s.Hq + kvh * G;  // first q head of the unit
  for (int e = tid; e < G * D; e += kThreads) {
    const int g = e / D, dd = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int x = 0; x < kWarps; ++x) M = fmaxf(M, s_m[x][g]);
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int x = 0; x < kWarps; ++x) {
      const float f = (s_m[x][g] == -INFINITY) ? 0.f : expf(s_m[x][g] - M);
      L += f * s_l[x][g];
      A += f * s_o[x][g][dd];
    }
    if (s.splits == 1) {
      st_f(o + (hbase + g) * D + dd, A / L);
    } else {
      const long long pidx = (hbase + g) * s.splits + split;
      ws_o[pidx * D + dd] = A;
      if (dd == 0) {
        ws_ml[2 * pidx] = M;
        ws_ml[2 * pidx + 1] = L;
      }
    }
  }
  if (s.splits == 1) return;

  // ---- the last CTA of the unit merges the partials by log-sum-exp
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t ticket = atomicAdd(&ws_cnt[unit], 1u);
    s_last = (ticket == (uint32_t)(s.splits - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int P = s.splits;
  for (int e = tid; e < G * P; e += kThreads) s_w[e] = __ldcg(&ws_ml[2 * (hbase * P + e)]);
  __syncthreads();
  for (int g = w; g < G; g += kWarps) {
    float M = -INFINITY;
    for (int x = lane; x < P; x += 32) M = fmaxf(M, s_w[g * P + x]);
    M = warp_max(M);
    float L = 0.f;
    for (int x = lane; x < P; x += 32) {
      const float mx = s_w[g * P + x];
      const float f = (mx == -INFINITY) ? 0.f : expf(mx - M);
      L += f * __ldcg(&ws_ml[2 * (hbase * P + g * P + x) + 1]);
      s_w[g * P + x] = f;
    }
    L = warp_sum(L);
    if (lane == 0) s_L[g] = L;
  }
  __syncthreads();
  for (int e = tid; e < G * (D / 4); e += kThreads) {
    const int g = e / (D / 4), d4 = e % (D / 4);
    const float4* src = reinterpret_cast<const float4*>(ws_o + (hbase + g) * P * D) + d4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int x = 0; x < P; ++x) {
      const float4 v = __ldcg(src + (size_t)x * (D / 4));
      const float f = s_w[g * P + x];
      a.x = fmaf(f, v.x, a.x);
      a.y = fmaf(f, v.y, a.y);
      a.z = fmaf(f, v.z, a.z);
      a.w = fmaf(f, v.w, a.w);
    }
    const float inv = 1.f / s_L[g];
    T* dst = o + (hbase + g) * D + d4 * 4;
    st_f(dst + 0, a.x * inv);
    st_f(dst + 1, a.y * inv);
    st_f(dst + 2, a.z * inv);
    st_f(dst + 3, a.w * inv);
  }
}

int decode_stages(const DecodeShape& s, size_t elem) {
  const size_t stage = (size_t)2 * s.b * s.d * elem;
  int nst = (int)((96u << 10) / stage);
  return max(2, min(kMaxStages, nst));
}

template <typename T, int D, int G>
cudaError_t decode_t(const DecodeShape& s, const void* q, const void* kc, const void* vc,
                     const int32_t* idx, const float* gates, void* o, void* ws, const DevCtx& ctx,
                     cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  const size_t parts = (size_t)s.B * s.Hq * s.splits;
  float* ws_ml = reinterpret_cast<float*>(w);
  float* ws_o = reinterpret_cast<float*>(w + ((2 * parts * sizeof(float) + 255) & ~(size_t)255));
  uint32_t* ws_cnt = reinterpret_cast<uint32_t*>(
      reinterpret_cast<char*>(ws_o) + ((parts * D * sizeof(float) + 255) & ~(size_t)255));
  cudaError_t e;
  if (s.splits > 1) {
    // Tickets start at zero on every call, whatever the workspace held before.
    e = cudaMemsetAsync(ws_cnt, 0, sizeof(uint32_t) * (size_t)s.B * s.Hkv, st);
    if (e != cudaSuccess) return e;
    note_launches(1);
  }
  const int nst = decode_stages(s, sizeof(T));
  const size_t smem = (size_t)nst * 2 * s.b * D * sizeof(T);
  auto kern = decode_kernel<T, D, G>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(s.splits, s.Hkv, s.B);
  kern<<<grid, kThreads, smem, st>>>((const T*)q, (const T*)kc, (const T*)vc, idx, gates, s, nst,
                                     (T*)o, ws_ml, ws_o, ws_cnt, ctx);
  note_launches(1);
  return cudaGetLastError();
}
template <typename T, int D>
cudaError_t decode_g(const DecodeShape& s, const void* q, const void* kc, const void* vc,
                     const int32_t* idx, const float* gates, void* o, void* ws, const DevCtx& ctx,
                     cudaStream_t st) {
  switch (s.Hq / s.Hkv) {
    case 1: return decode_t<T, D, 1>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 2: return decode_t<T, D, 2>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 3: return decode_t<T, D, 3>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 4: return decode_t<T, D, 4>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 5: return decode_t<T, D, 5>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 6: return decode_t<T, D, 6>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 7: return decode_t<T, D, 7>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    case 8: return decode_t<T, D, 8>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

void decode_plan(DecodeShape& s) {
  // CTAs in one wave (148 SMs, two CTAs each). A sparse call's lists are
  // short (tens of blocks per (batch, KV head)): about 1.5 CTAs per SM gave
  // the shortest times there (fewer, longer CTAs pay less prologue and merge
  // per block; 1 and 2 per SM were slower for the Qwen3-14B 512K or the
  // Qwen3-4B 64K decode), and at most 16 splits per unit, so that they merge
  // inside one cluster. The dense comparison streams long lists, two per SM.
  // One CTA per SM with twice the stages was slower for both: each CTA's
  // S -> softmax -> PV chain, not the bytes in flight, sets the pace.
  const int nslots = s.dense ? s.C + 1 : s.K + 1;
  const int units = s.B * s.Hkv;
  const int target = s.dense ? 2 * 148 : 3 * 148 / 2;
  int splits = target / units;
  splits = max(1, min(splits, min(nslots, s.dense ? kMaxSplits : 16)));
  int bps = (nslots + splits - 1) / splits;
  splits = (nslots + bps - 1) / bps;
  s.splits = splits;
  s.bps = bps;
  s.cluster = false;
}

size_t decode_workspace_bytes(const DecodeShape& s) {
  const size_t parts = (size_t)s.B * s.Hq * s.splits;
  const size_t a = (2 * parts * sizeof(float) + 255) & ~(size_t)255;
  const size_t b = (parts * s.d * sizeof(float) + 255) & ~(size_t)255;
  const size_t c = ((size_t)s.B * s.Hkv * sizeof(uint32_t) + 255) & ~(size_t)255;
  return a + b + c;
}

// ---------------------------------------------------------------------------
// Scratch for decode calls that must not allocate: a fixed array in device
// memory, present on every device that loads the library until the process
// exits. Its address is looked up once per device (with that device current);
// in host code the array's name is only a host-side handle, never a pointer
// the GPU can use.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];
std::mutex g_scratch_mu;
constexpr int kMaxScratchDevices = 64;
void* g_scratch_ptr[kMaxScratchDevices] = {nullptr};
}  // namespace

size_t decode_noalloc_capacity() { return kNoAllocScratchBytes; }

cudaError_t decode_noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

cudaError_t launch_decode(sas_dtype_t dt, const DecodeShape& s, const void* q, const void* kc,
                          const void* vc, const int32_t* idx, const float* gates, void* o,
                          void* ws, const DevCtx& ctx, cudaStream_t st) {
  if (tc_decode_supported(dt, s)) return launch_decode_tc(s, q, kc, vc, idx, gates, o, ws, ctx, st);
  if (dt == SAS_F32) {
    if (s.d == 64) return decode_g<float, 64>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
    return decode_g<float, 128>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
  }
  if (s.d == 64) return decode_g<__nv_bfloat16, 64>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
  return decode_g<__nv_bfloat16, 128>(s, q, kc, vc, idx, gates, o, ws, ctx, st);
}

}  // namespace sas
