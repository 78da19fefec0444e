// One-token decode on the sm_100a tensor cores (bf16 cache, head dim 128,
// block size 64, up to 8 query heads per KV head): the selected history
// blocks plus the current block, with or without the log-gate bias (picx.dev
// SAS summary, Methodology Eq. 9; evolve.pub review, Summary: hard selection
// kept at inference), and the dense decode (every block) used as comparison.
//
// The G query rows of a (batch, KV head) form the A operand of a 128-row MMA
// tile: an 8-row Q box (2 KB) read with a zero stride between 8-row groups,
// so all 16 row groups see the same rows (rows past G are never read),
// so each 64-key K/V block costs one S = Q K^T (8 MMAs, N = 64) and one
// O_n = P V (4 MMAs, N = 128): the CUDA cores only run the softmax of G rows,
// and the kernel streams the cache at HBM speed instead of FMA speed.
//
// One CTA per (split, KV head, batch); a split is a run of block slots.
//   warp 2  list of the split's blocks, TMA producer: Q once, then K and V of
//           each block into a three-stage ring (32 KB a stage)
//   warp 1  MMA issuer: S(n+1) is issued before PV(n) so the softmax of block
//           n overlaps the next QK^T
//   warp 0  softmax, one thread per query row (TMEM lane): masks keys past
//           the cache length, P as bf16 back into the S columns of TMEM (the
//           A operand of PV). O accumulates in TMEM over the blocks against a
//           per-row reference max: P = 2^(s * scale + bias - m_ref) stays
//           below 2^8 and O is rescaled in TMEM only when a row max rises
//           past that, so the softmax of block n + 1 never waits for PV(n)
// TMEM: S[2] at columns 0 / 64, O at 128 (256 columns, so two CTAs share an
// SM). Cache rows past L lie outside the tensor map and are read as zeros.
// Partial (max, sum, o) of each split go to the workspace; the last CTA of a
// (batch, KV head), found with an atomic ticket, merges them by log-sum-exp.
// Every wait is bounded.
#include <math.h>

#include "sas_internal.h"
#include "tc_common.cuh"

namespace sas {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kB = 64;
constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kSoftmaxWarp = 0;  // TMEM lanes 0..31 (warp % 4 == 0)
constexpr int kProducerWarp = 2;
constexpr uint32_t kTmemCols = 256;
constexpr int kMaxG = 8;
constexpr int kMaxSlotsPerSplit = 512;

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kStages = 3;
constexpr uint32_t kOffQ = 0;           // [k half][8 rows][128 B]
constexpr uint32_t kOffKV = 2048;       // stages x (K halves 16 KB, V halves 16 KB)
constexpr uint32_t kOffCtl = kOffKV + kStages * 32768;
constexpr uint32_t kColS = 0, kColO = 128;

struct Ctl {
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], p_full[2], o_full, o_final,
      drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxSlotsPerSplit];
  float bias[kMaxSlotsPerSplit];  // log2-domain gate bias
  float wgt[kMaxG * 64];          // merge weights of the last CTA
  float lsum[kMaxG];
  int last;
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;

template <int G>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ idx,
                 const float* __restrict__ gates, DecodeShape s, __nv_bfloat16* __restrict__ o,
                 float* __restrict__ ws_ml, float* __restrict__ ws_o, uint32_t* __restrict__ ws_cnt,
                 DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, bi = blockIdx.z;
  const int unit = bi * s.Hkv + kvh;
  const int nslots = s.dense ? s.C + 1 : s.K + 1;
  const int sl0 = split * s.bps, sl1 = min(nslots, sl0 + s.bps);
  const long long hbase = (long long)bi * s.Hq + kvh * G;  // first q head of the unit
  volatile int* abort = &c.abort;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      mbar_init(&c.q_full, 1);
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&c.kv_full[i], 1);
        mbar_init(&c.kv_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.s_full[i], 1);
        mbar_init(&c.p_full[i], 1);
      }
      mbar_init(&c.o_full, 1);
      mbar_init(&c.o_final, 1);
      mbar_init(&c.drain, 1);
      fence_mbar_init();
      c.abort = 0;
      c.last = 0;
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(&c.q_full, 2 * 1024);
      for (int kb = 0; kb < 2; ++kb)
        tma_load_3d(base + kOffQ + kb * 1024, &tm_q, kb * 64, (int)hbase, 0, &c.q_full);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    // The split's blocks in slot order: selected history blocks (bias log g
    // when gates are on), then the current block C; empty slots are skipped.
    const int32_t* ix = s.dense ? nullptr : idx + (long long)unit * s.K;
    int n = 0;
    for (int sb = sl0; sb < sl1; sb += 32) {
      const int sl = sb + lane;
      int m = -1;
      float bias = 0.f;
      if (sl < sl1) {
        if (s.dense || sl == s.K) {
          m = s.dense ? sl : s.C;
        } else {
          m = ix[sl];
          if (m >= s.C || m < -1) {
            report(ctx, kDevErrBadIndex);
            m = -1;
          } else if (m >= 0 && s.use_gates) {
            bias = log2f(gates[(long long)unit * s.C + m]);
          }
        }
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, m >= 0);
      if (m >= 0) {
        const int pos = n + __popc(mask & ((1u << lane) - 1u));
        c.blocks[pos] = m;
        c.bias[pos] = bias;
      }
      n += __popc(mask);
    }
    if (lane == 0) c.nblk = n;
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  const int nblk = c.nblk;
  const long long plane = unit;  // (batch, kv head) plane of the cache maps

  float m_run = -INFINITY, l_run = 0.f;
  float acc[kD];
  bool ok_sm = true;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int n = 0; n < nblk; ++n) {
        const int st = n % kStages;
        if (n >= kStages &&
            !wait_or_abort(ctx, &c.kv_empty[st], ((n - kStages) / kStages) & 1, abort))
          break;
        const int m = c.blocks[n];
        unsigned char* kv = base + kOffKV + st * 32768;
        mbar_arrive_expect_tx(&c.kv_full[st], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, (int)plane, &c.kv_full[st]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, (int)plane, &c.kv_full[st]);
        }
        issued = n + 1;
      }
      // The Q copy lands before the CTA leaves, even when the split is empty.
      (void)mbar_wait(ctx, &c.q_full, 0);
      if (*abort)
        for (int n = max(0, issued - kStages); n < issued; ++n)
          (void)mbar_wait(ctx, &c.kv_full[n % kStages], (n / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && nblk > 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_o = idesc_bf16(128, 128, false, true);
      const uint64_t dq0 = sdesc_sw128(sbase + kOffQ, 16, 0);  // 8 rows, repeated
      const uint64_t dk0 = sdesc_sw128(sbase + kOffKV, 16, 1024);     // K, K-major
      const uint64_t dv0 = sdesc_sw128(sbase + kOffKV + 16384, 8192, 1024);  // V, MN-major
      auto issue_s = [&](int n) -> bool {
        const int st = n % kStages, sb = n & 1;
        if (!wait_or_abort(ctx, &c.kv_full[st], (n / kStages) & 1, abort)) return false;
        fence_after_sync();
        const uint64_t kd = dk0 + ((st * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = ((ks >> 2) * 8192 + (ks & 3) * 32) >> 4;
          mma_bf16_ss(tmem + kColS + sb * 64, dq0 + ((((ks >> 2) * 1024 + (ks & 3) * 32)) >> 4),
                      kd + off, id_s, ks > 0);
        }
        mma_commit(&c.s_full[sb]);
        return true;
      };
      bool ok = wait_or_abort(ctx, &c.q_full, 0, abort) && issue_s(0);
      for (int n = 0; ok && n < nblk; ++n) {
        const int st = n % kStages, sb = n & 1;
        if (n + 1 < nblk && !issue_s(n + 1)) break;
        if (!wait_or_abort(ctx, &c.p_full[sb], (n >> 1) & 1, abort)) break;
        fence_after_sync();
        // O += P(n) V(n): P in S[n & 1] columns 0..31 (two bf16 per column);
        // block 0 starts O.
        const uint64_t vd = dv0 + ((st * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ts(tmem + kColO, tmem + kColS + sb * 64 + ks * 8, vd + ((ks * 2048) >> 4), id_o,
                      n > 0 || ks > 0);
        mma_commit(&c.o_full);
        mma_commit(&c.kv_empty[st]);
      }
      mma_commit(&c.o_final);  // O complete: every PV issued above is done
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp == kSoftmaxWarp) {
    // Thread `lane` owns query row `lane` of the tile (head lane < G).
    constexpr float kLazy = 8.f;  // log2 headroom of P over the reference max
    const float sc = s.scale * kLog2e;
    const uint32_t tl = tmem;  // lanes 0..31
    for (int n = 0; n < nblk; ++n) {
      const int st = n & 1;
      if (!warp_wait(ctx, &c.s_full[st], (n >> 1) & 1, abort)) {
        ok_sm = false;
        break;
      }
      fence_after_sync();
      const int m = c.blocks[n];
      const float bias = c.bias[n];
      const int kvalid = min(kB, s.L - m * kB);
      // Two passes over the two 32-column halves of S: the row max first,
      // then p = 2^(s*scale + bias - m_ref) as bf16 into the S columns
      // already read (P(n) takes columns 0..31).
      float smax = -INFINITY;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sr[32];
        tmem_ld32(tl + kColS + st * 64 + hf * 32, sr);
        tmem_ld_wait();
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const bool v0 = hf * 32 + i < kvalid, v1 = hf * 32 + i + 1 < kvalid;
          const bool v2 = hf * 32 + i + 2 < kvalid, v3 = hf * 32 + i + 3 < kvalid;
          m0 = fmax3(m0, v0 ? __uint_as_float(sr[i]) : -INFINITY,
                     v1 ? __uint_as_float(sr[i + 1]) : -INFINITY);
          m1 = fmax3(m1, v2 ? __uint_as_float(sr[i + 2]) : -INFINITY,
                     v3 ? __uint_as_float(sr[i + 3]) : -INFINITY);
        }
        smax = fmax3(smax, m0, m1);
      }
      const float mx = (smax == -INFINITY) ? -INFINITY : fmaf(smax, sc, bias);
      // Reference update: the first finite max sets it (nothing accumulated
      // for the row yet); a max more than kLazy above it rescales O.
      const bool need = lane < G && m_run != -INFINITY && mx > m_run + kLazy;
      if (m_run == -INFINITY) m_run = mx;
      if (__any_sync(0xffffffffu, need)) {
        // O must hold every PV issued so far. Seeing S(n) complete already
        // implies PV(n - 2) completed, so waiting for the parity of PV(n - 1)
        // is unambiguous.
        if (n >= 1 && !warp_wait(ctx, &c.o_full, (n - 1) & 1, abort)) {
          ok_sm = false;
          break;
        }
        fence_after_sync();
        const float alpha = need ? ex2(m_run - mx) : 1.f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ov[32], lo16[16], hi16[16];
          tmem_ld32(tl + kColO + ch * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            lo16[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            hi16[i] = __float_as_uint(__uint_as_float(ov[16 + i]) * alpha);
          }
          tmem_st16(tl + kColO + ch * 32, lo16);
          tmem_st16(tl + kColO + ch * 32 + 16, hi16);
        }
        l_run *= alpha;
        if (need) m_run = mx;
      }
      const float off = (m_run == -INFINITY) ? -INFINITY : bias - m_run;
      const uint64_t sc2 = f2u(sc, sc), off2 = f2u(off, off);
      uint64_t accp = 0;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sr[32], pk[16];
        tmem_ld32(tl + kColS + st * 64 + hf * 32, sr);
        tmem_ld_wait();
        if (kvalid < kB) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (hf * 32 + i >= kvalid) sr[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t a = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                   sc2, off2);
          const float p0 = ex2(lo_f(a)), p1 = ex2(hi_f(a));
          accp = fadd2(accp, f2u(p0, p1));
          pk[i] = pack_bf16(p0, p1);
        }
        tmem_st16(tl + kColS + st * 64 + hf * 16, pk);
      }
      l_run += lo_f(accp) + hi_f(accp);
      // P(n) (and a rescaled O) in TMEM before PV(n) is issued.
      tmem_st_wait();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.p_full[st]);
    }
#pragma unroll
    for (int i = 0; i < kD; ++i) acc[i] = 0.f;
    if (ok_sm && nblk > 0) {
      if (!warp_wait(ctx, &c.o_final, 0, abort)) {
        ok_sm = false;
      } else {
        fence_after_sync();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tl + kColO + ch * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[ch * 32 + i] = __uint_as_float(ov[i]);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (*abort) return;

  // ---- this split's partial: row `lane` of the softmax warp is head lane < G
  if (warp == kSoftmaxWarp && ok_sm && lane < G) {
    const long long h = hbase + lane;
    if (s.splits == 1) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = o + h * kD;
#pragma unroll
      for (int q4 = 0; q4 < kD / 8; ++q4) {
        uint4 v;
        v.x = pack_bf16(acc[8 * q4 + 0] * inv, acc[8 * q4 + 1] * inv);
        v.y = pack_bf16(acc[8 * q4 + 2] * inv, acc[8 * q4 + 3] * inv);
        v.z = pack_bf16(acc[8 * q4 + 4] * inv, acc[8 * q4 + 5] * inv);
        v.w = pack_bf16(acc[8 * q4 + 6] * inv, acc[8 * q4 + 7] * inv);
        *reinterpret_cast<uint4*>(orow + 8 * q4) = v;
      }
    } else {
      const long long pidx = h * s.splits + split;
      float4* dst = reinterpret_cast<float4*>(ws_o + pidx * kD);
#pragma unroll
      for (int q4 = 0; q4 < kD / 4; ++q4)
        dst[q4] = make_float4(acc[4 * q4], acc[4 * q4 + 1], acc[4 * q4 + 2], acc[4 * q4 + 3]);
      ws_ml[2 * pidx] = m_run;  // log2 domain
      ws_ml[2 * pidx + 1] = l_run;
    }
  }
  if (s.splits == 1) return;

  // ---- the last CTA of the unit merges the partials by log-sum-exp
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t ticket = atomicAdd(&ws_cnt[unit], 1u);
    c.last = (ticket == (uint32_t)(s.splits - 1));
  }
  __syncthreads();
  if (!c.last) return;
  __threadfence();
  const int P = s.splits;
  for (int g = warp; g < G; g += kWarps) {
    float M = -INFINITY;
    for (int x = lane; x < P; x += 32) M = fmaxf(M, __ldcg(&ws_ml[2 * ((hbase + g) * P + x)]));
    M = warp_max(M);
    float Lsum = 0.f;
    for (int x = lane; x < P; x += 32) {
      const float mx = __ldcg(&ws_ml[2 * ((hbase + g) * P + x)]);
      const float f = (mx == -INFINITY) ? 0.f : ex2(mx - M);
      Lsum += f * __ldcg(&ws_ml[2 * ((hbase + g) * P + x) + 1]);
      c.wgt[g * 64 + x] = f;
    }
    Lsum = warp_sum(Lsum);
    if (lane == 0) c.lsum[g] = Lsum;
  }
  __syncthreads();
  for (int e = tid; e < G * (kD / 4); e += kThreads) {
    const int g = e / (kD / 4), d4 = e % (kD / 4);
    const float4* src = reinterpret_cast<const float4*>(ws_o + (hbase + g) * P * kD) + d4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int x = 0; x < P; ++x) {
      const float4 v = __ldcg(src + (size_t)x * (kD / 4));
      const float f = c.wgt[g * 64 + x];
      a.x = fmaf(f, v.x, a.x);
      a.y = fmaf(f, v.y, a.y);
      a.z = fmaf(f, v.z, a.z);
      a.w = fmaf(f, v.w, a.w);
    }
    const float inv = c.lsum[g] > 0.f ? 1.f / c.lsum[g] : 0.f;
    __nv_bfloat16* dst = o + (hbase + g) * kD + d4 * 4;
    uint2 pk;
    pk.x = pack_bf16(a.x * inv, a.y * inv);
    pk.y = pack_bf16(a.z * inv, a.w * inv);
    *reinterpret_cast<uint2*>(dst) = pk;
  }
}

template <int G>
cudaError_t launch_g(const DecodeShape& s, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, const int32_t* idx, const float* gates, void* o,
                     float* ws_ml, float* ws_o, uint32_t* ws_cnt, const DevCtx& ctx,
                     cudaStream_t st) {
  auto kern = decode_tc_kernel<G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(s.splits, s.Hkv, s.B);
  kern<<<grid, kThreads, kSmem, st>>>(tq, tk, tv, idx, gates, s, (__nv_bfloat16*)o, ws_ml, ws_o,
                                      ws_cnt, ctx);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool tc_decode_supported(sas_dtype_t dt, const DecodeShape& s) {
  const int G = s.Hq / s.Hkv;
  return dt == SAS_BF16 && s.d == kD && s.b == kB && G >= 1 && G <= kMaxG && s.splits <= 64 &&
         s.bps <= kMaxSlotsPerSplit;
}

cudaError_t launch_decode_tc(const DecodeShape& s, const void* q, const void* kc, const void* vc,
                             const int32_t* idx, const float* gates, void* o, void* ws,
                             const DevCtx& ctx, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  // q as [B*Hq rows][128]; the cache as [B*Hkv planes][L rows][128] with a
  // plane pitch of Lcap rows, so rows past L read as zeros.
  if ((e = make_tmap_bf16_rows8(&tq, q, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_pitched(&tk, kc, s.L, s.Lcap, s.B * s.Hkv)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_pitched(&tv, vc, s.L, s.Lcap, s.B * s.Hkv)) != cudaSuccess) return e;
  char* w = static_cast<char*>(ws);
  const size_t parts = (size_t)s.B * s.Hq * s.splits;
  float* ws_ml = reinterpret_cast<float*>(w);
  float* ws_o = reinterpret_cast<float*>(w + ((2 * parts * sizeof(float) + 255) & ~(size_t)255));
  uint32_t* ws_cnt = reinterpret_cast<uint32_t*>(
      reinterpret_cast<char*>(ws_o) + ((parts * s.d * sizeof(float) + 255) & ~(size_t)255));
  if (s.splits > 1) {
    // Tickets start at zero on every call, whatever the workspace held before.
    e = cudaMemsetAsync(ws_cnt, 0, sizeof(uint32_t) * (size_t)s.B * s.Hkv, st);
    if (e != cudaSuccess) return e;
    note_launches(1);
  }
  switch (s.Hq / s.Hkv) {
    case 1: return launch_g<1>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 2: return launch_g<2>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 3: return launch_g<3>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 4: return launch_g<4>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 5: return launch_g<5>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 6: return launch_g<6>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 7: return launch_g<7>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    case 8: return launch_g<8>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, ctx, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sas
