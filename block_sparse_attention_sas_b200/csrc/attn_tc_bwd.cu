// Gated block-sparse causal attention, backward, on the sm_100a tensor cores
// (bf16 inputs, fp32 accumulation; head dim 128, block size 64, G = 2 or 4).
//
// Chain rule through Eq. 9 of the picx.dev SAS summary (Methodology), with
// P = exp(q.k * scale + log g - lse) recomputed from the forward's lse:
//   dP = dO V^T,  D_i = sum_t P_it dP_it,  dS = P * (dP - D),
//   dq = scale dS K,  dk = scale dS^T q,  dv = P^T dO,
//   da(j,m) = sum of dS over the (query block j, key block m) tile, all G
//   heads -- equal to g_m * dg_m of Eq. 5 (Gradient Analysis, inner form) --
//   which the gate Jacobian of Eq. 6 then turns into d scores.
// D is summed exactly from P and dP (a first sweep of kernel A) instead of
// dO . o from the stored bf16 o, whose rounding would reach every gradient.
//
// Kernel A (query-outer), one CTA per (query block j, 128-row tile of two
//   heads, KV head, batch): sweep 1 over the attended blocks sums D; sweep 2
//   forms dS, accumulates dQ += dS K in TMEM (K read as an MN-major operand)
//   and the tile's sum of dS per selected block; writes dq, D and da.
// Kernel B (key-outer), one CTA per (key block m, KV head, batch): over the
//   diagonal block and every query block whose selection holds m (a reverse
//   index), per 128-row tile: S = Q K^T and dP = dO V^T into TMEM, P and dS
//   into swizzled shared memory, then dV^T += dO^T P and dK^T += Q^T dS with
//   the Q / dO tiles read again as MN-major operands (no transposes).
// Warp roles as in the forward: warp 0 TMA producer, warp 1 MMA issuer,
// warps 4-7 the elementwise work, one thread per tile row. Waits are bounded.
#include <math.h>

#include "sas_internal.h"
#include "tc_common.cuh"

namespace sas {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kB = 64;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxList = 257;

// ============================================================================
// Kernel A: dq, D, da
// ============================================================================
namespace ka {
constexpr int kStages = 3;              // K/V ring depth
constexpr uint32_t kOffQ = 0;            // [k half][128 rows][128 B]
constexpr uint32_t kOffDO = 32768;       // same layout
constexpr uint32_t kOffKV = 65536;       // kStages x (K halves, V halves) 32 KB
constexpr uint32_t kOffDS = kOffKV + kStages * 32768;  // 2 buffers x [128 rows][128 B]
constexpr uint32_t kOffCtl = kOffDS + 32768;
struct Ctl {
  uint64_t qdo_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_free[2], ds_full[2],
      dq_done[2], drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxList], slots[kMaxList];
  float bias[kMaxList];
  float red[kMaxList][4];  // per-warp partial sums of dS per block
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
// TMEM columns: S[b] at 64 b, dP[b] at 128 + 64 b, dQ at 256.
}  // namespace ka

template <int TILES>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const float* __restrict__ lse, const int32_t* __restrict__ idx,
                 const float* __restrict__ gates, AttnShape s, __nv_bfloat16* __restrict__ dq,
                 float* __restrict__ Dv, float* __restrict__ da, DevCtx ctx) {
  using namespace ka;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, kvh = blockIdx.y / TILES, u = blockIdx.y % TILES, bi = blockIdx.z;
  const int G = 2 * TILES;
  const int h0 = kvh * G + 2 * u;  // the tile's two heads: h0, h0 + 1
  const long long irow = ((long long)(bi * s.Hkv + kvh) * s.N + j);

  if (tid == 0) {
    mbar_init(&c.qdo_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&c.kv_full[i], 1);
      mbar_init(&c.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_free[i], 128);
      mbar_init(&c.ds_full[i], 128);
      mbar_init(&c.dq_done[i], 1);
    }
    mbar_init(&c.drain, 1);
    fence_mbar_init();
    c.abort = 0;
    // Q and dO do not depend on the selection: start their loads first.
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    mbar_arrive_expect_tx(&c.qdo_full, 2 * 4 * 8192);
    for (int hh = 0; hh < 2; ++hh)
      for (int kb = 0; kb < 2; ++kb) {
        tma_load_3d(base + kOffQ + kb * 16384 + hh * 8192, &tm_q, kb * 64, j * kB,
                    bi * s.Hq + h0 + hh, &c.qdo_full);
        tma_load_3d(base + kOffDO + kb * 16384 + hh * 8192, &tm_do, kb * 64, j * kB,
                    bi * s.Hq + h0 + hh, &c.qdo_full);
      }
  }
  if (warp == 0) {
    // Attended blocks: the selected history blocks in slot order, then block j.
    __syncwarp();
    const int n = warp_build_list(idx + irow * s.K, gates ? gates + irow * s.N : nullptr, s.K, j,
                                  0, c.blocks, c.slots, c.bias, ctx);
    if (lane == 0) {
      c.blocks[n] = j;
      c.slots[n] = -1;
      c.bias[n] = 0.f;
      c.nblk = n + 1;
    }
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
  const int nit = 2 * nblk;  // sweep 1 then sweep 2 over the same blocks
  volatile int* abort = &c.abort;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int it = 0; it < nit; ++it) {
        const int st = it % kStages;
        if (it >= kStages &&
            !wait_or_abort(ctx, &c.kv_empty[st], ((it - kStages) / kStages) & 1, abort))
          break;
        const int m = c.blocks[it % nblk];
        unsigned char* kv = base + kOffKV + st * 32768;
        mbar_arrive_expect_tx(&c.kv_full[st], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, bi * s.Hkv + kvh, &c.kv_full[st]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, bi * s.Hkv + kvh,
                      &c.kv_full[st]);
        }
        issued = it + 1;
      }
      if (*abort) {
        (void)mbar_wait(ctx, &c.qdo_full, 0);
        for (int it = max(0, issued - kStages); it < issued; ++it)
          (void)mbar_wait(ctx, &c.kv_full[it % kStages], (it / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_q = idesc_bf16(128, 128, false, true);
      bool ok = wait_or_abort(ctx, &c.qdo_full, 0, abort);
      fence_after_sync();
      auto issue_s = [&](int it) -> bool {
        const int st = it % kStages, b = it & 1;
        if (!wait_or_abort(ctx, &c.kv_full[st], (it / kStages) & 1, abort)) return false;
        if (it >= 2 && !wait_or_abort(ctx, &c.s_free[b], ((it - 2) >> 1) & 1, abort)) return false;
        fence_after_sync();
        const uint32_t kva = sbase + kOffKV + st * 32768;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + b * 64, sdesc_sw128(sbase + kOffQ + ao, 16, 1024),
                      sdesc_sw128(kva + bo, 16, 1024), id_s, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 128 + b * 64, sdesc_sw128(sbase + kOffDO + ao, 16, 1024),
                      sdesc_sw128(kva + 16384 + bo, 16, 1024), id_s, ks > 0);
        }
        mma_commit(&c.s_full[b]);
        if (it < nblk) mma_commit(&c.kv_empty[st]);  // sweep 1 only reads S and dP
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int it = 0; ok && it < nit; ++it) {
        if (it + 1 < nit && !issue_s(it + 1)) break;
        if (it < nblk) continue;
        const int i2 = it - nblk, st = it % kStages;
        if (!wait_or_abort(ctx, &c.ds_full[i2 & 1], (i2 >> 1) & 1, abort)) break;
        fence_after_sync();
        const uint32_t dsa = sbase + kOffDS + (i2 & 1) * 16384;
        const uint32_t ka_ = sbase + kOffKV + st * 32768;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem + 256, sdesc_sw128(dsa + ks * 32, 16, 1024),
                      sdesc_sw128(ka_ + ks * 2048, 8192, 1024), id_q, (i2 > 0 || ks > 0));
        mma_commit(&c.dq_done[i2 & 1]);
        mma_commit(&c.kv_empty[st]);
      }
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int rowi = quarter * 32 + lane;
    const int hh = rowi >> 6, r = rowi & 63;
    const int head = h0 + hh;
    const int qrow = j * kB + r;
    const bool live = qrow < s.T;
    const long long hrow = (long long)(bi * s.Hq + head) * s.T + qrow;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const float lse2 = live ? lse[hrow] * kLog2e : 0.f;
    float Dsum = 0.f;
    bool ok = true;
    for (int it = 0; it < nit; ++it) {
      const int b = it & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(ctx, &c.s_full[b], (it >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int n = it % nblk;
      const int m = c.blocks[n];
      const float bias = c.bias[n];
      const bool cur = (n == nblk - 1);
      const int kvalid = min(kB, s.T - m * kB);
      const bool sweep2 = it >= nblk;
      uint32_t sr[64], pr[64];
      tmem_ld32(tl + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tl + 128 + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld32(tl + 128 + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
      fence_before_sync();
      mbar_arrive(&c.s_free[b]);
      if (cur || kvalid < kB) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= kvalid || (cur && i > r)) sr[i] = __float_as_uint(-INFINITY);
      }
      // p = 2^(s*scale + bias - lse2); rows past the sequence contribute nothing.
      const uint64_t sc2 = f2u(sc, sc);
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off);
      uint32_t pk[32];
      uint64_t acc0 = 0, acc1 = 0;
      const uint64_t negD = f2u(-Dsum, -Dsum);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                  sc2, off2);
        const uint64_t p2 = f2u(ex2(lo_f(a2)), ex2(hi_f(a2)));
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        if (!sweep2) {
          if (i & 1) acc1 = ffma2(p2, dp2, acc1);
          else acc0 = ffma2(p2, dp2, acc0);
        } else {
          const uint64_t ds2 = fmul2(p2, fadd2(dp2, negD));
          if (i & 1) acc1 = fadd2(acc1, ds2);
          else acc0 = fadd2(acc0, ds2);
          pk[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
        }
      }
      const uint64_t accs = fadd2(acc0, acc1);
      if (!sweep2) {
        Dsum += lo_f(accs) + hi_f(accs);
        continue;
      }
      const float rowsum = lo_f(accs) + hi_f(accs);
      const int i2 = it - nblk;
      // dS buffer (i2 & 1) is free once dQ(i2 - 2) has completed.
      if (i2 >= 2 && !__all_sync(0xffffffffu, wait_or_abort(ctx, &c.dq_done[i2 & 1],
                                                            ((i2 - 2) >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      unsigned char* drow = base + kOffDS + (i2 & 1) * 16384 + rowi * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(drow + ((ch ^ (rowi & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      fence_before_sync();
      mbar_arrive(&c.ds_full[i2 & 1]);
      if (!cur) {
        const float t = warp_sum(rowsum);
        if (lane == 0) c.red[n][quarter] = t;
      }
    }
    if (ok) {
      const int nl = nblk - 1;
      if (__all_sync(0xffffffffu,
                     wait_or_abort(ctx, &c.dq_done[nl & 1], (nl >> 1) & 1, abort))) {
        fence_after_sync();
        __nv_bfloat16* drow = dq + hrow * kD;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tl + 256 + ch * 32, ov);
          tmem_ld_wait();
          if (live) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(ov[8 * q4 + 0]) * s.scale, __uint_as_float(ov[8 * q4 + 1]) * s.scale);
              v.y = pack_bf16(__uint_as_float(ov[8 * q4 + 2]) * s.scale, __uint_as_float(ov[8 * q4 + 3]) * s.scale);
              v.z = pack_bf16(__uint_as_float(ov[8 * q4 + 4]) * s.scale, __uint_as_float(ov[8 * q4 + 5]) * s.scale);
              v.w = pack_bf16(__uint_as_float(ov[8 * q4 + 6]) * s.scale, __uint_as_float(ov[8 * q4 + 7]) * s.scale);
              *reinterpret_cast<uint4*>(drow + ch * 32 + q4 * 8) = v;
            }
          }
        }
        if (live) Dv[hrow] = Dsum;
      }
    }
    // da of each selected block: the four warps' partials in a fixed order.
    // Every softmax warp reaches this barrier, whichever path it took.
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (da != nullptr && !*abort) {
      for (int n = rowi; n < nblk - 1; n += 128) {
        const float t = (c.red[n][0] + c.red[n][1]) + (c.red[n][2] + c.red[n][3]);
        const long long o0 = (((long long)(bi * s.Hq + h0)) * s.N + j) * s.K + c.slots[n];
        da[o0] = t;
        da[o0 + (long long)s.N * s.K] = 0.f;  // head h0 + 1: the tile's sum sits on h0
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ============================================================================
// Kernel B: dk, dv
// ============================================================================
namespace kb_ {
constexpr uint32_t kOffK = 0;         // [d half][64 rows][128 B]
constexpr uint32_t kOffV = 16384;
constexpr uint32_t kOffQD = 32768;    // 2 stages x (Q tile 32 KB, dO tile 32 KB)
constexpr uint32_t kOffP = 163840;    // [128 rows][128 B]
constexpr uint32_t kOffDS = 180224;
constexpr uint32_t kOffCtl = 196608;
struct Ctl {
  uint64_t kv_full, qdo_full[2], qdo_empty[2], s_full[2], s_free[2], pds_full, pds_free, acc_done,
      drain;
  uint32_t tmem_base;
  int abort;
  // Per stage, staged by the producer warp with the Q/dO tiles: the step's
  // query block, its log2-domain gate bias, and lse / D of the tile's rows.
  int step_j[2];
  float step_bias[2];
  float lse2[2][128], D[2][128];
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
// TMEM columns: S[b] at 64 b, dP[b] at 128 + 64 b, dV^T at 256, dK^T at 320.
}  // namespace kb_

template <int TILES>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ lse,
                   const float* __restrict__ Dv, const float* __restrict__ gates,
                   const int32_t* __restrict__ csr_off, const int32_t* __restrict__ csr_list,
                   AttnShape s, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                   DevCtx ctx) {
  using namespace kb_;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = blockIdx.x, kvh = blockIdx.y, bi = blockIdx.z;
  const int G = 2 * TILES;
  const int bh = bi * s.Hkv + kvh;
  const int lo = csr_off[(long long)bh * (s.N + 1) + m];
  const int nl = csr_off[(long long)bh * (s.N + 1) + m + 1] - lo;
  const int32_t* lst = csr_list + (long long)bh * s.N * s.K + lo;
  const int nsteps = (1 + nl) * TILES;
  // Step s covers tile (s % TILES) of query block j(s): first the diagonal
  // block m, then the selecting blocks in ascending order.
  auto qblock = [&](int st) -> int {
    const int jj = st / TILES;
    return jj == 0 ? m : lst[jj - 1] / s.K;
  };

  if (tid == 0) {
    mbar_init(&c.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.qdo_full[i], 2);  // tiles (expect_tx) + staged scalars
      mbar_init(&c.qdo_empty[i], 1);
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_free[i], 128);
    }
    mbar_init(&c.pds_full, 128);
    mbar_init(&c.pds_free, 1);
    mbar_init(&c.acc_done, 1);
    mbar_init(&c.drain, 1);
    fence_mbar_init();
    c.abort = 0;
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort = &c.abort;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&c.kv_full, 32768);
      for (int h2 = 0; h2 < 2; ++h2) {
        tma_load_3d(base + kOffK + h2 * 8192, &tm_k, h2 * 64, m * kB, bh, &c.kv_full);
        tma_load_3d(base + kOffV + h2 * 8192, &tm_v, h2 * 64, m * kB, bh, &c.kv_full);
      }
    }
    int issued = 0;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int stg = st_i & 1;
      bool go = true;
      if (lane == 0 && st_i >= 2)
        go = wait_or_abort(ctx, &c.qdo_empty[stg], ((st_i - 2) >> 1) & 1, abort);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      const int j = qblock(st_i), u = st_i % TILES;
      if (lane == 0) {
        unsigned char* qd = base + kOffQD + stg * 65536;
        mbar_arrive_expect_tx(&c.qdo_full[stg], 65536);
        for (int hh = 0; hh < 2; ++hh)
          for (int kb = 0; kb < 2; ++kb) {
            const int plane = bi * s.Hq + kvh * G + 2 * u + hh;
            tma_load_3d(qd + kb * 16384 + hh * 8192, &tm_q, kb * 64, j * kB, plane,
                        &c.qdo_full[stg]);
            tma_load_3d(qd + 32768 + kb * 16384 + hh * 8192, &tm_do, kb * 64, j * kB, plane,
                        &c.qdo_full[stg]);
          }
      }
      // Scalars of the step: every lane stages 4 rows of lse (log2 domain) and D.
      for (int rr = lane; rr < 128; rr += 32) {
        const int head = kvh * G + 2 * u + (rr >> 6), qrow = j * kB + (rr & 63);
        const bool live = qrow < s.T;
        const long long hrow = (long long)(bi * s.Hq + head) * s.T + qrow;
        c.lse2[stg][rr] = live ? lse[hrow] * kLog2e : 0.f;
        c.D[stg][rr] = live ? Dv[hrow] : 0.f;
      }
      if (lane == 0) {
        c.step_j[stg] = j;
        c.step_bias[stg] = (j == m || gates == nullptr)
                               ? 0.f
                               : logf(gates[((long long)bh * s.N + j) * s.N + m]) * kLog2e;
      }
      __threadfence_block();
      __syncwarp();
      // The consumers see the staged scalars once this stage's Q/dO tiles
      // have landed: the arrival below is part of the same barrier phase.
      if (lane == 0) mbar_arrive(&c.qdo_full[stg]);
      issued = st_i + 1;
    }
    if (lane == 0 && *abort) {
      (void)mbar_wait(ctx, &c.kv_full, 0);
      for (int st_i = max(0, issued - 2); st_i < issued; ++st_i)
        (void)mbar_wait(ctx, &c.qdo_full[st_i & 1], (st_i >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_t = idesc_bf16(128, 64, true, true);
      bool ok = wait_or_abort(ctx, &c.kv_full, 0, abort);
      fence_after_sync();
      auto issue_s = [&](int st_i) -> bool {
        const int stg = st_i & 1, b = st_i & 1;
        if (!wait_or_abort(ctx, &c.qdo_full[stg], (st_i >> 1) & 1, abort)) return false;
        if (st_i >= 2 && !wait_or_abort(ctx, &c.s_free[b], ((st_i - 2) >> 1) & 1, abort))
          return false;
        fence_after_sync();
        const uint32_t qa = sbase + kOffQD + stg * 65536;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + b * 64, sdesc_sw128(qa + ao, 16, 1024),
                      sdesc_sw128(sbase + kOffK + bo, 16, 1024), id_s, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 128 + b * 64, sdesc_sw128(qa + 32768 + ao, 16, 1024),
                      sdesc_sw128(sbase + kOffV + bo, 16, 1024), id_s, ks > 0);
        }
        mma_commit(&c.s_full[b]);
        return true;
      };
      // dV^T[d][key] += sum_q dO[q][d] P[q][key]; dK^T[d][key] += sum_q Q[q][d] dS[q][key]
      auto retire = [&](int st_i) {
        fence_after_sync();
        const uint32_t qa = sbase + kOffQD + (st_i & 1) * 65536;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + 256, sdesc_sw128(qa + 32768 + ks * 2048, 16384, 1024),
                      sdesc_sw128(sbase + kOffP + ks * 2048, 8192, 1024), id_t,
                      (st_i > 0 || ks > 0));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + 320, sdesc_sw128(qa + ks * 2048, 16384, 1024),
                      sdesc_sw128(sbase + kOffDS + ks * 2048, 8192, 1024), id_t,
                      (st_i > 0 || ks > 0));
        mma_commit(&c.pds_free);
        mma_commit(&c.qdo_empty[st_i & 1]);
      };
      if (ok) ok = issue_s(0);
      // Order by readiness: the next step's S/dP go first when its Q/dO tile
      // has landed (they then overlap this step's softmax); otherwise this
      // step's dV/dK go first, which frees the stage that the load after the
      // next one is waiting for.
      for (int st_i = 0; ok && st_i < nsteps; ++st_i) {
        const int nxt = st_i + 1;
        bool next_issued = nxt >= nsteps;
        bool retired = false;
        for (unsigned long long polls = 0; ok && !retired; ++polls) {
          if (!next_issued && mbar_try_wait(&c.qdo_full[nxt & 1], (nxt >> 1) & 1)) {
            if (!issue_s(nxt)) ok = false;
            next_issued = true;
          }
          if (ok && mbar_try_wait(&c.pds_full, st_i & 1)) {
            retire(st_i);
            retired = true;
          } else if (polls >= ctx.wait_limit) {
            report(ctx, kDevErrTimeout);
            *abort = 1;
            ok = false;
          } else if ((polls & 63) == 63 && *abort) {
            ok = false;
          }
        }
        if (ok && !next_issued && !issue_s(nxt)) ok = false;
      }
      mma_commit(&c.acc_done);
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int rowi = quarter * 32 + lane;  // tile row (query) / d index in the epilogue
    const int r = rowi & 63;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const int kvalid = min(kB, s.T - m * kB);
    bool ok = true;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int b = st_i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(ctx, &c.s_full[b], (st_i >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int stg = st_i & 1;
      const int j = c.step_j[stg];
      const int qrow = j * kB + r;
      const bool live = qrow < s.T;
      const float lse2 = c.lse2[stg][rowi];
      const float Di = c.D[stg][rowi];
      const bool cur = (j == m);
      const float bias = c.step_bias[stg];
      uint32_t sr[64], pr[64], pp[32], dd[32];
      tmem_ld32(tl + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tl + 128 + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld32(tl + 128 + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
      fence_before_sync();
      mbar_arrive(&c.s_free[b]);
      if (cur || kvalid < kB) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= kvalid || (cur && i > r)) sr[i] = __float_as_uint(-INFINITY);
      }
      const uint64_t sc2 = f2u(sc, sc);
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off), negD = f2u(-Di, -Di);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                  sc2, off2);
        const float p0 = ex2(lo_f(a2)), p1 = ex2(hi_f(a2));
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        const uint64_t ds2 = fmul2(f2u(p0, p1), fadd2(dp2, negD));
        pp[i] = pack_bf16(p0, p1);
        dd[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
      }
      // The P / dS buffers are free once step st_i - 1's dV/dK MMAs completed.
      if (st_i >= 1 && !__all_sync(0xffffffffu,
                                   wait_or_abort(ctx, &c.pds_free, (st_i - 1) & 1, abort))) {
        ok = false;
        break;
      }
      unsigned char* prow = base + kOffP + rowi * 128;
      unsigned char* drow = base + kOffDS + rowi * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t sw = (ch ^ (rowi & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pp[4 * ch], pp[4 * ch + 1],
                                                          pp[4 * ch + 2], pp[4 * ch + 3]);
        *reinterpret_cast<uint4*>(drow + sw) = make_uint4(dd[4 * ch], dd[4 * ch + 1],
                                                          dd[4 * ch + 2], dd[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      fence_before_sync();
      mbar_arrive(&c.pds_full);
    }
    if (ok && __all_sync(0xffffffffu, wait_or_abort(ctx, &c.acc_done, 0, abort))) {
      // Epilogue: thread rowi holds dimension d = rowi of all 64 keys.
      fence_after_sync();
      const int d = rowi;
      const long long kb0 = ((long long)bh * s.T + (long long)m * kB) * kD;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = which == 0 ? dv : dk;
        const float mul = which == 0 ? 1.f : s.scale;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld32(tl + 256 + which * 64 + half * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = half * 32 + i;
            if (key < kvalid) out[kb0 + (long long)key * kD + d] =
                __float2bfloat16_rn(__uint_as_float(v[i]) * mul);
          }
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
}

}  // namespace

bool tc_bwd_supported(sas_dtype_t dt, const AttnShape& s) {
  const int G = s.Hq / s.Hkv;
  return dt == SAS_BF16 && s.d == kD && s.b == kB && (G == 2 || G == 4) && !s.dense;
}

cudaError_t launch_attn_bwd_tc(const AttnShape& s, const void* q, const void* k, const void* v,
                               const float* lse, const void* dO, const int32_t* idx,
                               const float* gates, void* dq, void* dk, void* dv, float* dscores,
                               void* ws, const DevCtx& ctx, cudaStream_t st) {
  const BwdWorkspace L = bwd_workspace_layout(s);
  char* w = static_cast<char*>(ws);
  float* Dv = reinterpret_cast<float*>(w + L.off_D);
  float* da = reinterpret_cast<float*>(w + L.off_da);
  int32_t* coff = reinterpret_cast<int32_t*>(w + L.off_csr_off);
  int32_t* clist = reinterpret_cast<int32_t*>(w + L.off_csr_list);
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tq, q, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tdo, dO, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, s.T, s.B * s.Hkv)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, s.T, s.B * s.Hkv)) != cudaSuccess) return e;
  if ((e = launch_bwd_csr(s, idx, coff, clist, ctx, st)) != cudaSuccess) return e;
  const int G = s.Hq / s.Hkv;
  const int tiles = G / 2;
  {
    dim3 grid(s.N, s.Hkv * tiles, s.B);
    auto kern = tiles == 2 ? tc_bwd_dq_kernel<2> : tc_bwd_dq_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ka::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, ka::kSmem, st>>>(tq, tk, tv, tdo, lse, idx, gates, s,
                                            (__nv_bfloat16*)dq, Dv, dscores ? da : nullptr, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    dim3 grid(s.N, s.Hkv, s.B);
    auto kern = tiles == 2 ? tc_bwd_dkdv_kernel<2> : tc_bwd_dkdv_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kb_::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kb_::kSmem, st>>>(tq, tk, tv, tdo, lse, Dv, gates, coff, clist, s,
                                             (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dscores) return launch_bwd_jacobian(s, da, idx, gates, dscores, st);
  return cudaSuccess;
}

}  // namespace sas
