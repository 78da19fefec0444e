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
// D is summed exactly from P and dP instead of taken as dO . o from the
// stored bf16 o, whose rounding would reach every gradient.
//
// Three kernels, run in this order after the reverse index (for each key
// block, the query blocks that selected it) and a launch order:
//   tc_bwd_d_kernel (query-outer), one CTA per (query block j, 128-row tile
//     of two heads, KV head, batch): S = Q K^T and dP = dO V^T per attended
//     block, D_i = sum_t P_it dP_it; writes D.
//   tc_bwd_dkdv_kernel (key-outer), one CTA per (key block m, KV head,
//     batch): over the diagonal block and every query block whose selection
//     holds m, per 128-row tile: S and dP into TMEM, P and dS into swizzled
//     shared memory, then dV^T += dO^T P and dK^T += Q^T dS with the Q / dO
//     tiles read again as MN-major operands (no transposes). It writes dk,
//     dv, every dS tile (bf16, 16 KB) to the workspace, and the tile's sum of
//     dS per selected block (da) in eight fixed shares.
//   tc_bwd_dq_kernel (query-outer), one CTA per (query block, 128-row tile,
//     KV head, batch): dq = scale * sum over the attended blocks of dS K from
//     the stored tiles; no recomputation.
// The gate Jacobian (a separate small kernel) turns da into d scores.
// OUTER (outer gating, the ablation variant): P recomputed from the
// ungated lse is the gated weight g p, so D and dV need no change; dS =
// g p (dP - D / g) and da sums g p dP (Eq. 5, outer form, times g).
// Every result comes from one CTA in a fixed order: no atomics, so the
// gradients are deterministic. Warp roles: a TMA producer warp, one MMA
// issuing thread, elementwise warps with one thread per tile row (TMEM
// lane). Every wait is bounded.
#include <math.h>

#include "sas_internal.h"
#include "tc_common.cuh"

namespace sas {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kB = 64;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxList = 257;

// ============================================================================
// Kernel D: D_i = sum over the attended keys of P_it dP_it, summed exactly
// rather than taken as dO . o: the forward's o is stored in bf16, and its
// rounding (up to 2^-9 |o|) would reach every gradient through D.
// ============================================================================
// One CTA per (query block j, 128-row tile of two heads, KV head, batch),
// two CTAs per SM (256 TMEM columns, 97 KB of shared memory), so one CTA's
// prologue and bubbles are filled by the other's MMAs. Q (through a 32 KB
// staging buffer) and dO (through the second K/V stage, before its first
// use) land together and are copied into TMEM (the A operand of every S / dP
// MMA); K/V blocks stream through a two-stage ring. The S/dP accumulators are
// single-buffered: the full barrier of K/V block n also takes one arrival
// per elementwise warp once it has read S/dP(n-1), so the MMA thread waits
// once per block. S and dP have separate commits, so P is formed while the
// dP MMAs run.
namespace kd {
constexpr int kThreadsD = 256;   // warp 0 producer + list, warp 1 MMA, warps 4-7 rows
constexpr uint32_t kTmemColsD = 256;
constexpr uint32_t kColQ = 0, kColDO = 64, kColS = 128, kColDP = 192;
constexpr uint32_t kOffStage = 0;       // Q: [k half][128 rows][128 B]; dO in KV stage 1
constexpr uint32_t kOffKV = 32768;      // 2 stages x (K halves, V halves)
constexpr uint32_t kOffCtl = kOffKV + 2 * 32768;
struct Ctl {
  uint64_t qd_full, qd_free, kv_full[2], kv_empty[2], s_full, dp_full, drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxList];
  float bias[kMaxList];
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
}  // namespace kd

template <int TILES>
__global__ void __launch_bounds__(kd::kThreadsD, 2)
tc_bwd_d_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const float* __restrict__ lse, const int32_t* __restrict__ idx,
                const float* __restrict__ gates, AttnShape s, float* __restrict__ Dv, DevCtx ctx) {
  using namespace kd;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The longest query blocks first (in the dense comparison, every history
  // block), so the short ones fill the last wave.
  const int j = s.N - 1 - (int)blockIdx.x;
  const int kvh = blockIdx.y / TILES, u = blockIdx.y % TILES, bi = blockIdx.z;
  const int G = 2 * TILES;
  const int h0 = kvh * G + 2 * u;  // the tile's two heads: h0, h0 + 1
  const long long irow = ((long long)(bi * s.Hkv + kvh) * s.N + j);
  volatile int* abort = &c.abort;
  // Block n of the list: the selected blocks then j; dense: 0 .. j.
  auto blk = [&](int n) -> int { return s.dense ? n : c.blocks[n]; };

  const int quarter = warp & 3;
  const int rowi = quarter * 32 + lane;
  const int r = rowi & 63;
  const int qrow = j * kB + r;
  const bool live = qrow < s.T;
  const long long hrow = (long long)(bi * s.Hq + h0 + (rowi >> 6)) * s.T + qrow;
  float lse2 = 0.f;
  if (warp >= 4 && live) lse2 = lse[hrow] * kLog2e;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&c.qd_full, 1);
      mbar_init(&c.qd_free, 4);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.kv_full[i], 5);  // expect-tx arrival + one per elementwise warp
        mbar_init(&c.kv_empty[i], 1);
      }
      mbar_init(&c.s_full, 1);
      mbar_init(&c.dp_full, 1);
      mbar_init(&c.drain, 1);
      fence_mbar_init();
      c.abort = 0;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      // Q into the staging buffer and dO into K/V stage 1, one phase.
      mbar_arrive_expect_tx(&c.qd_full, 8 * 8192);
      for (int h2 = 0; h2 < 2; ++h2)
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(base + kOffStage + kb * 16384 + h2 * 8192, &tm_q, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qd_full);
          tma_load_3d(base + kOffKV + 32768 + kb * 16384 + h2 * 8192, &tm_do, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qd_full);
        }
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    __syncwarp();
    int n = j;
    if (!s.dense) {
      n = warp_build_list(idx + irow * s.K, gates ? gates + irow * s.N : nullptr, s.K, j, 0,
                          c.blocks, nullptr, c.bias, ctx);
      if (lane == 0) {
        c.blocks[n] = j;
        c.bias[n] = 0.f;
      }
    }
    if (lane == 0) c.nblk = n + 1;
    __syncwarp();
    if (lane == 0) {
      for (; issued < n + 1 && issued < 1; ++issued) {  // stage 1 holds dO until it is in TMEM
        const int m = blk(issued);
        unsigned char* kv = base + kOffKV + issued * 32768;
        mbar_arrive_expect_tx(&c.kv_full[issued], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, bi * s.Hkv + kvh, &c.kv_full[issued]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, bi * s.Hkv + kvh,
                      &c.kv_full[issued]);
        }
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemColsD);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  const int nblk = c.nblk;

  if (warp == 0) {
    if (lane == 0) {
      // Block 1 goes into stage 1 once dO has moved from there into TMEM.
      bool go = wait_or_abort(ctx, &c.qd_free, 0, abort);
      for (int n = issued; go && n < nblk; ++n) {
        const int st = n & 1;
        if (n >= 2 && !wait_or_abort(ctx, &c.kv_empty[st], ((n - 2) >> 1) & 1, abort)) break;
        const int m = blk(n);
        unsigned char* kv = base + kOffKV + st * 32768;
        mbar_arrive_expect_tx(&c.kv_full[st], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, bi * s.Hkv + kvh, &c.kv_full[st]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, bi * s.Hkv + kvh,
                      &c.kv_full[st]);
        }
        issued = n + 1;
      }
      // The Q / dO copies land before the CTA leaves.
      (void)mbar_wait(ctx, &c.qd_full, 0);
      if (*abort)
        for (int n = max(0, issued - 2); n < issued; ++n)
          (void)mbar_wait(ctx, &c.kv_full[n & 1], (n >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint64_t dkv0 = sdesc_sw128(sbase + kOffKV, 16, 1024);
      bool ok = true;
      for (int n = 0; n < nblk; ++n) {
        const int st = n & 1;
        if (!wait_or_abort(ctx, &c.kv_full[st], (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        fence_after_sync();
        const uint64_t kd = dkv0 + ((st * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColS, tmem + kColQ + ks * 8,
                      kd + (((ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
        mma_commit(&c.s_full);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColDP, tmem + kColDO + ks * 8,
                      kd + ((16384 + (ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
        mma_commit(&c.dp_full);
        mma_commit(&c.kv_empty[st]);
      }
      (void)ok;
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const uint64_t sc2 = f2u(sc, sc);
    // Q (staging buffer) and dO (K/V stage 1) into this row's TMEM lane.
    bool ok = warp_wait(ctx, &c.qd_full, 0, abort);
    if (ok) {
      tile_row_to_tmem(base + kOffStage, rowi, tl + kColQ);
      tile_row_to_tmem(base + kOffKV + 32768, rowi, tl + kColDO);
      tmem_st_wait();
    }
    fence_before_sync();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&c.qd_free);     // stage 1 may take block 1
      mbar_arrive(&c.kv_full[0]);  // Q, dO in TMEM: S/dP(0) may start
    }
    float Dsum = 0.f;
    for (int n = 0; ok && n < nblk; ++n) {
      if (!warp_wait(ctx, &c.s_full, n & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int m = blk(n);
      const float bias = s.dense ? 0.f : c.bias[n];
      const bool cur = (n == nblk - 1);
      const int kvalid = min(kB, s.T - m * kB);
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off);
      // P from S while the dP MMAs run.
      uint64_t p2[32];
      {
        uint32_t sr[64];
        tmem_ld32(tl + kColS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tl + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        if (cur || kvalid < kB) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= kvalid || (cur && i > r)) sr[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                    sc2, off2);
          // A quarter of the exponentials on the FMA pipe (MUFU-bound phase).
          p2[i] = ((i & 3) == 3) ? ex2_poly2(a2) : f2u(ex2(lo_f(a2)), ex2(hi_f(a2)));
        }
      }
      if (!warp_wait(ctx, &c.dp_full, n & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pr[32];
        tmem_ld32(tl + kColDP + hf * 32, pr);
        tmem_ld_wait();
        if (hf == 1) {
          // S/dP(n) are in registers: S/dP(n + 1) may overwrite the accumulators.
          fence_before_sync();
          __syncwarp();
          if (lane == 0 && n + 1 < nblk) mbar_arrive(&c.kv_full[(n + 1) & 1]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
          if (i & 1) acc1 = ffma2(p2[hf * 16 + i], dp2, acc1);
          else acc0 = ffma2(p2[hf * 16 + i], dp2, acc0);
        }
      }
      const uint64_t accs = fadd2(acc0, acc1);
      Dsum += lo_f(accs) + hi_f(accs);
    }
    if (ok && live) Dv[hrow] = Dsum;
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemColsD);
  }
}

// ============================================================================
// Kernel R: dq with S and dP recomputed, for problems whose dS tiles are not
// kept (the dense comparison, where they would take B*Hkv*N*N*(G/2)*16 KB).
// ============================================================================
// One CTA per (query block j, 128-row tile of two heads, KV head, batch),
// laid out as the D kernel: Q and dO are copied into TMEM (the A operand of
// S and dP), K/V stream through a two-stage ring. Per block: S and dP into
// TMEM; the elementwise warps form dS = P (dP - D) as bf16 in a swizzled
// shared tile; dQ += dS K (four M=128 N=128 MMAs, K read as an MN-major
// operand) accumulates in TMEM, and the block's stage is freed once those
// MMAs are done. The epilogue scales dQ and stores it.
namespace kr {
constexpr int kThreadsR = 256;   // warp 0 producer + list, warp 1 MMA, warps 4-7 rows
constexpr uint32_t kTmemColsR = 512;
constexpr uint32_t kColQ = 0, kColDO = 64, kColS = 128, kColDP = 192, kColDQ = 256;
constexpr uint32_t kOffStage = 0;       // Q: [k half][128 rows][128 B]; dO in KV stage 1
constexpr uint32_t kOffKV = 32768;      // 2 stages x (K halves, V halves)
constexpr uint32_t kOffDS = kOffKV + 2 * 32768;  // dS: [128 rows][128 B]
constexpr uint32_t kOffCtl = kOffDS + 16384;
struct Ctl {
  uint64_t qd_full, qd_free, kv_full[2], kv_empty[2], s_full, dp_full, ds_full, ds_free, dq_done,
      drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxList];
  float bias[kMaxList];
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
}  // namespace kr

template <int TILES>
__global__ void __launch_bounds__(kr::kThreadsR, 1)
tc_bwd_dq_recompute_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ lse,
                           const float* __restrict__ Dv, const int32_t* __restrict__ idx,
                           const float* __restrict__ gates, AttnShape s,
                           __nv_bfloat16* __restrict__ dq, DevCtx ctx) {
  using namespace kr;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = s.N - 1 - (int)blockIdx.x;  // longest query blocks first
  const int kvh = blockIdx.y / TILES, u = blockIdx.y % TILES, bi = blockIdx.z;
  const int G = 2 * TILES;
  const int h0 = kvh * G + 2 * u;
  const long long irow = ((long long)(bi * s.Hkv + kvh) * s.N + j);
  volatile int* abort = &c.abort;
  auto blk = [&](int n) -> int { return s.dense ? n : c.blocks[n]; };

  const int quarter = warp & 3;
  const int rowi = quarter * 32 + lane;
  const int r = rowi & 63;
  const int qrow = j * kB + r;
  const bool live = qrow < s.T;
  const long long hrow = (long long)(bi * s.Hq + h0 + (rowi >> 6)) * s.T + qrow;
  float lse2 = 0.f, Di = 0.f;
  if (warp >= 4 && live) {
    lse2 = lse[hrow] * kLog2e;
    Di = Dv[hrow];
  }

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&c.qd_full, 1);
      mbar_init(&c.qd_free, 4);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.kv_full[i], 5);  // expect-tx arrival + one per elementwise warp
        mbar_init(&c.kv_empty[i], 1);
      }
      mbar_init(&c.s_full, 1);
      mbar_init(&c.dp_full, 1);
      mbar_init(&c.ds_full, 4);
      mbar_init(&c.ds_free, 1);
      mbar_init(&c.dq_done, 1);
      mbar_init(&c.drain, 1);
      fence_mbar_init();
      c.abort = 0;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&c.qd_full, 8 * 8192);
      for (int h2 = 0; h2 < 2; ++h2)
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(base + kOffStage + kb * 16384 + h2 * 8192, &tm_q, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qd_full);
          tma_load_3d(base + kOffKV + 32768 + kb * 16384 + h2 * 8192, &tm_do, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qd_full);
        }
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    __syncwarp();
    int n = j;
    if (!s.dense) {
      n = warp_build_list(idx + irow * s.K, gates ? gates + irow * s.N : nullptr, s.K, j, 0,
                          c.blocks, nullptr, c.bias, ctx);
      if (lane == 0) {
        c.blocks[n] = j;
        c.bias[n] = 0.f;
      }
    }
    if (lane == 0) c.nblk = n + 1;
    __syncwarp();
    if (lane == 0) {
      for (; issued < n + 1 && issued < 1; ++issued) {  // stage 1 holds dO until it is in TMEM
        const int m = blk(issued);
        unsigned char* kv = base + kOffKV + issued * 32768;
        mbar_arrive_expect_tx(&c.kv_full[issued], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, bi * s.Hkv + kvh, &c.kv_full[issued]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, bi * s.Hkv + kvh,
                      &c.kv_full[issued]);
        }
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemColsR);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  const int nblk = c.nblk;

  if (warp == 0) {
    if (lane == 0) {
      bool go = wait_or_abort(ctx, &c.qd_free, 0, abort);
      for (int n = issued; go && n < nblk; ++n) {
        const int st = n & 1;
        if (n >= 2 && !wait_or_abort(ctx, &c.kv_empty[st], ((n - 2) >> 1) & 1, abort)) break;
        const int m = blk(n);
        unsigned char* kv = base + kOffKV + st * 32768;
        mbar_arrive_expect_tx(&c.kv_full[st], 32768);
        for (int h2 = 0; h2 < 2; ++h2) {
          tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, bi * s.Hkv + kvh, &c.kv_full[st]);
          tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, bi * s.Hkv + kvh,
                      &c.kv_full[st]);
        }
        issued = n + 1;
      }
      (void)mbar_wait(ctx, &c.qd_full, 0);
      if (*abort)
        for (int n = max(0, issued - 2); n < issued; ++n)
          (void)mbar_wait(ctx, &c.kv_full[n & 1], (n >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, 64, false, false);
      const uint32_t id_q = idesc_bf16(128, 128, false, true);
      const uint64_t dkv0 = sdesc_sw128(sbase + kOffKV, 16, 1024);
      const uint64_t dds0 = sdesc_sw128(sbase + kOffDS, 16, 1024);          // dS, K-major
      const uint64_t dkb0 = sdesc_sw128(sbase + kOffKV, 8192, 1024);        // K as MN-major B
      // S/dP of block n + 1 are issued as soon as the row warps hold S/dP(n)
      // in registers, so they run while dS(n) is formed.
      auto issue_sdp = [&](int n) -> bool {
        const int st = n & 1;
        if (!wait_or_abort(ctx, &c.kv_full[st], (n >> 1) & 1, abort)) return false;
        fence_after_sync();
        const uint64_t kd = dkv0 + ((st * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColS, tmem + kColQ + ks * 8,
                      kd + (((ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
        mma_commit(&c.s_full);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColDP, tmem + kColDO + ks * 8,
                      kd + ((16384 + (ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
        mma_commit(&c.dp_full);
        return true;
      };
      bool ok = nblk > 0 && issue_sdp(0);
      for (int n = 0; ok && n < nblk; ++n) {
        const int st = n & 1;
        if (n + 1 < nblk && !issue_sdp(n + 1)) break;
        if (!wait_or_abort(ctx, &c.ds_full, n & 1, abort)) break;
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem + kColDQ, dds0 + ((ks * 32) >> 4),
                      dkb0 + ((st * 32768 + ks * 2048) >> 4), id_q, (n > 0 || ks > 0));
        mma_commit(&c.ds_free);
        mma_commit(&c.kv_empty[st]);
      }
      mma_commit(&c.dq_done);
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const uint64_t sc2 = f2u(sc, sc);
    bool ok = warp_wait(ctx, &c.qd_full, 0, abort);
    if (ok) {
      tile_row_to_tmem(base + kOffStage, rowi, tl + kColQ);
      tile_row_to_tmem(base + kOffKV + 32768, rowi, tl + kColDO);
      tmem_st_wait();
    }
    fence_before_sync();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&c.qd_free);     // stage 1 may take block 1
      mbar_arrive(&c.kv_full[0]);  // Q, dO in TMEM: S/dP(0) may start
    }
    unsigned char* dsrow = base + kOffDS + rowi * 128;
    for (int n = 0; ok && n < nblk; ++n) {
      if (!warp_wait(ctx, &c.s_full, n & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int m = blk(n);
      const float bias = s.dense ? 0.f : c.bias[n];
      const bool cur = (n == nblk - 1);
      const int kvalid = min(kB, s.T - m * kB);
      const float dinv = s.outer ? fminf(ex2(-bias), 3.0e38f) : 1.f;
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off);
      float pf[64];
      {
        uint32_t sr[64];
        tmem_ld32(tl + kColS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tl + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        if (cur || kvalid < kB) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= kvalid || (cur && i > r)) sr[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                    sc2, off2);
          const uint64_t p2 = ((i & 3) == 3) ? ex2_poly2(a2) : f2u(ex2(lo_f(a2)), ex2(hi_f(a2)));
          pf[2 * i] = lo_f(p2);
          pf[2 * i + 1] = hi_f(p2);
        }
      }
      if (!warp_wait(ctx, &c.dp_full, n & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint32_t pr[64];
      tmem_ld32(tl + kColDP, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld32(tl + kColDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
      // S/dP(n) are in registers: S/dP(n + 1) may overwrite the accumulators.
      fence_before_sync();
      __syncwarp();
      if (lane == 0 && n + 1 < nblk) mbar_arrive(&c.kv_full[(n + 1) & 1]);
      uint32_t dd[32];
      const uint64_t negD = f2u(-Di * dinv, -Di * dinv);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        const uint64_t ds2 = fmul2(f2u(pf[2 * i], pf[2 * i + 1]), fadd2(dp2, negD));
        dd[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
      }
      // The dS tile is free once dQ(n - 1) has read it.
      if (n >= 1 && !warp_wait(ctx, &c.ds_free, (n - 1) & 1, abort)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(dsrow + ((ch ^ (rowi & 7)) << 4)) =
            make_uint4(dd[4 * ch], dd[4 * ch + 1], dd[4 * ch + 2], dd[4 * ch + 3]);
      fence_proxy_async_smem();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.ds_full);
    }
    if (ok && warp_wait(ctx, &c.dq_done, 0, abort)) {
      fence_after_sync();
      __nv_bfloat16* drow = dq + hrow * kD;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ov[32];
        tmem_ld32(tl + kColDQ + ch * 32, ov);
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
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemColsR);
  }
}

// ============================================================================
// Kernel Q: dq = scale * sum over the attended blocks of dS K, from the dS
// tiles the dK/dV kernel stored (no recomputation of S / dP)
// ============================================================================
// One CTA per (query block j, 128-row tile, KV head, batch), two CTAs per
// SM: each attended block brings its 16 KB dS tile and 16 KB K block through
// a three-stage TMA ring; dQ (128 x 128 fp32) accumulates in TMEM with four
// M=128 N=128 MMAs per block, in the block list's order.
namespace kq {
constexpr int kThreadsQ = 256;   // warp 0 producer + list, warp 1 MMA, warps 4-7 epilogue
constexpr uint32_t kTmemColsQ = 128;
constexpr int kStages = 3;
constexpr uint32_t kOffCtl = kStages * 32768;  // stage: dS tile 16 KB, then K halves
struct Ctl {
  uint64_t kv_full[kStages], kv_empty[kStages], dq_done, drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxList], slots[kMaxList];
  float bias[kMaxList];
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
}  // namespace kq

template <int TILES>
__global__ void __launch_bounds__(kq::kThreadsQ, 2)
tc_bwd_dq_kernel(const __nv_bfloat16* __restrict__ ds, const __grid_constant__ CUtensorMap tm_k,
                 const int32_t* __restrict__ idx, AttnShape s, __nv_bfloat16* __restrict__ dq,
                 DevCtx ctx) {
  using namespace kq;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(base);
  Ctl& c = *reinterpret_cast<Ctl*>(base + kOffCtl);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The longest query blocks (most attended blocks) start first, so the
  // short ones fill the last wave.
  const int j = s.N - 1 - (int)blockIdx.x;
  const int kvh = blockIdx.y / TILES, u = blockIdx.y % TILES, bi = blockIdx.z;
  const int G = 2 * TILES;
  const int h0 = kvh * G + 2 * u;
  const long long irow = ((long long)(bi * s.Hkv + kvh) * s.N + j);
  // dS tiles of this (query block, tile): plane index of slot sl.
  const long long plane0 = (irow * TILES + u) * (s.K + 1);
  volatile int* abort = &c.abort;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&c.kv_full[i], 1);
        mbar_init(&c.kv_empty[i], 1);
      }
      mbar_init(&c.dq_done, 1);
      mbar_init(&c.drain, 1);
      fence_mbar_init();
      c.abort = 0;
      tma_prefetch_desc(&tm_k);
    }
    __syncwarp();
    const int n = warp_build_list(idx + irow * s.K, nullptr, s.K, j, 0, c.blocks, c.slots, c.bias,
                                  ctx);
    if (lane == 0) {
      c.blocks[n] = j;
      c.slots[n] = s.K;  // the current block's tile sits after the K slots
      c.nblk = n + 1;
    }
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemColsQ);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  const int nblk = c.nblk;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int n = 0; n < nblk; ++n) {
        const int st = n % kStages;
        if (n >= kStages &&
            !wait_or_abort(ctx, &c.kv_empty[st], ((n - kStages) / kStages) & 1, abort))
          break;
        unsigned char* sb = base + st * 32768;
        mbar_arrive_expect_tx(&c.kv_full[st], 32768);
        bulk_g2s(sb, ds + (plane0 + c.slots[n]) * (128 * 64), 16384, &c.kv_full[st]);
        for (int h2 = 0; h2 < 2; ++h2)
          tma_load_3d(sb + 16384 + h2 * 8192, &tm_k, h2 * 64, c.blocks[n] * kB, bi * s.Hkv + kvh,
                      &c.kv_full[st]);
        issued = n + 1;
      }
      if (*abort)
        for (int n = max(0, issued - kStages); n < issued; ++n)
          (void)mbar_wait(ctx, &c.kv_full[n % kStages], (n / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_q = idesc_bf16(128, 128, false, true);
      const uint64_t dds0 = sdesc_sw128(sbase, 16, 1024);            // dS, K-major
      const uint64_t dk0 = sdesc_sw128(sbase + 16384, 8192, 1024);   // K as MN-major B
      for (int n = 0; n < nblk; ++n) {
        const int st = n % kStages;
        if (!wait_or_abort(ctx, &c.kv_full[st], (n / kStages) & 1, abort)) break;
        fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem, dds0 + ((st * 32768 + ks * 32) >> 4),
                      dk0 + ((st * 32768 + ks * 2048) >> 4), id_q, (n > 0 || ks > 0));
        mma_commit(&c.kv_empty[st]);
      }
      mma_commit(&c.dq_done);
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int rowi = quarter * 32 + lane;
    const int r = rowi & 63;
    const int qrow = j * kB + r;
    const long long hrow = (long long)(bi * s.Hq + h0 + (rowi >> 6)) * s.T + qrow;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    if (warp_wait(ctx, &c.dq_done, 0, abort)) {
      fence_after_sync();
      __nv_bfloat16* drow = dq + hrow * kD;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ov[32];
        tmem_ld32(tl + ch * 32, ov);
        tmem_ld_wait();
        if (qrow < s.T) {
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
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemColsQ);
  }
}

// ============================================================================
// Launch order of kernel B: the (batch, KV head, key block) units sorted by
// descending reverse-list length, so the longest CTAs start first and the
// short ones fill in behind them. Any order gives the same results (every
// unit's outputs come from one CTA); ties are left in whatever order the
// atomics produce.
// ============================================================================
__global__ void __launch_bounds__(1024)
order_kernel(const int32_t* __restrict__ off_all, AttnShape s, int32_t* __restrict__ order) {
  extern __shared__ int32_t hist[];  // N + 1 buckets (list length 0..N-1)
  const int U = s.B * s.Hkv * s.N;
  const int nb = s.N + 1;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int bh = u / s.N, m = u % s.N;
    const int len = off_all[(long long)bh * (s.N + 1) + m + 1] - off_all[(long long)bh * (s.N + 1) + m];
    atomicAdd(&hist[s.N - len], 1);  // bucket 0 holds the longest lists
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < nb; ++i) {
      const int c = hist[i];
      hist[i] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int bh = u / s.N, m = u % s.N;
    const int len = off_all[(long long)bh * (s.N + 1) + m + 1] - off_all[(long long)bh * (s.N + 1) + m];
    order[atomicAdd(&hist[s.N - len], 1)] = u;
  }
}

// ============================================================================
// Kernel B: dk, dv
// ============================================================================
// One CTA per (key block m, KV head, batch) steps over 128-row query tiles
// (the diagonal block's, then those of every query block that selected m).
// The MMA stream goes by pairs of steps: S/dP(s), S/dP(s + 1), dV/dK(s),
// dV/dK(s + 1). P/dS are double-buffered in shared memory, so while the
// elementwise warps turn S/dP(s + 1) into P/dS the tensor pipe runs dV/dK(s),
// and a Q/dO stage freed by dV/dK(s) reloads while dV/dK(s + 1) and the next
// S/dP run. Each hand-off has its own barrier, so a stage is refilled as
// soon as the MMAs that read it are done, whatever the dS store warp is
// doing.
namespace kb_ {
constexpr int kWarps = 12;
constexpr int kThreadsB = kWarps * 32;
// Tile offsets from the first 1024-byte boundary after the control block.
constexpr uint32_t kOffK = 0;         // [d half][64 rows][128 B]
constexpr uint32_t kOffV = 16384;
constexpr uint32_t kOffQD = 32768;    // 2 stages x (Q tile 32 KB, dO tile 32 KB)
constexpr uint32_t kOffPD = 163840;   // 2 buffers x (P [128 rows][128 B], dS at +16 KB)
constexpr uint32_t kTileBytes = 229376;
// TMEM columns: S[b] at 64 b, dP[b] at 128 + 64 b, dV^T at 256, dK^T at 320.
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320;
struct Ctl {
  // qdo_full[stg]: the producer's expect-tx arrival plus tile bytes, and its
  // arrival once the step's scalars are staged. s_full[b] / dp_full[b]: MMA
  // commits after S and after dP. pds_full[b]: one arrival per elementwise
  // warp once P/dS of the step are in buffer b; da_full[b]: the same once its
  // share of the tile sum of dS is in dapart. stage_free[b]: MMA commit after dV/dK of the step (the
  // Q/dO stage and its scalars may be refilled). buf_free[b]: the dS store
  // warp, once dV/dK of the step are done and it has copied dS out of
  // buffer b (the buffer and its scalars may be rewritten).
  uint64_t kv_full, qdo_full[2], s_full[2], dp_full[2], pds_full[2], da_full[2];
  uint64_t stage_free[2], buf_free[2];
  uint64_t acc_done, drain;
  uint32_t tmem_base;
  int abort;
  // Per stage, staged by the producer warp with the Q/dO tiles: the step's
  // query block, its log2-domain gate bias, and lse / D of the tile's rows.
  int step_j[2], step_slot[2];
  float step_bias[2];
  float lse2[2][128], D[2][128];
  // Per P/dS buffer, written by the elementwise warps for the store warp:
  // the step's query block and slot, and per-warp shares of its tile sum of dS.
  int buf_j[2], buf_slot[2];
  float dapart[2][8];
};
// The control block sits at the start of dynamic shared memory and the tiles
// at the next 1024-byte boundary. With a 1024-aligned base (the case when a
// kernel declares no static shared memory) this is exactly the 227 KB limit;
// the kernel checks the carve-out and reports kDevErrLayout otherwise.
constexpr uint32_t kCtlSpan = 3072;
static_assert(sizeof(Ctl) <= kCtlSpan, "control block outgrew its span");
constexpr size_t kSmem = kCtlSpan + kTileBytes;
static_assert(kSmem <= 232448, "over the per-block shared memory limit");
}  // namespace kb_

template <int TILES, bool OUTER>
__global__ void __launch_bounds__(kb_::kThreadsB, 1)
tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ lse,
                   const float* __restrict__ Dv, const float* __restrict__ gates,
                   const int32_t* __restrict__ csr_off, const int32_t* __restrict__ csr_list,
                   const int32_t* __restrict__ order, AttnShape s,
                   __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                   __nv_bfloat16* __restrict__ ds_out, float* __restrict__ da, DevCtx ctx) {
  using namespace kb_;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t tiles_off = ((raw + (uint32_t)sizeof(Ctl) + 1023u) & ~1023u) - raw;
  if (tiles_off + kTileBytes > kSmem) {  // uniform over the CTA: nothing started yet
    if (threadIdx.x == 0) report(ctx, kDevErrLayout);
    return;
  }
  Ctl& c = *reinterpret_cast<Ctl*>(smem_raw);
  unsigned char* base = smem_raw + tiles_off;
  const uint32_t sbase = smem_u32(base);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Dense: key block m is attended by every query block j >= m; the units
  // go longest list (smallest m) first without a reverse index.
  const int BH = s.B * s.Hkv;
  const int unit = s.dense ? 0 : order[blockIdx.x];
  const int m = s.dense ? (int)blockIdx.x / BH : unit % s.N;
  const int bh = s.dense ? (int)blockIdx.x % BH : unit / s.N;
  const int kvh = bh % s.Hkv, bi = bh / s.Hkv;
  const int G = 2 * TILES;
  const int lo = s.dense ? 0 : csr_off[(long long)bh * (s.N + 1) + m];
  const int nl = s.dense ? s.N - 1 - m : csr_off[(long long)bh * (s.N + 1) + m + 1] - lo;
  const int32_t* lst = s.dense ? nullptr : csr_list + (long long)bh * s.N * s.K + lo;
  const int nsteps = (1 + nl) * TILES;
  // Step s covers tile (s % TILES) of query block j(s): first the diagonal
  // block m, then the selecting blocks in ascending order (entry / K of the
  // reverse list is the query block).
  volatile int* abort = &c.abort;

  if (tid == 0) {
    mbar_init(&c.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.qdo_full[i], 2);
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.dp_full[i], 1);
      mbar_init(&c.pds_full[i], 8);
      mbar_init(&c.da_full[i], 8);
      mbar_init(&c.stage_free[i], 1);
      mbar_init(&c.buf_free[i], 1);
    }
    mbar_init(&c.acc_done, 1);
    mbar_init(&c.drain, 1);
    fence_mbar_init();
    c.abort = 0;
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    mbar_arrive_expect_tx(&c.kv_full, 32768);
    for (int h2 = 0; h2 < 2; ++h2) {
      tma_load_3d(base + kOffK + h2 * 8192, &tm_k, h2 * 64, m * kB, bh, &c.kv_full);
      tma_load_3d(base + kOffV + h2 * 8192, &tm_v, h2 * 64, m * kB, bh, &c.kv_full);
    }
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;

  if (warp == 0) {
    // Scalars of a step (lse in the log2 domain and D of the tile's 128 rows,
    // four per lane, the query block, its slot and its gate) are loaded into
    // registers two steps ahead (global loads are slow under this kernel's
    // traffic), so staging them costs only shared stores.
    struct Pre {
      float lse[4], D[4], bias;
      int j, slot;
    };
    // The reverse list in a register window (lane l holds entry win_lo + l),
    // with the next window already in flight.
    int win_lo = 0;
    int win = (lst && lane < nl) ? lst[lane] : 0;
    int win_next = (lst && 32 + lane < nl) ? lst[32 + lane] : 0;
    auto prefetch = [&](int st_i) -> Pre {
      Pre p;
      const int jj = st_i / TILES, u = st_i % TILES;
      int j = m, slot = s.K;  // the diagonal step's tile sits after the K slots
      if (jj > 0 && s.dense) {
        j = m + jj;
        slot = 0;
      } else if (jj > 0) {
        const int ix = jj - 1;
        while (ix >= win_lo + 32) {
          win = win_next;
          win_lo += 32;
          win_next = win_lo + 32 + lane < nl ? lst[win_lo + 32 + lane] : 0;
        }
        const int e = __shfl_sync(0xffffffffu, win, ix - win_lo);
        j = e / s.K;
        slot = e % s.K;
      }
      p.j = j;
      p.slot = slot;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int rr = lane + 32 * q4;
        const int head = kvh * G + 2 * u + (rr >> 6), qrow = j * kB + (rr & 63);
        const bool live = qrow < s.T;
        const long long hrow = (long long)(bi * s.Hq + head) * s.T + qrow;
        p.lse[q4] = live ? lse[hrow] : 0.f;
        p.D[q4] = live ? Dv[hrow] : 0.f;
      }
      p.bias = (j == m || gates == nullptr) ? 1.f : gates[((long long)bh * s.N + j) * s.N + m];
      return p;
    };
    Pre cur = prefetch(0);
    Pre nxt = nsteps > 1 ? prefetch(1) : cur;
    int issued = 0;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int stg = st_i & 1;
      bool go = true;
      // The stage is free once dV/dK of step st_i - 2 completed.
      if (lane == 0 && st_i >= 2)
        go = wait_or_abort(ctx, &c.stage_free[stg], ((st_i - 2) >> 1) & 1, abort);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      const int j = cur.j, u = st_i % TILES;
      if (lane == 0) {
        // One 64 x 64 x 2 box per k-half brings both heads' rows of the tile.
        unsigned char* qd = base + kOffQD + stg * 65536;
        const int plane = bi * s.Hq + kvh * G + 2 * u;
        mbar_arrive_expect_tx(&c.qdo_full[stg], 65536);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(qd + kb * 16384, &tm_q, kb * 64, j * kB, plane, &c.qdo_full[stg]);
          tma_load_3d(qd + 32768 + kb * 16384, &tm_do, kb * 64, j * kB, plane, &c.qdo_full[stg]);
        }
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        c.lse2[stg][lane + 32 * q4] = cur.lse[q4] * kLog2e;
        c.D[stg][lane + 32 * q4] = cur.D[q4];
      }
      if (lane == 0) {
        c.step_j[stg] = j;
        c.step_slot[stg] = cur.slot;
        c.step_bias[stg] = logf(cur.bias) * kLog2e;
      }
      // The arrival that completes this stage's phase also waits until the
      // store warp has released P/dS buffer st_i & 1 (step st_i - 2), so the
      // elementwise warps may write it as soon as S/dP of this step are done;
      // the wait overlaps the tile loads. The consumers see the staged
      // scalars once the phase completes: the warp's stores are ordered
      // before lane 0's (release) arrival by the warp barrier.
      if (lane == 0 && st_i >= 2)
        go = wait_or_abort(ctx, &c.buf_free[stg], ((st_i - 2) >> 1) & 1, abort);
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.qdo_full[stg]);
      issued = st_i + 1;
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      cur = nxt;
      if (st_i + 2 < nsteps) {
        nxt = prefetch(st_i + 2);
        // Under this kernel's load a stage's tiles take ~2000 cycles to land
        // from HBM, more than the MMAs between a stage's release and its next
        // use; pulling the tiles of step st_i + 2 into L2 now hides that.
        if (lane == 0) {
          const int plane2 = bi * s.Hq + kvh * G + 2 * ((st_i + 2) % TILES);
          for (int kb = 0; kb < 2; ++kb) {
            tma_prefetch_l2_3d(&tm_q, kb * 64, nxt.j * kB, plane2);
            tma_prefetch_l2_3d(&tm_do, kb * 64, nxt.j * kB, plane2);
          }
        }
      }
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
      const uint64_t dq0 = sdesc_sw128(sbase + kOffQD, 16, 1024);    // Q/dO stages, K-major
      const uint64_t dk0 = sdesc_sw128(sbase + kOffK, 16, 1024);     // K (V at +16 KB)
      const uint64_t dqt0 = sdesc_sw128(sbase + kOffQD, 16384, 1024);  // Q/dO as MN-major A
      const uint64_t dp0 = sdesc_sw128(sbase + kOffPD, 8192, 1024);  // P[b] (dS[b] at +16 KB)
      auto issue_sdp = [&](int st_i) {
        const int b = st_i & 1;
        const uint64_t qa = dq0 + ((b * 65536) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + kColS + b * 64, qa + (ao >> 4), dk0 + (bo >> 4), id_s, ks > 0);
        }
        mma_commit(&c.s_full[b]);  // P can be formed while dP runs
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = 16384 + (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + kColDP + b * 64, qa + (ao >> 4), dk0 + (bo >> 4), id_s, ks > 0);
        }
        mma_commit(&c.dp_full[b]);
      };
      // dV^T[d][key] += sum_q dO[q][d] P[q][key]; dK^T[d][key] += sum_q Q[q][d] dS[q][key]
      auto issue_dvdk = [&](int st_i) {
        const int b = st_i & 1;
        const uint64_t qa = dqt0 + ((b * 65536) >> 4);
        const uint64_t pa = dp0 + ((b * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + kColDV, qa + ((32768 + ks * 2048) >> 4), pa + ((ks * 2048) >> 4),
                      id_t, (st_i > 0 || ks > 0));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + kColDK, qa + ((ks * 2048) >> 4), pa + ((16384 + ks * 2048) >> 4),
                      id_t, (st_i > 0 || ks > 0));
        mma_commit(&c.stage_free[b]);
      };
      bool ok = wait_or_abort(ctx, &c.kv_full, 0, abort);
      for (int s0 = 0; ok && s0 < nsteps; s0 += 2) {
        const int npair = min(2, nsteps - s0);
        const uint32_t ph = (s0 >> 1) & 1;
        for (int e = 0; ok && e < npair; ++e) {
          if (!wait_or_abort(ctx, &c.qdo_full[e], ph, abort)) { ok = false; break; }
          fence_after_sync();
          issue_sdp(s0 + e);
        }
        for (int e = 0; ok && e < npair; ++e) {
          if (!wait_or_abort(ctx, &c.pds_full[e], ph, abort)) { ok = false; break; }
          fence_after_sync();
          issue_dvdk(s0 + e);
        }
      }
      mma_commit(&c.acc_done);
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp == 2) {
    // dS store warp: once P/dS of step s are in buffer s & 1, copy the raw
    // 16 KB dS tile (swizzled, as the dq kernel's MMA reads it) to the
    // workspace with the TMA engine and write the step's da shares; once the
    // copy has read the buffer and dV/dK of the step are done, its arrival
    // on buf_free lets the elementwise warps rewrite the buffer.
    if (lane == 0) {
      for (int st_i = 0; st_i < nsteps; ++st_i) {
        const int b = st_i & 1, u = st_i % TILES;
        const uint32_t ph = (st_i >> 1) & 1;
        if (!wait_or_abort(ctx, &c.pds_full[b], ph, abort)) break;
        const int j = c.buf_j[b], slot = c.buf_slot[b];
        const long long tile = (((long long)bh * s.N + j) * TILES + u) * (s.K + 1) + slot;
        if (ds_out != nullptr) {  // the dense comparison keeps no tiles
          bulk_s2g(ds_out + tile * (128 * 64), base + kOffPD + b * 32768 + 16384, 16384);
          bulk_commit();
        }
        if (da != nullptr && !wait_or_abort(ctx, &c.da_full[b], ph, abort)) break;
        if (da != nullptr && slot < s.K) {
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const int head = kvh * G + 2 * u + ((p & 3) >> 1), rc = (p >> 2) * 2 + (p & 1);
            da[(((long long)(bi * s.Hq + head) * s.N + j) * 4 + rc) * s.K + slot] = c.dapart[b][p];
          }
        }
        bulk_wait_read_all();
        if (!wait_or_abort(ctx, &c.stage_free[b], ph, abort)) break;
        mbar_arrive(&c.buf_free[b]);
      }
      bulk_wait_all();
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3, grp = (warp - 4) >> 2;
    const int rowi = quarter * 32 + lane;  // tile row (query) / d index in the epilogue
    const int r = rowi & 63;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const int kvalid = min(kB, s.T - m * kB) - 32 * grp;
    const uint64_t sc2 = f2u(sc, sc);
    bool ok = true;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int b = st_i & 1;
      if (!warp_wait(ctx, &c.s_full[b], (st_i >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int j = c.step_j[b];
      const int qrow = j * kB + r;
      const bool live = qrow < s.T;
      const float lse2 = c.lse2[b][rowi];
      const float Di = c.D[b][rowi];
      const bool cur = (j == m);
      const float bias = c.step_bias[b];
      // Buffer b is free: the producer's arrival in this step's Q/dO phase,
      // which S(st_i) waited for, came after the store warp released it.
      unsigned char* prow = base + kOffPD + b * 32768 + rowi * 128;
      unsigned char* drow = prow + 16384;
      float pf[32];
      {  // P = exp2(S * scale * log2 e + log2 gate - lse * log2 e), while dP is computed
        uint32_t sr[32], pp[16];
        tmem_ld32(tl + kColS + b * 64 + 32 * grp, sr);
        tmem_ld_wait();
        if (cur || kvalid < 32) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i >= kvalid || (cur && i + 32 * grp > r)) sr[i] = __float_as_uint(-INFINITY);
        }
        const float off = live ? bias - lse2 : -INFINITY;
        const uint64_t off2 = f2u(off, off);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                    sc2, off2);
          if ((i & 3) == 3) {  // a quarter of the exponentials on the FMA pipe
            const uint64_t e = ex2_poly2(a2);
            pf[2 * i] = lo_f(e);
            pf[2 * i + 1] = hi_f(e);
          } else {
            pf[2 * i] = ex2(lo_f(a2));
            pf[2 * i + 1] = ex2(hi_f(a2));
          }
          pp[i] = pack_bf16(pf[2 * i], pf[2 * i + 1]);
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint32_t sw = ((4 * grp + ch) ^ (rowi & 7)) << 4;
          *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pp[4 * ch], pp[4 * ch + 1],
                                                            pp[4 * ch + 2], pp[4 * ch + 3]);
        }
      }
      if (!warp_wait(ctx, &c.dp_full[b], (st_i >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      uint64_t dsum = 0;
      {  // dS = P (dP - D); outer gating: P (dP - D / g)
        uint32_t pr[32], dd[16];
        tmem_ld32(tl + kColDP + b * 64 + 32 * grp, pr);
        tmem_ld_wait();
        const float dinv = OUTER ? fminf(ex2(-bias), 3.0e38f) : 1.f;
        const uint64_t negD = f2u(-Di * dinv, -Di * dinv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
          const uint64_t p2 = f2u(pf[2 * i], pf[2 * i + 1]);
          const uint64_t ds2 = fmul2(p2, fadd2(dp2, negD));
          dsum = OUTER ? ffma2(p2, dp2, dsum) : fadd2(dsum, ds2);
          dd[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint32_t sw = ((4 * grp + ch) ^ (rowi & 7)) << 4;
          *reinterpret_cast<uint4*>(drow + sw) = make_uint4(dd[4 * ch], dd[4 * ch + 1],
                                                            dd[4 * ch + 2], dd[4 * ch + 3]);
        }
      }
      if (lane == 0 && warp == 4) {
        c.buf_j[b] = j;
        c.buf_slot[b] = c.step_slot[b];
      }
      fence_proxy_async_smem();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.pds_full[b]);
      {  // this warp's share of the tile sum of dS, for the store warp, off the MMA's path
        const float t = warp_sum(lo_f(dsum) + hi_f(dsum));
        if (lane == 0) {
          c.dapart[b][grp * 4 + quarter] = t;
          mbar_arrive(&c.da_full[b]);
        }
      }
    }
    // Epilogue: thread rowi holds dimension d = rowi; group grp the keys
    // 32 grp .. 32 grp + 31. The key block's dV and dK rows are contiguous
    // 16 KB ranges of dv and dk, so they are staged as [key][d] bf16 tiles in
    // the first Q/dO stage (no MMA reads it after acc_done, no load fills it)
    // and leave in two bulk copies. Every elementwise warp reaches the
    // barrier; the copies go only when no wait of the CTA gave up.
    unsigned char* st_dv = base + kOffQD;
    unsigned char* st_dk = base + kOffQD + 16384;
    if (ok && warp_wait(ctx, &c.acc_done, 0, abort)) {
      fence_after_sync();
      const int d = rowi;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(which == 0 ? st_dv : st_dk);
        const float mul = which == 0 ? 1.f : s.scale;
        uint32_t v[32];
        tmem_ld32(tl + (which == 0 ? kColDV : kColDK) + grp * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          t[(grp * 32 + i) * kD + d] = __float2bfloat16_rn(__uint_as_float(v[i]) * mul);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 32 * 8);
    if (warp == 4 && lane == 0 && *abort == 0) {
      const long long kb0 = ((long long)bh * s.T + (long long)m * kB) * kD;
      const uint32_t bytes = (uint32_t)min(kB, s.T - m * kB) * kD * 2;
      bulk_s2g(dv + kb0, st_dv, bytes);
      bulk_s2g(dk + kb0, st_dk, bytes);
      bulk_commit();
      bulk_wait_read_all();
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
  return dt == SAS_BF16 && s.d == kD && s.b == kB && (G == 2 || G == 4);
}

namespace {
// D_i = dO_i . (o_i + o_res_i) for every query row: one warp per row, four
// columns a lane, rows in the [B][Hq][T] order of the D array. With the
// forward's residual, o + o_res carries its fp32 output (P entered PV as two
// bf16 terms), so this is Sum_t P_it dP_it to fp32 rounding.
__global__ void __launch_bounds__(256)
d_from_o_kernel(const __nv_bfloat16* __restrict__ dO, const __nv_bfloat16* __restrict__ o,
                const __nv_bfloat16* __restrict__ o_res, long long rows, float* __restrict__ Dv) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const long long off = r * kD + lane * 4;
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(dO + off));
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(o + off));
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(o_res + off));
    auto lo = [](uint32_t x) { return __uint_as_float(x << 16); };
    auto hi = [](uint32_t x) { return __uint_as_float(x & 0xffff0000u); };
    float acc = lo(a.x) * (lo(b.x) + lo(c.x));
    acc = fmaf(hi(a.x), hi(b.x) + hi(c.x), acc);
    acc = fmaf(lo(a.y), lo(b.y) + lo(c.y), acc);
    acc = fmaf(hi(a.y), hi(b.y) + hi(c.y), acc);
    acc = warp_sum(acc);
    if (lane == 0) Dv[r] = acc;
  }
}

cudaError_t launch_d_from_o(const AttnShape& s, const void* dO, const void* o, const void* o_res,
                            float* Dv, cudaStream_t st) {
  const long long rows = (long long)s.B * s.Hq * s.T;
  const long long want = (rows + 7) / 8;
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  d_from_o_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)dO, (const __nv_bfloat16*)o,
                                        (const __nv_bfloat16*)o_res, rows, Dv);
  note_launches(1);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_attn_bwd_tc(const AttnShape& s, const void* q, const void* k, const void* v,
                               const void* o, const void* o_res, const float* lse, const void* dO,
                               const int32_t* idx, const float* gates, void* dq, void* dk, void* dv,
                               float* dscores, void* ws, const DevCtx& ctx, cudaStream_t st) {
  const BwdWorkspace L = bwd_workspace_layout(s, true);
  char* w = static_cast<char*>(ws);
  float* Dv = reinterpret_cast<float*>(w + L.off_D);
  float* da = reinterpret_cast<float*>(w + L.off_da);
  int32_t* coff = reinterpret_cast<int32_t*>(w + L.off_csr_off);
  int32_t* clist = reinterpret_cast<int32_t*>(w + L.off_csr_list);
  int32_t* order = reinterpret_cast<int32_t*>(w + L.off_order);
  __nv_bfloat16* dsbuf = reinterpret_cast<__nv_bfloat16*>(w + L.off_ds);
  const int G = s.Hq / s.Hkv;
  const int tiles = G / 2;
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_tmap_bf16(&tq, q, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tdo, dO, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, s.T, s.B * s.Hkv)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, s.T, s.B * s.Hkv)) != cudaSuccess) return e;
  CUtensorMap tq2, tdo2;  // 64 x 64 x 2 boxes for the dK/dV kernel's 128-row tiles
  if ((e = make_tmap_bf16_2planes(&tq2, q, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_2planes(&tdo2, dO, s.T, s.B * s.Hq)) != cudaSuccess) return e;
  if (s.dense) {
    // Every block: no reverse index, no dS tiles (dq recomputes them), no da.
    if (o_res) {
      if ((e = launch_d_from_o(s, dO, o, o_res, Dv, st)) != cudaSuccess) return e;
    } else {
      dim3 grid(s.N, s.Hkv * tiles, s.B);
      auto kern = tiles == 2 ? tc_bwd_d_kernel<2> : tc_bwd_d_kernel<1>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kd::kSmem);
      if (e != cudaSuccess) return e;
      kern<<<grid, kd::kThreadsD, kd::kSmem, st>>>(tq, tk, tv, tdo, lse, nullptr, nullptr, s, Dv,
                                                   ctx);
      note_launches(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
      dim3 grid(s.N * s.Hkv * s.B);
      auto kern = tiles == 2 ? tc_bwd_dkdv_kernel<2, false> : tc_bwd_dkdv_kernel<1, false>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kb_::kSmem);
      if (e != cudaSuccess) return e;
      kern<<<grid, kb_::kThreadsB, kb_::kSmem, st>>>(tq2, tk, tv, tdo2, lse, Dv, nullptr, nullptr,
                                                     nullptr, nullptr, s, (__nv_bfloat16*)dk,
                                                     (__nv_bfloat16*)dv, nullptr, nullptr, ctx);
      note_launches(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
      dim3 grid(s.N, s.Hkv * tiles, s.B);
      auto kern = tiles == 2 ? tc_bwd_dq_recompute_kernel<2> : tc_bwd_dq_recompute_kernel<1>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kr::kSmem);
      if (e != cudaSuccess) return e;
      kern<<<grid, kr::kThreadsR, kr::kSmem, st>>>(tq, tk, tv, tdo, lse, Dv, nullptr, nullptr, s,
                                                   (__nv_bfloat16*)dq, ctx);
      note_launches(1);
      return cudaGetLastError();
    }
  }
  if ((e = launch_bwd_csr(s, idx, coff, clist, ctx, st)) != cudaSuccess) return e;
  {
    const size_t smem = sizeof(int32_t) * ((size_t)s.N + 1);
    e = cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    order_kernel<<<1, 1024, smem, st>>>(coff, s, order);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (o_res) {  // D from the forward's output and its residual
    if ((e = launch_d_from_o(s, dO, o, o_res, Dv, st)) != cudaSuccess) return e;
  } else {  // D, recomputed exactly
    dim3 grid(s.N, s.Hkv * tiles, s.B);
    auto kern = tiles == 2 ? tc_bwd_d_kernel<2> : tc_bwd_d_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kd::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kd::kThreadsD, kd::kSmem, st>>>(tq, tk, tv, tdo, lse, idx, gates, s, Dv, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {  // dK, dV, dS tiles, da
    dim3 grid(s.N * s.Hkv * s.B);
    const bool outer = s.outer && gates != nullptr;
    auto kern = tiles == 2 ? (outer ? tc_bwd_dkdv_kernel<2, true> : tc_bwd_dkdv_kernel<2, false>)
                           : (outer ? tc_bwd_dkdv_kernel<1, true> : tc_bwd_dkdv_kernel<1, false>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kb_::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kb_::kThreadsB, kb_::kSmem, st>>>(tq2, tk, tv, tdo2, lse, Dv, gates, coff, clist,
                                                   order, s, (__nv_bfloat16*)dk,
                                                   (__nv_bfloat16*)dv, dsbuf,
                                                   dscores ? da : nullptr, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {  // dq
    dim3 grid(s.N, s.Hkv * tiles, s.B);
    auto kern = tiles == 2 ? tc_bwd_dq_kernel<2> : tc_bwd_dq_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kq::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kq::kThreadsQ, kq::kSmem, st>>>(dsbuf, tk, idx, s, (__nv_bfloat16*)dq, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dscores) return launch_bwd_jacobian(s, da, idx, gates, dscores, 4, st);
  return cudaSuccess;
}

}  // namespace sas
