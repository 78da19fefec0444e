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
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxList = 257;

// ============================================================================
// Kernel A: dq, D, da
// ============================================================================
// Q and dO of the tile are copied into TMEM once and used as the A operand of
// every S / dP MMA, and dS goes back into TMEM as the A operand of the dQ MMA:
// the MMAs then read only K / V from shared memory. Two groups of four
// elementwise warps split each block's 64 keys (group g takes keys 32g ..).
//
// Every mbarrier wait costs the MMA-issuing thread far more than an MMA issue
// slot, so it waits once per iteration: the full barrier of K/V stage `it`
// also collects one arrival from each elementwise warp, given when that warp
// is done with the S/dP buffer of iteration it - 2 (and, in sweep 2, has
// written that iteration's dS). The MMA stream is S/dP(0), S/dP(1), ...,
// with dQ(it - 2) issued right before S/dP(it) in sweep 2.
namespace ka {
constexpr int kStages = 6;                // K/V ring depth (stages 4, 5 reuse the Q/dO area)
constexpr int kWarps = 12;
constexpr int kThreadsA = kWarps * 32;
constexpr uint32_t kOffQ = 0;             // [k half][128 rows][128 B]
constexpr uint32_t kOffDO = 32768;        // same layout
constexpr uint32_t kOffKV = 65536;        // stages 0..3; stage = (K halves, V halves) 32 KB
// TMEM columns.
constexpr uint32_t kColQ = 0, kColDO = 64, kColS = 128, kColDP = 256, kColDQ = 384;
struct Ctl {
  // kv_full[st]: the producer's expect-tx arrival, the TMA bytes and one
  // arrival per elementwise warp (9 arrivals per phase).
  uint64_t qdo_full, kv_full[kStages], kv_empty[kStages], s_full[2], ds_tail[2], dq_done, drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxList], slots[kMaxList];
  float bias[kMaxList];
  float red[kMaxList][8];  // per-warp partial sums of dS per block
  float dpart[2][128];     // per-group partial D per row
};
constexpr uint32_t kOffCtl = kOffKV + 4 * 32768;
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
__device__ __forceinline__ uint32_t stage_off(int st) {
  return st < 4 ? kOffKV + st * 32768u : kOffQ + (st - 4) * 32768u;
}
}  // namespace ka

template <int TILES>
__global__ void __launch_bounds__(ka::kThreadsA, 1)
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
  volatile int* abort = &c.abort;

  // Elementwise warps: tile row, its head and its lse, read before the CTA barrier.
  const int quarter = warp & 3, grp = (warp - 4) >> 2;
  const int rowi = quarter * 32 + lane;
  const int hh = rowi >> 6, r = rowi & 63;
  const int qrow = j * kB + r;
  const bool live = qrow < s.T;
  const long long hrow = (long long)(bi * s.Hq + h0 + hh) * s.T + qrow;
  float lse2 = 0.f;
  if (warp >= 4 && live) lse2 = lse[hrow] * kLog2e;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&c.qdo_full, 1);
      for (int i = 0; i < kStages; ++i) {
        mbar_init(&c.kv_full[i], 9);
        mbar_init(&c.kv_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&c.s_full[i], 1);
        mbar_init(&c.ds_tail[i], 8);
      }
      mbar_init(&c.dq_done, 1);
      mbar_init(&c.drain, 1);
      fence_mbar_init();
      c.abort = 0;
      // Q and dO do not depend on the selection: start their loads first.
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&c.qdo_full, 2 * 4 * 8192);
      for (int h2 = 0; h2 < 2; ++h2)
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(base + kOffQ + kb * 16384 + h2 * 8192, &tm_q, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qdo_full);
          tma_load_3d(base + kOffDO + kb * 16384 + h2 * 8192, &tm_do, kb * 64, j * kB,
                      bi * s.Hq + h0 + h2, &c.qdo_full);
        }
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
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
    __syncwarp();
    // Stages 0..3 are free: start their loads before the CTA barrier.
    if (lane == 0) {
      const int nit0 = 2 * (n + 1);  // sweep 1 then sweep 2 over the same blocks
      for (; issued < nit0 && issued < 4; ++issued) {
        const int m = c.blocks[issued % (n + 1)];
        unsigned char* kv = base + stage_off(issued);
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
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  const int nblk = c.nblk;
  const int nit = 2 * nblk;
  const int tail_first = max(nblk, nit - 2);  // sweep-2 iterations whose dQ follows the loop

  if (warp == 0) {
    if (lane == 0) {
      for (int it = issued; it < nit; ++it) {
        const int st = it % kStages;
        bool go = true;
        // Stages 4 and 5 reuse the Q/dO area: free once every elementwise
        // warp has moved its rows into TMEM (their first kv_full arrivals).
        if (it == 4) go = wait_or_abort(ctx, &c.kv_full[0], 0, abort);
        if (go && it >= kStages)
          go = wait_or_abort(ctx, &c.kv_empty[st], ((it - kStages) / kStages) & 1, abort);
        if (!go) break;
        const int m = c.blocks[it % nblk];
        unsigned char* kv = base + stage_off(st);
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
      // K-major K / V tiles: k-step ks at half (ks >> 2), byte (ks & 3) * 32.
      const uint64_t dkv0 = sdesc_sw128(sbase, 16, 1024);
      // K as the MN-major B operand of dQ: 16 keys per k-step (2048 B).
      const uint64_t dkq0 = sdesc_sw128(sbase, 8192, 1024);
      // dQ += dS K for sweep-2 iteration x; dS of keys 0..31 sits in S[x & 1]
      // columns 0..15, keys 32..63 in columns 32..47.
      auto issue_dq = [&](int x) {
        const uint64_t kd = dkq0 + (stage_off(x % kStages) >> 4);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ts(tmem + kColDQ, tmem + kColS + (x & 1) * 64 + (ks >> 1) * 32 + (ks & 1) * 8,
                      kd + ((ks * 2048) >> 4), id_q, (x > nblk || ks > 0));
      };
      bool ok = true;
      for (int it = 0; it < nit; ++it) {
        const int st = it % kStages, b = it & 1;
        if (!wait_or_abort(ctx, &c.kv_full[st], (it / kStages) & 1, abort)) {
          ok = false;
          break;
        }
        fence_after_sync();
        if (it >= nblk + 2) {
          issue_dq(it - 2);
          mma_commit(&c.kv_empty[(it - 2) % kStages]);
        }
        const uint64_t kd = dkv0 + (stage_off(st) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColS + b * 64, tmem + kColQ + ks * 8,
                      kd + (((ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + kColDP + b * 64, tmem + kColDO + ks * 8,
                      kd + ((16384 + (ks >> 2) * 8192 + (ks & 3) * 32) >> 4), id_s, ks > 0);
        mma_commit(&c.s_full[b]);
        if (it < nblk) mma_commit(&c.kv_empty[st]);  // sweep 1 only reads S and dP
      }
      for (int x = tail_first; ok && x < nit; ++x) {
        if (!wait_or_abort(ctx, &c.ds_tail[x - tail_first], 0, abort)) {
          ok = false;
          break;
        }
        fence_after_sync();
        issue_dq(x);
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
    // Arrival on the full barrier of iteration x (when there is one).
    auto arrive_w = [&](int x) {
      if (lane == 0 && x < nit) mbar_arrive(&c.kv_full[x % kStages]);
    };
    bool ok = warp_wait(ctx, &c.qdo_full, 0, abort);
    if (ok) {
      // Group 0 moves the Q rows into TMEM, group 1 the dO rows.
      tile_row_to_tmem(base + (grp == 0 ? kOffQ : kOffDO), rowi,
                       tl + (grp == 0 ? kColQ : kColDO));
      tmem_st_wait();
    }
    fence_before_sync();
    __syncwarp();
    arrive_w(0);
    arrive_w(1);
    float Dsum = 0.f;
    const uint64_t sc2 = f2u(sc, sc);
    // Sweep 1: D = sum over the attended keys of P * dP.
    for (int it = 0; ok && it < nblk; ++it) {
      const int b = it & 1;
      if (!warp_wait(ctx, &c.s_full[b], (it >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int m = c.blocks[it];
      const float bias = c.bias[it];
      const bool cur = (it == nblk - 1);
      const int kvalid = min(kB, s.T - m * kB) - 32 * grp;
      uint32_t sr[32], pr[32];
      tmem_ld32(tl + kColS + b * 64 + 32 * grp, sr);
      tmem_ld32(tl + kColDP + b * 64 + 32 * grp, pr);
      tmem_ld_wait();
      fence_before_sync();
      __syncwarp();
      arrive_w(it + 2);
      if (cur || kvalid < 32) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i >= kvalid || (cur && i + 32 * grp > r)) sr[i] = __float_as_uint(-INFINITY);
      }
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off);
      uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                  sc2, off2);
        const uint64_t p2 = f2u(ex2(lo_f(a2)), ex2(hi_f(a2)));
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        if (i & 1) acc1 = ffma2(p2, dp2, acc1);
        else acc0 = ffma2(p2, dp2, acc0);
      }
      const uint64_t accs = fadd2(acc0, acc1);
      Dsum += lo_f(accs) + hi_f(accs);
    }
    // The two groups' halves of D meet here; every elementwise warp arrives
    // exactly once, whichever path it took.
    c.dpart[grp][rowi] = Dsum;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    Dsum = c.dpart[0][rowi] + c.dpart[1][rowi];
    ok = ok && !*abort;
    const uint64_t negD = f2u(-Dsum, -Dsum);
    // Sweep 2: dS = P * (dP - D) back into TMEM for the dQ MMA, and its tile sums.
    for (int it = nblk; ok && it < nit; ++it) {
      const int b = it & 1, n = it - nblk;
      if (!warp_wait(ctx, &c.s_full[b], (it >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      fence_after_sync();
      const int m = c.blocks[n];
      const float bias = c.bias[n];
      const bool cur = (n == nblk - 1);
      const int kvalid = min(kB, s.T - m * kB) - 32 * grp;
      uint32_t sr[32], pr[32];
      tmem_ld32(tl + kColS + b * 64 + 32 * grp, sr);
      tmem_ld32(tl + kColDP + b * 64 + 32 * grp, pr);
      tmem_ld_wait();
      if (cur || kvalid < 32) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i >= kvalid || (cur && i + 32 * grp > r)) sr[i] = __float_as_uint(-INFINITY);
      }
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off);
      uint32_t pk[16];
      uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                  sc2, off2);
        const uint64_t p2 = f2u(ex2(lo_f(a2)), ex2(hi_f(a2)));
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        const uint64_t ds2 = fmul2(p2, fadd2(dp2, negD));
        if (i & 1) acc1 = fadd2(acc1, ds2);
        else acc0 = fadd2(acc0, ds2);
        pk[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
      }
      tmem_st16(tl + kColS + b * 64 + 32 * grp, pk);
      tmem_st_wait();
      fence_before_sync();
      __syncwarp();
      if (it + 2 < nit) arrive_w(it + 2);
      else if (lane == 0) mbar_arrive(&c.ds_tail[it - tail_first]);
      if (!cur) {
        const uint64_t accs = fadd2(acc0, acc1);
        const float t = warp_sum(lo_f(accs) + hi_f(accs));
        if (lane == 0) c.red[n][grp * 4 + quarter] = t;
      }
    }
    if (ok) {
      if (warp_wait(ctx, &c.dq_done, 0, abort)) {
        fence_after_sync();
        __nv_bfloat16* drow = dq + hrow * kD + grp * 64;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tl + kColDQ + grp * 64 + ch * 32, ov);
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
        if (live && grp == 0) Dv[hrow] = Dsum;
      }
    }
    // da of each selected block: the eight warps' partials in a fixed order.
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (da != nullptr && !*abort) {
      for (int n = tid - 128; n < nblk - 1; n += 256) {
        const float* p = c.red[n];
        const float t = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
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
// One CTA per (key block m, KV head, batch) steps over 128-row query tiles
// (the diagonal block's, then those of every query block that selected m).
// MMA stream: per step s, S/dP(s) then dV/dK(s - 1). The MMA thread waits
// once per step, on the Q/dO stage barrier of step s, which also collects
// one arrival from each elementwise warp once it has written P/dS of step
// s - 1 to shared memory (so the S/dP buffer of step s - 2 is free as well).
// A commit after dV/dK(s - 1) lets the producer reuse that Q/dO stage and
// the elementwise warps the P/dS buffer.
namespace kb_ {
constexpr int kWarps = 12;
constexpr int kThreadsB = kWarps * 32;
constexpr uint32_t kOffK = 0;         // [d half][64 rows][128 B]
constexpr uint32_t kOffV = 16384;
constexpr uint32_t kOffQD = 32768;    // 2 stages x (Q tile 32 KB, dO tile 32 KB)
constexpr uint32_t kOffP = 163840;    // [128 rows][128 B]
constexpr uint32_t kOffDS = 180224;
constexpr uint32_t kOffCtl = 196608;
// TMEM columns: S[b] at 64 b, dP[b] at 128 + 64 b, dV^T at 256, dK^T at 320.
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320;
struct Ctl {
  // qdo_full[stg]: the producer's expect-tx arrival and tile bytes, its
  // arrival once the step's scalars are staged, and one arrival per
  // elementwise warp (10 arrivals per phase).
  uint64_t kv_full, qdo_full[2], s_full[2], dvdk_done[2], pds_tail, acc_done, drain;
  uint32_t tmem_base;
  int abort;
  // Per stage, staged by the producer warp with the Q/dO tiles: the step's
  // query block, its log2-domain gate bias, and lse / D of the tile's rows.
  int step_j[2];
  float step_bias[2];
  float lse2[2][128], D[2][128];
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
}  // namespace kb_

template <int TILES>
__global__ void __launch_bounds__(kb_::kThreadsB, 1)
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
  // block m, then the selecting blocks in ascending order (entry / K of the
  // reverse list is the query block).
  volatile int* abort = &c.abort;

  if (tid == 0) {
    mbar_init(&c.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.qdo_full[i], 10);
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.dvdk_done[i], 1);
    }
    mbar_init(&c.pds_tail, 8);
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
    // four per lane, the query block and its gate bias) are loaded into
    // registers one step ahead, so staging them costs only shared stores.
    float pre_lse[4], pre_D[4], pre_bias = 0.f;
    int pre_j = m;
    // The reverse list in a register window (lane l holds entry win_lo + l),
    // with the next window already in flight.
    int win_lo = 0;
    int win = lane < nl ? lst[lane] : 0;
    int win_next = 32 + lane < nl ? lst[32 + lane] : 0;
    auto prefetch = [&](int st_i) {
      const int jj = st_i / TILES, u = st_i % TILES;
      int j = m;
      if (jj > 0) {
        const int ix = jj - 1;
        while (ix >= win_lo + 32) {
          win = win_next;
          win_lo += 32;
          win_next = win_lo + 32 + lane < nl ? lst[win_lo + 32 + lane] : 0;
        }
        j = __shfl_sync(0xffffffffu, win, ix - win_lo) / s.K;
      }
      pre_j = j;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int rr = lane + 32 * q4;
        const int head = kvh * G + 2 * u + (rr >> 6), qrow = j * kB + (rr & 63);
        const bool live = qrow < s.T;
        const long long hrow = (long long)(bi * s.Hq + head) * s.T + qrow;
        pre_lse[q4] = live ? lse[hrow] : 0.f;
        pre_D[q4] = live ? Dv[hrow] : 0.f;
      }
      pre_bias = (j == m || gates == nullptr) ? 1.f : gates[((long long)bh * s.N + j) * s.N + m];
    };
    prefetch(0);
    int issued = 0;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int stg = st_i & 1;
      bool go = true;
      // The stage is free once dV/dK of step st_i - 2 completed.
      if (lane == 0 && st_i >= 2)
        go = wait_or_abort(ctx, &c.dvdk_done[stg], ((st_i - 2) >> 1) & 1, abort);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      const int j = pre_j, u = st_i % TILES;
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
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        c.lse2[stg][lane + 32 * q4] = pre_lse[q4] * kLog2e;
        c.D[stg][lane + 32 * q4] = pre_D[q4];
      }
      if (lane == 0) {
        c.step_j[stg] = j;
        c.step_bias[stg] = logf(pre_bias) * kLog2e;
      }
      __threadfence_block();
      __syncwarp();
      // The consumers see the staged scalars once this stage's barrier phase
      // completes: the arrival below is part of it.
      if (lane == 0) mbar_arrive(&c.qdo_full[stg]);
      issued = st_i + 1;
      if (st_i + 1 < nsteps) prefetch(st_i + 1);
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
      const uint64_t dp0 = sdesc_sw128(sbase + kOffP, 8192, 1024);   // P (dS at +16 KB)
      auto issue_sdp = [&](int st_i) {
        const int stg = st_i & 1, b = st_i & 1;
        const uint64_t qa = dq0 + ((stg * 65536) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + kColS + b * 64, qa + (ao >> 4), dk0 + (bo >> 4), id_s, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ao = 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t bo = 16384 + (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_bf16_ss(tmem + kColDP + b * 64, qa + (ao >> 4), dk0 + (bo >> 4), id_s, ks > 0);
        }
        mma_commit(&c.s_full[b]);
      };
      // dV^T[d][key] += sum_q dO[q][d] P[q][key]; dK^T[d][key] += sum_q Q[q][d] dS[q][key]
      auto issue_dvdk = [&](int st_i) {
        const uint64_t qa = dqt0 + (((st_i & 1) * 65536) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + kColDV, qa + ((32768 + ks * 2048) >> 4), dp0 + ((ks * 2048) >> 4),
                      id_t, (st_i > 0 || ks > 0));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + kColDK, qa + ((ks * 2048) >> 4), dp0 + ((16384 + ks * 2048) >> 4),
                      id_t, (st_i > 0 || ks > 0));
      };
      bool ok = wait_or_abort(ctx, &c.kv_full, 0, abort);
      // Per step s: one wait (the Q/dO tiles of step s have landed and P/dS
      // of step s - 1 is in shared memory), then S/dP(s), so the elementwise
      // warps can start on it, then dV/dK(s - 1); its commit frees the Q/dO
      // stage of step s - 1 and the P/dS buffer.
      for (int st_i = 0; ok && st_i < nsteps; ++st_i) {
        if (!wait_or_abort(ctx, &c.qdo_full[st_i & 1], (st_i >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        fence_after_sync();
        issue_sdp(st_i);
        if (st_i > 0) {
          issue_dvdk(st_i - 1);
          mma_commit(&c.dvdk_done[(st_i - 1) & 1]);
        }
      }
      if (ok && wait_or_abort(ctx, &c.pds_tail, 0, abort)) {
        fence_after_sync();
        issue_dvdk(nsteps - 1);
      }
      mma_commit(&c.acc_done);
      if (*abort) {
        mma_commit(&c.drain);
        (void)mbar_wait(ctx, &c.drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3, grp = (warp - 4) >> 2;
    const int rowi = quarter * 32 + lane;  // tile row (query) / d index in the epilogue
    const int r = rowi & 63;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = s.scale * kLog2e;
    const int kvalid = min(kB, s.T - m * kB) - 32 * grp;
    const uint64_t sc2 = f2u(sc, sc);
    // Step 0 has no P/dS of a previous step to wait for.
    if (lane == 0) mbar_arrive(&c.qdo_full[0]);
    bool ok = true;
    for (int st_i = 0; st_i < nsteps; ++st_i) {
      const int b = st_i & 1;
      if (!warp_wait(ctx, &c.s_full[b], (st_i >> 1) & 1, abort)) {
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
      uint32_t sr[32], pr[32], pp[16], dd[16];
      tmem_ld32(tl + kColS + b * 64 + 32 * grp, sr);
      tmem_ld32(tl + kColDP + b * 64 + 32 * grp, pr);
      tmem_ld_wait();
      if (cur || kvalid < 32) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i >= kvalid || (cur && i + 32 * grp > r)) sr[i] = __float_as_uint(-INFINITY);
      }
      const float off = live ? bias - lse2 : -INFINITY;
      const uint64_t off2 = f2u(off, off), negD = f2u(-Di, -Di);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint64_t a2 = ffma2(f2u(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                  sc2, off2);
        const float p0 = ex2(lo_f(a2)), p1 = ex2(hi_f(a2));
        const uint64_t dp2 = f2u(__uint_as_float(pr[2 * i]), __uint_as_float(pr[2 * i + 1]));
        const uint64_t ds2 = fmul2(f2u(p0, p1), fadd2(dp2, negD));
        pp[i] = pack_bf16(p0, p1);
        dd[i] = pack_bf16(lo_f(ds2), hi_f(ds2));
      }
      // The P / dS buffers are free once dV/dK of step st_i - 1 completed.
      if (st_i >= 1 && !warp_wait(ctx, &c.dvdk_done[(st_i - 1) & 1], ((st_i - 1) >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      unsigned char* prow = base + kOffP + rowi * 128;
      unsigned char* drow = base + kOffDS + rowi * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const uint32_t sw = ((4 * grp + ch) ^ (rowi & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pp[4 * ch], pp[4 * ch + 1],
                                                          pp[4 * ch + 2], pp[4 * ch + 3]);
        *reinterpret_cast<uint4*>(drow + sw) = make_uint4(dd[4 * ch], dd[4 * ch + 1],
                                                          dd[4 * ch + 2], dd[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (st_i + 1 < nsteps) mbar_arrive(&c.qdo_full[(st_i + 1) & 1]);
        else mbar_arrive(&c.pds_tail);
      }
    }
    if (ok && warp_wait(ctx, &c.acc_done, 0, abort)) {
      // Epilogue: thread rowi holds dimension d = rowi; group g the keys 32g .. 32g + 31.
      fence_after_sync();
      const int d = rowi;
      const long long kb0 = ((long long)bh * s.T + (long long)m * kB) * kD;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = which == 0 ? dv : dk;
        const float mul = which == 0 ? 1.f : s.scale;
        uint32_t v[32];
        tmem_ld32(tl + (which == 0 ? kColDV : kColDK) + grp * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = grp * 32 + i;
          if (i < kvalid) out[kb0 + (long long)key * kD + d] =
              __float2bfloat16_rn(__uint_as_float(v[i]) * mul);
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
    kern<<<grid, ka::kThreadsA, ka::kSmem, st>>>(tq, tk, tv, tdo, lse, idx, gates, s,
                                            (__nv_bfloat16*)dq, Dv, dscores ? da : nullptr, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    dim3 grid(s.N, s.Hkv, s.B);
    auto kern = tiles == 2 ? tc_bwd_dkdv_kernel<2> : tc_bwd_dkdv_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kb_::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kb_::kThreadsB, kb_::kSmem, st>>>(tq, tk, tv, tdo, lse, Dv, gates, coff, clist, s,
                                             (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, ctx);
    note_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dscores) return launch_bwd_jacobian(s, da, idx, gates, dscores, st);
  return cudaSuccess;
}

}  // namespace sas
