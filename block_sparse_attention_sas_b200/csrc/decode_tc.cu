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
// SM: one's softmax chain overlaps the other's). Cache rows past L lie outside the tensor map and are read as zeros.
// The splits of one (batch, KV head) merge their partial (max, sum, o) by
// log-sum-exp. Up to 16 splits run as one thread-block cluster: each CTA
// leaves its partial in its shared memory and, after a cluster barrier, CTA
// r merges the heads g = r, r + splits, ... by reading the others' partials
// through distributed shared memory (no workspace, no extra launch). More
// splits (the long dense comparison) go through the workspace, where the last
// CTA of the unit, found with an atomic ticket, merges them.
// The kernel waits for the previous grid of the stream (programmatic
// dependent launch) only once its prologue (barriers, TMEM, tensor-map
// prefetch) is done, so that prologue overlaps the tail of the Top-K.
// Every wait is bounded.
#include <math.h>
#include <stddef.h>

#include <mutex>

#include "sas_internal.h"
#include "tc_common.cuh"
#include "topk_select.cuh"

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
constexpr int kMaxClusterSplits = 16;  // largest (non-portable) cluster

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kStages = 3;  // 32 KB K/V stages; two CTAs share an SM
constexpr uint32_t kOffQ = 0;           // [k half][8 rows][128 B]
constexpr uint32_t kOffKV = 2048;       // stages x (K halves 16 KB, V halves 16 KB)
constexpr uint32_t kOffCtl = kOffKV + kStages * 32768;
constexpr uint32_t kColS = 0, kColO = 128;
constexpr int kSub = 4;  // most page boxes per 64-token block (pages of 16 tokens)

struct Ctl {
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], p_full[2], o_full, o_final,
      drain;
  uint32_t tmem_base;
  int abort, nblk;
  int blocks[kMaxSlotsPerSplit];
  float bias[kMaxSlotsPerSplit];  // log2-domain gate bias
  // 16-byte aligned: the cluster merge moves part_o rows as float4.
  union alignas(16) {
    struct {
      float wgt[kMaxG * 64];  // merge weights of the last CTA
      // This split's partial for the cluster merge: unnormalised o per head.
      float part_o[kMaxG][kD];
    };
    // Paged cache, while the blocks stream: the page of each of a block's
    // sub-boxes (-1: nothing to load), kSub entries per block.
    int pg[kMaxG * 64 + kMaxG * kD];
  };
  float lsum[kMaxG];
  int last;
  int Lseq;  // tokens of this unit's sequence
  // Running max (log2 domain) and sum of this split's partial per head.
  float2 part_ml[kMaxG];  // (max, sum) per head
  uint64_t sel_full[3];   // the pooled selector's staged key summaries
};
constexpr size_t kSmem = kOffCtl + sizeof(Ctl) + 1024;
static_assert(kOffCtl % 16 == 0 && offsetof(Ctl, part_o) % 16 == 0 && (kD * 4) % 16 == 0,
              "the float4 accesses of part_o need 16-byte alignment");

// The fused selection (gates and Top-K of the unit's score row, then the
// decode of the selected blocks in the same launch). Its scratch lives in the
// K/V ring, which no load touches before the block lists exist.
struct SelArgs {
  bool on;              // select in the launch (else idx / gates are given)
  const float* scores;  // [B * Hkv][C] selector scores (null when C == 0, or pooled)
  // Pooled selector (kbar != nullptr): the scores are formed in the launch,
  // s_m = sel_scale * qbar . kbar_m, qbar the mean of the unit's query heads.
  const float* kbar;          // [B * Hkv][C][128] fp32 block means, 16-byte aligned
  const __nv_bfloat16* q;     // [B * Hq][128]
  float sel_scale;
  float* gates_out;     // [B * Hkv][C] or nullptr
  int32_t* idx_out;     // [B * Hkv][K] or nullptr
  int chunk;            // entries of the row per split (<= 512)
};
constexpr uint32_t kOffSelList = (sizeof(SelShared) + 127) & ~127u;  // from kOffKV
static_assert(kOffSelList + 16 * 256 * 8 <= kStages * 32768,
              "the selection scratch and list fit in the K/V ring");
// The pooled selector stages the key summaries of its entries through the
// ring (free until the selection's first cluster barrier: no CTA touches
// another's shared memory before it) in kSelBufs pieces of kSelRows rows,
// then keeps qbar and the 512 scores after them.
constexpr int kSelRows = 60;
constexpr int kSelBufs = 3;
constexpr uint32_t kSelPiece = kSelRows * kD * 4;
constexpr uint32_t kOffSelScores = kSelBufs * kSelPiece;  // from kOffKV
static_assert(kOffSelScores + (kD + 512) * 4 <= kStages * 32768 && kSelPiece % 16 == 0,
              "the staged summaries, qbar and the scores fit in the K/V ring");

template <int G, bool SEL>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ idx,
                 const float* __restrict__ gates, DecodeShape s, __nv_bfloat16* __restrict__ o,
                 float* __restrict__ ws_ml, float* __restrict__ ws_o, uint32_t* __restrict__ ws_cnt,
                 PagedArgs pa, SelArgs sa, DevCtx ctx) {
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
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
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
    }
    // The inputs may come from the previous grid of the stream: nothing of
    // them is read before it has completed.
    grid_dependency_wait();
    if (lane == 0) {
      mbar_arrive_expect_tx(&c.q_full, 2 * 1024);
      for (int kb = 0; kb < 2; ++kb)
        tma_load_3d(base + kOffQ + kb * 1024, &tm_q, kb * 64, (int)hbase, 0, &c.q_full);
    }
    // The split's blocks in slot order: selected history blocks (bias log g
    // when gates are on), then the current block C; empty slots are skipped.
    // A paged cache has its own length per sequence, so its own C.
    const int32_t* ix = s.dense ? nullptr : idx + (long long)unit * s.K;
    int Lq = s.L, Cq = s.C;
    bool seq_ok = true;
    if (s.paged) {
      Lq = pa.lens[bi];
      seq_ok = Lq >= 1 && Lq <= s.L;
      if (!seq_ok && lane == 0) report(ctx, kDevErrBadIndex);
      Cq = seq_ok ? (Lq - 1) / kB : 0;
    }
    int n = 0;
    for (int sb = sl0; !SEL && seq_ok && sb < sl1; sb += 32) {
      const int sl = sb + lane;
      int m = -1;
      float bias = 0.f;
      if (sl < sl1) {
        if (s.dense || sl == s.K) {
          m = s.dense ? sl : Cq;
        } else {
          m = ix[sl];
          if (m >= Cq || m < -1) {
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
        if (s.paged) {
          // Pages of the block's sub-boxes of min(P, 64) tokens; boxes that
          // start past the sequence, or whose page is missing, load nothing.
          const int rows = min(pa.P, kB), nsub = kB / rows;
          const long long p0 = pa.indptr[bi], np = pa.indptr[bi + 1] - p0;
          for (int i = 0; i < kSub; ++i) {
            int page = -1;
            const int t0 = m * kB + i * rows;
            if (i < nsub && t0 < Lq) {
              const long long lp = t0 / pa.P;
              if (lp < np) page = pa.indices[p0 + lp];
              if (lp >= np || page < 0 || page >= pa.num_pages) {
                report(ctx, kDevErrBadIndex);
                page = -1;
              }
            }
            c.pg[pos * kSub + i] = page;
          }
        }
      }
      n += __popc(mask);
    }
    if (lane == 0) {
      if (!SEL) c.nblk = n;
      c.Lseq = Lq;
    }
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if constexpr (SEL) {
    // ---- the unit's gates and Top-K, selected by its splits together
    // (cluster_select); rank 0 stores each selected block, with its bias,
    // into the control block of the split that owns its slot.
    grid_dependency_wait();  // the scores may come from the previous grid
    const int CS = s.splits, C = s.C, kk = min(s.K, C);
    SelShared& sh = *reinterpret_cast<SelShared*>(base + kOffKV);
    uint64_t* list = reinterpret_cast<uint64_t*>(base + kOffKV + kOffSelList);
    const int lo = split * sa.chunk;
    float f[4];
    bool okf[4];
    if (sa.kbar) {
      // The pooled selector's scores of this split's entries: qbar (the mean
      // of the unit's G query heads) against each block's mean key. The
      // summaries arrive by bulk copies, up to three pieces in flight; a warp
      // takes a row at a time, a lane four columns of it.
      static_assert(kThreads == kD, "one thread per column of qbar");
      float* qb = reinterpret_cast<float*>(base + kOffKV + kOffSelScores);
      float* scr = qb + kD;
      const float* kb = sa.kbar + ((long long)unit * C + lo) * kD;
      const int here = max(0, min(sa.chunk, C - lo));
      const int npieces = (here + kSelRows - 1) / kSelRows;
      auto issue = [&](int p) {
        const uint32_t bytes = (uint32_t)min(kSelRows, here - p * kSelRows) * kD * 4;
        uint64_t* bar = &c.sel_full[p % kSelBufs];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(base + kOffKV + (p % kSelBufs) * kSelPiece, kb + (long long)p * kSelRows * kD,
                 bytes, bar);
      };
      if (tid == 0) {
        for (int i = 0; i < kSelBufs; ++i) mbar_init(&c.sel_full[i], 1);
        fence_mbar_init();
        for (int p = 0; p < min(kSelBufs, npieces); ++p) issue(p);
      }
      {
        float a = 0.f;
        for (int g = 0; g < G; ++g) a += __bfloat162float(sa.q[(hbase + g) * kD + tid]);
        qb[tid] = a / (float)G;
      }
      __syncthreads();
      const float4 qv = reinterpret_cast<const float4*>(qb)[lane];
      for (int p = 0; p < npieces; ++p) {
        const int rows = min(kSelRows, here - p * kSelRows);
        if (!mbar_wait(ctx, &c.sel_full[p % kSelBufs], (p / kSelBufs) & 1)) *abort = 1;
        const float4* buf =
            reinterpret_cast<const float4*>(base + kOffKV + (p % kSelBufs) * kSelPiece);
        for (int r0 = warp * 4; r0 < rows; r0 += 4 * kWarps) {
          float acc[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 v = r0 + u < rows ? buf[(r0 + u) * (kD / 4) + lane]
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
            float a = 0.f;  // the standalone selector kernel's order of terms
            a = fmaf(qv.x, v.x, a);
            a = fmaf(qv.y, v.y, a);
            a = fmaf(qv.z, v.z, a);
            acc[u] = fmaf(qv.w, v.w, a);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float a = warp_sum(acc[u]);
            if (lane == 0 && r0 + u < rows) scr[p * kSelRows + r0 + u] = a * sa.sel_scale;
          }
        }
        __syncthreads();  // every read of the piece is done: its buffer takes the next
        if (tid == 0 && p + kSelBufs < npieces) {
          fence_proxy_async_smem();
          issue(p + kSelBufs);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = lo + tid + kThreads * e;
        okf[e] = i < C && i < lo + sa.chunk;
        f[e] = okf[e] ? scr[tid + kThreads * e] : -INFINITY;
      }
    } else {
      const float* srow = C > 0 ? sa.scores + (long long)unit * C : nullptr;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = lo + tid + kThreads * e;
        okf[e] = i < C && i < lo + sa.chunk;
        f[e] = okf[e] ? srow[i] : -INFINITY;
      }
    }
    float lse = 0.f;
    if (kk > 0) {  // the same in every split of the unit
      const int m = cluster_select<kThreads, 4>(f, okf, lo, sa.chunk, C, kk, CS, sh, list);
      lse = sh.lse;
      if (split == 0) {
        int32_t* iout = sa.idx_out ? sa.idx_out + (long long)unit * s.K : nullptr;
        place_by_rank<kThreads>(list, m, kk, [&](int rk, uint64_t key) {
          const int owner = rk / s.bps, pos = rk - owner * s.bps;
          const int blk = ckey_index(key);
          const float bias = s.use_gates ? (ckey_score(key) - lse) * kLog2e : 0.f;
          dsmem_st_u32(dsmem_addr(&c.blocks[pos], (uint32_t)owner), (uint32_t)blk);
          dsmem_st_f32(dsmem_addr(&c.bias[pos], (uint32_t)owner), bias);
          if (iout) iout[rk] = blk;
        });
      }
    }
    if (split == 0 && sa.idx_out)
      for (int p = kk + tid; p < s.K; p += kThreads) sa.idx_out[(long long)unit * s.K + p] = -1;
    // This split's list: its selected slots [sl0, min(sl1, kk)), then the
    // current block (slot K) when the split holds that slot.
    if (tid == 0) {
      int nb = max(0, min(sl1, kk) - sl0);
      if (s.K >= sl0 && s.K < sl1) {
        c.blocks[nb] = C;
        c.bias[nb] = 0.f;
        ++nb;
      }
      c.nblk = nb;
    }
    sel_sync(CS);  // (4) every split's list is complete
    if (sa.gates_out) {
      float* grow = sa.gates_out + (long long)unit * C;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (okf[e]) grow[lo + tid + kThreads * e] = fast_gate(f[e], lse, SAS_PHI_SOFTMAX);
    }
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
        if (!s.paged) {
          mbar_arrive_expect_tx(&c.kv_full[st], 32768);
          for (int h2 = 0; h2 < 2; ++h2) {
            tma_load_3d(kv + h2 * 8192, &tm_k, h2 * 64, m * kB, (int)plane, &c.kv_full[st]);
            tma_load_3d(kv + 16384 + h2 * 8192, &tm_v, h2 * 64, m * kB, (int)plane,
                        &c.kv_full[st]);
          }
        } else {
          // Sub-box i (rows rows, 8-row aligned, so the 128-byte swizzle
          // phase is that of a whole-block load) from page pg[i].
          const int rows = min(pa.P, kB), nsub = kB / rows;
          const int row0 = pa.P > kB ? (m * kB) % pa.P : 0;
          uint32_t bytes = 0;
          for (int i = 0; i < nsub; ++i) bytes += c.pg[n * kSub + i] >= 0 ? 512u * rows : 0u;
          mbar_arrive_expect_tx(&c.kv_full[st], bytes);
          for (int i = 0; i < nsub; ++i) {
            const int page = c.pg[n * kSub + i];
            if (page < 0) continue;
            const int pl = page * s.Hkv + kvh;
            for (int h2 = 0; h2 < 2; ++h2) {
              tma_load_3d(kv + h2 * 8192 + i * rows * 128, &tm_k, h2 * 64, row0, pl,
                          &c.kv_full[st]);
              tma_load_3d(kv + 16384 + h2 * 8192 + i * rows * 128, &tm_v, h2 * 64, row0, pl,
                          &c.kv_full[st]);
            }
          }
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
    // Lane l owns query row l % 8 (the 8-row Q box repeats down the tile, so
    // lanes l, l + 8, l + 16, l + 24 hold the same S row) and, as lane group
    // g = l / 8, the 16 columns 16 g .. 16 g + 15 of every block: each group
    // is a split of its own (running max, sum and O in its TMEM lane; P is
    // zero outside its columns) and the four are merged at the end. So a lane
    // forms 16 probabilities per block, not 64.
    constexpr float kLazy = 8.f;  // log2 headroom of P over the reference max
    const float sc = s.scale * kLog2e;
    const uint32_t tl = tmem;  // lanes 0..31
    const int grp = lane >> 3;
    const bool row_live = (lane & 7) < G;
    for (int n = 0; n < nblk; ++n) {
      const int st = n & 1;
      if (!warp_wait(ctx, &c.s_full[st], (n >> 1) & 1, abort)) {
        ok_sm = false;
        break;
      }
      fence_after_sync();
      const int m = c.blocks[n];
      const float bias = c.bias[n];
      const int kvalid = min(kB, c.Lseq - m * kB);
      // This group's 16 columns of S (the ld is warp-wide; each group keeps its own).
      float sv[16];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sr[32];
        tmem_ld32(tl + kColS + st * 64 + hf * 32, sr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (grp == 2 * hf) sv[i] = __uint_as_float(sr[i]);
          else if (grp == 2 * hf + 1) sv[i] = __uint_as_float(sr[16 + i]);
        }
      }
      float smax = -INFINITY;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (16 * grp + i >= kvalid) sv[i] = -INFINITY;
        smax = fmaxf(smax, sv[i]);
      }
      const float mx = (smax == -INFINITY) ? -INFINITY : fmaf(smax, sc, bias);
      // Reference update: the first finite max sets it (nothing accumulated
      // for the lane yet); a max more than kLazy above it rescales O.
      const bool need = row_live && m_run != -INFINITY && mx > m_run + kLazy;
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
      uint32_t pk8[8], pk[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t a = ffma2(f2u(sv[2 * i], sv[2 * i + 1]), sc2, off2);
        const float p0 = ex2(lo_f(a)), p1 = ex2(hi_f(a));
        accp = fadd2(accp, f2u(p0, p1));
        pk8[i] = pack_bf16(p0, p1);
      }
      // P(n) into the S columns already read: word w holds columns 2w, 2w + 1,
      // so this group's words are 8 g .. 8 g + 7 and the rest are zero.
#pragma unroll
      for (int w = 0; w < 32; ++w) pk[w] = ((w >> 3) == grp) ? pk8[w & 7] : 0u;
      tmem_st32(tl + kColS + st * 64, pk);
      l_run += lo_f(accp) + hi_f(accp);
      if (s.paged && kvalid < kB) {
        // Rows past the sequence in a page hold other tokens or stale data:
        // zero them (whole 128-byte rows, so the swizzle does not matter) so
        // that PV reads 0 there; their P is 0 already.
        unsigned char* vst = base + kOffKV + (n % kStages) * 32768 + 16384;
        const int nz = (kB - kvalid) * 8;  // 16-byte chunks per d-half
        for (int e = lane; e < 2 * nz; e += 32) {
          const int h2 = e / nz, x = e - h2 * nz;
          *reinterpret_cast<uint4*>(vst + h2 * 8192 + kvalid * 128 + x * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
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
    // Merge the four column groups of each row (lanes l, l ^ 8, l ^ 16,
    // l ^ 24) by log-sum-exp; every lane of the row ends with the result.
    {
      float Mr = fmaxf(m_run, __shfl_xor_sync(0xffffffffu, m_run, 8));
      Mr = fmaxf(Mr, __shfl_xor_sync(0xffffffffu, Mr, 16));
      const float wgt = (m_run == -INFINITY) ? 0.f : ex2(m_run - Mr);
      float lt = wgt * l_run;
      lt += __shfl_xor_sync(0xffffffffu, lt, 8);
      lt += __shfl_xor_sync(0xffffffffu, lt, 16);
#pragma unroll
      for (int i = 0; i < kD; ++i) {
        float a = wgt * acc[i];
        a += __shfl_xor_sync(0xffffffffu, a, 8);
        a += __shfl_xor_sync(0xffffffffu, a, 16);
        acc[i] = a;
      }
      m_run = Mr;
      l_run = lt;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  const bool ok_cta = !*abort;  // uniform: read after the barrier above

  if (s.cluster) {
    // ---- cluster merge: partials in shared memory, read by rank
    if (warp == kSoftmaxWarp && lane < G) {
      const bool good = ok_cta && ok_sm;
      float4* dst = reinterpret_cast<float4*>(c.part_o[lane]);
#pragma unroll
      for (int q4 = 0; q4 < kD / 4; ++q4)
        dst[q4] = make_float4(acc[4 * q4], acc[4 * q4 + 1], acc[4 * q4 + 2], acc[4 * q4 + 3]);
      c.part_ml[lane] = good ? make_float2(m_run, l_run) : make_float2(-INFINITY, 0.f);
    }
    cluster_sync_all();
    const int P = s.splits;
    for (int g = split; g < G; g += P) {
      // Thread t (t < 32) owns columns 4t .. 4t + 3 of head g: it issues the
      // loads of every split's (max, sum) and partial columns at once (one
      // round trip through distributed shared memory), then merges them.
      if (tid < kD / 4) {
        float2 ml[kMaxClusterSplits];
        float4 v[kMaxClusterSplits];
#pragma unroll
        for (int x = 0; x < kMaxClusterSplits; ++x)
          if (x < P) {
            ml[x] = dsmem_ld_f32x2(dsmem_addr(&c.part_ml[g], (uint32_t)x));
            v[x] = dsmem_ld_f32x4(dsmem_addr(&c.part_o[g][4 * tid], (uint32_t)x));
          }
        float M = -INFINITY;
#pragma unroll
        for (int x = 0; x < kMaxClusterSplits; ++x)
          if (x < P) M = fmaxf(M, ml[x].x);
        float Lsum = 0.f;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int x = 0; x < kMaxClusterSplits; ++x) {
          if (x >= P || ml[x].x == -INFINITY) continue;
          const float f = ex2(ml[x].x - M);
          Lsum = fmaf(f, ml[x].y, Lsum);
          a.x = fmaf(f, v[x].x, a.x);
          a.y = fmaf(f, v[x].y, a.y);
          a.z = fmaf(f, v[x].z, a.z);
          a.w = fmaf(f, v[x].w, a.w);
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        uint2 pk;
        pk.x = pack_bf16(a.x * inv, a.y * inv);
        pk.y = pack_bf16(a.z * inv, a.w * inv);
        *reinterpret_cast<uint2*>(o + (hbase + g) * kD + 4 * tid) = pk;
      }
    }
    // Every rank's shared memory stays alive until all reads above are done.
    cluster_sync_all();
    return;
  }
  if (!ok_cta) return;

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

// Launch through cudaLaunchKernelEx: as a programmatic dependent of the
// previous grid (its prologue overlaps that grid's tail), and with the
// unit's splits as one cluster when s.cluster is set.
template <int G, bool SEL>
cudaError_t launch_g(const DecodeShape& s, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, const int32_t* idx, const float* gates, void* o,
                     float* ws_ml, float* ws_o, uint32_t* ws_cnt, const PagedArgs& pa,
                     const SelArgs& sa, const DevCtx& ctx, cudaStream_t st, bool pdl) {
  auto kern = decode_tc_kernel<G, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  const bool cluster = s.cluster || SEL;  // a fused selection always runs as one cluster
  if (cluster && s.splits > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.splits, s.Hkv, s.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)s.splits;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, idx, gates, s, (__nv_bfloat16*)o, ws_ml, ws_o,
                         ws_cnt, pa, sa, ctx);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

// Whether a cluster of `splits` decode CTAs (G heads) fits on the device,
// asked once per (G, splits) and process.
template <int G>
bool cluster_fits(int splits) {
  static std::mutex mu;
  static signed char fits[17] = {};
  std::lock_guard<std::mutex> lk(mu);
  if (fits[splits] == 0) {
    auto kern = decode_tc_kernel<G, false>;
    bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem) ==
              cudaSuccess;
    if (ok && splits > 8)
      ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
           cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, 1, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (ok) ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess;
    (void)cudaGetLastError();
    fits[splits] = (ok && n > 0) ? 1 : -1;
  }
  return fits[splits] > 0;
}

template <int G>
cudaError_t launch_any(DecodeShape s, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const int32_t* idx, const float* gates, void* o,
                       float* ws_ml, float* ws_o, uint32_t* ws_cnt, const PagedArgs& pa,
                       const SelArgs& sa, const DevCtx& ctx, cudaStream_t st) {
  s.cluster = s.splits >= 2 && s.splits <= kMaxClusterSplits && cluster_fits<G>(s.splits);
  if (sa.on) {
    // The fused selection needs the unit's splits in one cluster.
    if (!s.cluster && s.splits != 1) return cudaErrorNotSupported;
    return launch_g<G, true>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st,
                             true);
  }
  if (!s.cluster && s.splits > 1) {
    // Tickets start at zero on every call, whatever the workspace held before.
    cudaError_t e = cudaMemsetAsync(ws_cnt, 0, sizeof(uint32_t) * (size_t)s.B * s.Hkv, st);
    if (e != cudaSuccess) return e;
    note_launches(1);
  }
  // Only a kernel may precede a programmatic dependent: after the memset the
  // launch is an ordinary one.
  const bool pdl = s.cluster || s.splits == 1;
  return launch_g<G, false>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st,
                            pdl);
}

}  // namespace

bool tc_decode_supported(sas_dtype_t dt, const DecodeShape& s) {
  const int G = s.Hq / s.Hkv;
  return dt == SAS_BF16 && s.d == kD && s.b == kB && G >= 1 && G <= kMaxG && s.splits <= 64 &&
         s.bps <= kMaxSlotsPerSplit;
}

namespace {
cudaError_t launch_tc_maps(const DecodeShape& s, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, const PagedArgs& pa, const int32_t* idx,
                           const float* gates, void* o, void* ws, const SelArgs& sa,
                           const DevCtx& ctx, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  const size_t parts = (size_t)s.B * s.Hq * s.splits;
  float* ws_ml = reinterpret_cast<float*>(w);
  float* ws_o = reinterpret_cast<float*>(w + ((2 * parts * sizeof(float) + 255) & ~(size_t)255));
  uint32_t* ws_cnt = reinterpret_cast<uint32_t*>(
      reinterpret_cast<char*>(ws_o) + ((parts * s.d * sizeof(float) + 255) & ~(size_t)255));
  switch (s.Hq / s.Hkv) {
    case 1:
      return launch_any<1>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 2:
      return launch_any<2>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 3:
      return launch_any<3>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 4:
      return launch_any<4>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 5:
      return launch_any<5>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 6:
      return launch_any<6>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 7:
      return launch_any<7>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    case 8:
      return launch_any<8>(s, tq, tk, tv, idx, gates, o, ws_ml, ws_o, ws_cnt, pa, sa, ctx, st);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

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
  const PagedArgs none = {nullptr, nullptr, nullptr, 0, 0};
  const SelArgs nosel = {false, nullptr, nullptr, nullptr, 0.f, nullptr, nullptr, 0};
  return launch_tc_maps(s, tq, tk, tv, none, idx, gates, o, ws, nosel, ctx, st);
}

cudaError_t launch_decode_select_tc(const DecodeShape& s0, const void* q, const void* kc,
                                    const void* vc, const float* scores, const float* kbar,
                                    float sel_scale, float* gates_out, int32_t* idx_out, void* o,
                                    void* ws, const DevCtx& ctx, cudaStream_t st) {
  // A row longer than 512 entries a split widens the cluster: the extra
  // CTAs (slot ranges past the last slot) help select and stream nothing.
  DecodeShape s = s0;
  const int need = (s.C + 511) / 512;
  if (need > s.splits) s.splits = need;
  if (s.dense || s.paged || s.splits > kSelMaxCta || s.K > 256) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_tmap_bf16_rows8(&tq, q, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_pitched(&tk, kc, s.L, s.Lcap, s.B * s.Hkv)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_pitched(&tv, vc, s.L, s.Lcap, s.B * s.Hkv)) != cudaSuccess) return e;
  const PagedArgs none = {nullptr, nullptr, nullptr, 0, 0};
  const SelArgs sa = {true,      scores,  kbar,    (const __nv_bfloat16*)q, sel_scale,
                      gates_out, idx_out, (s.C + s.splits - 1) / s.splits};
  return launch_tc_maps(s, tq, tk, tv, none, nullptr, nullptr, o, ws, sa, ctx, st);
}

cudaError_t launch_decode_paged_tc(const DecodeShape& s, const PagedArgs& pa, const void* q,
                                   const void* kpages, const void* vpages, const int32_t* idx,
                                   const float* gates, void* o, void* ws, const DevCtx& ctx,
                                   cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  // Pages as [num_pages * Hkv planes][P rows][128], boxes of min(P, 64) rows.
  const int rows = pa.P < kB ? pa.P : kB;
  if ((e = make_tmap_bf16_rows8(&tq, q, s.B * s.Hq)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_box(&tk, kpages, pa.P, pa.num_pages * s.Hkv, rows)) != cudaSuccess)
    return e;
  if ((e = make_tmap_bf16_box(&tv, vpages, pa.P, pa.num_pages * s.Hkv, rows)) != cudaSuccess)
    return e;
  const SelArgs nosel = {false, nullptr, nullptr, nullptr, 0.f, nullptr, nullptr, 0};
  return launch_tc_maps(s, tq, tk, tv, pa, idx, gates, o, ws, nosel, ctx, st);
}

}  // namespace sas
