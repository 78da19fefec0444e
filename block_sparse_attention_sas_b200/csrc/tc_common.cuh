// Blackwell (sm_100a) tensor-core helpers: TMA tile loads, tcgen05 MMA with
// TMEM accumulators, TMEM load/store, shared-memory matrix descriptors.
//
// Operand layouts used by the kernels (bf16, 128-byte swizzle, the layout a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes):
//   K-major  (rows x 64 elements per 128-byte row, 8-row / 1024-byte atoms):
//            descriptor LBO = 16 B (unused), SBO = 1024 B; one MMA K-step of
//            16 elements advances the start address by 32 B inside the row,
//            a second 64-element K half lives in its own region.
//   MN-major (rows = K index, 64 MN elements per 128-byte row): SBO = 1024 B
//            between 8-row K groups, LBO = byte offset between 64-element MN
//            groups; one K-step of 16 advances the start by 2 * SBO.
// Every tile base is 1024-byte aligned so the hardware swizzle (address bits
// [4,7) xor [7,10)) matches the TMA's.
#pragma once

#include "exp2_poly.h"
#include <cuda.h>
#include <stdint.h>

#include "sas_common.cuh"

namespace sas {
namespace tc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- instruction descriptor of tcgen05.mma kind::f16 (bf16 in, fp32 accumulate)
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)  // A major
         | ((b_mn_major ? 1u : 0u) << 16)  // B major
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// ---- shared-memory matrix descriptor (sm_100 version 1), 128-byte swizzle
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// ---- TMEM allocation (one full warp)
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ---- ordering of tcgen05 operations around thread synchronisation
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy shared-memory writes become visible to the async proxy (MMA, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- MMA: D[tmem] (+)= A[smem] * B[smem], issued by one thread
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
      "r"(z), "r"(z)
      : "memory");
}
// MMA with A in TMEM: D[tmem] (+)= A[tmem] * B[smem]. A (M rows x K, 16-bit)
// sits with row m in lane m and consecutive K elements packed two per 32-bit
// column (the even element in the low half), so one K-step of 16 advances the
// A address by 8 columns.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z),
      "r"(z), "r"(z)
      : "memory");
}

// Arrives once on `bar` when every MMA this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// ---- TMEM <-> registers: 32 lanes x 32 consecutive 32-bit columns per warp
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Copies row `row` of a [128 rows x 128] bf16 tile held in shared memory in
// the K-major 128-byte-swizzle layout (two 64-element halves, 16 KB apart)
// into 64 TMEM columns of this thread's lane, in the A-operand packing.
// Called by all 32 lanes of a warp (tcgen05.st is warp-wide).
__device__ __forceinline__ void tile_row_to_tmem(const unsigned char* tile, int row,
                                                 uint32_t taddr) {
  uint32_t w[64];
#pragma unroll
  for (int kb = 0; kb < 2; ++kb)
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile + kb * 16384 + row * 128 +
                                                      ((ch ^ (row & 7)) << 4));
      w[kb * 32 + ch * 4 + 0] = v.x;
      w[kb * 32 + ch * 4 + 1] = v.y;
      w[kb * 32 + ch * 4 + 2] = v.z;
      w[kb * 32 + ch * 4 + 3] = v.w;
    }
  tmem_st32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&w[0]));
  tmem_st32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&w[32]));
}


// ---- TMA tile load (3-D tensor map), completion counted on `bar`; no multicast
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
// ---- untiled bulk copy shared -> global (bulk-group completion), no multicast
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The source shared memory of every committed bulk store has been read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Barrier `id` (1..15; 0 is __syncthreads') among `nthreads` threads of the
// CTA, whole warps, every one of which must reach it.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Prefetch one tile of a 3D tensor map into L2: no shared-memory destination
// and no completion to wait for (a later load of the same tile hits L2).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- fast exp2 on the MUFU unit (relative error ~2^-22)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot for two lanes of work).
__device__ __forceinline__ uint64_t f2u(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo_f(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---- exp2 of a pair on the FMA pipe, to take part of the ex2 work off the
// MUFU unit where an elementwise phase is bound by it. x = n + f with
// n = round(x) (adding 1.5 * 2^23 rounds to nearest and leaves n in the low
// mantissa bits), f in [-1/2, 1/2]; 2^f by the degree-5 polynomial of
// exp2_poly.h in Horner form; n is then added to the exponent field (the
// magic constant's low 9 bits are zero, so bits(t) << 23 == n << 23). Inputs
// are clamped to -125, so -inf gives 2^-125 (~2.4e-38) where ex2.approx.ftz
// gives 0. Relative error ~2.5e-7 on [-125, 127].
__device__ __forceinline__ uint64_t ex2_poly2(uint64_t x2) {
  const float xa = fmaxf(lo_f(x2), -125.f), xb = fmaxf(hi_f(x2), -125.f);
  const uint64_t x = f2u(xa, xb);
  const uint64_t t = fadd2(x, f2u(12582912.f, 12582912.f));
  const uint64_t n = fadd2(t, f2u(-12582912.f, -12582912.f));
  const uint64_t f = ffma2(n, f2u(-1.f, -1.f), x);
  uint64_t p = ffma2(f2u(kExp2C5, kExp2C5), f, f2u(kExp2C4, kExp2C4));
  p = ffma2(p, f, f2u(kExp2C3, kExp2C3));
  p = ffma2(p, f, f2u(kExp2C2, kExp2C2));
  p = ffma2(p, f, f2u(kExp2C1, kExp2C1));
  p = ffma2(p, f, f2u(kExp2C0, kExp2C0));
  const uint32_t ra = (uint32_t)p + ((uint32_t)t << 23);
  const uint32_t rb = (uint32_t)(p >> 32) + ((uint32_t)(t >> 32) << 23);
  return ((uint64_t)rb << 32) | ra;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The attended-block list of one query block, built by one full warp: lane
// l reads idx slot base + l, valid entries (0 <= m < j) are compacted in slot
// order after `first` already-placed entries, with their log2-domain gate
// bias (0 without gates); entries >= j or below -1 (-1 marks an empty slot)
// are reported and skipped. Returns the list length.
__device__ __forceinline__ int warp_build_list(const int32_t* idx_row, const float* gate_row,
                                               int K, int j, int first, int* blocks, int* slots,
                                               float* bias, const DevCtx& ctx) {
  const int lane = threadIdx.x & 31;
  int n = first;
  for (int base = 0; base < K; base += 32) {
    const int sl = base + lane;
    const int m = sl < K ? idx_row[sl] : -1;
    const bool bad = m >= j || m < -1;
    if (bad) report(ctx, kDevErrBadIndex);
    const bool ok = m >= 0 && !bad;
    const float g = (ok && gate_row) ? gate_row[m] : 1.f;
    const uint32_t mask = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const int pos = n + __popc(mask & ((1u << lane) - 1u));
      blocks[pos] = m;
      if (slots) slots[pos] = sl;
      bias[pos] = gate_row ? logf(g) * 1.4426950408889634f : 0.f;
    }
    n += __popc(mask);
  }
  return n;
}

// Bounded mbarrier wait that also gives up when another thread of the CTA has
// set *abort (checked every 64 polls). On running out of polls it records a
// timeout, sets *abort and returns false.
__device__ __forceinline__ bool wait_or_abort(const DevCtx& c, uint64_t* bar, uint32_t parity,
                                              volatile int* abort) {
  for (unsigned long long i = 0; i < c.wait_limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63 && *abort) return false;
  }
  report(c, kDevErrTimeout);
  *abort = 1;
  return false;
}

// One lane of the warp polls the barrier; the others wait at the shuffle.
__device__ __forceinline__ bool warp_wait(const DevCtx& ctx, uint64_t* bar, uint32_t parity,
                                          volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(ctx, bar, parity, abort) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

}  // namespace tc
}  // namespace sas
