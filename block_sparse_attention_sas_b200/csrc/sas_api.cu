// C ABI of the SAS library: argument validation on the host, dispatch to the
// kernels, device-side error reporting. Every check here runs before any
// launch, so a rejected call leaves the device untouched.
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "sas_common.cuh"
#include "sas_internal.h"

namespace sas {

// Per-device error word (one instance per device that loads the library).
static __device__ uint32_t g_dev_error;

namespace {

constexpr unsigned long long kDefaultWaitLimit = 1ull << 22;
std::atomic<unsigned long long> g_wait_limit{kDefaultWaitLimit};
std::atomic<unsigned long long> g_launches{0};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_err_ptr[kMaxDevices] = {nullptr};

// Device address of g_dev_error for the current device (looked up once per
// device; in host code the symbol itself is only a host-side handle).
cudaError_t device_ctx(DevCtx& ctx) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dev_error);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  ctx.err = g_err_ptr[dev];
  ctx.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  return cudaSuccess;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sas_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA; }

float resolve_scale(float scale, int d) {
  return scale > 0.f ? scale : 1.0f / sqrtf((float)d);
}

bool valid_dtype(sas_dtype_t dt) { return dt == SAS_F32 || dt == SAS_BF16; }

// Shared checks of the attention calls (forward, backward, dense).
sas_status_t check_attn(sas_dtype_t dt, int B, int Hq, int Hkv, int T, int d, int b, int K,
                        bool dense, float scale) {
  if (!valid_dtype(dt)) return SAS_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || T < 1 || d < 1 || b < 1) return SAS_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SAS_ERR_INVALID_ARG;
  if (!dense && K < 1) return SAS_ERR_INVALID_ARG;
  if (!isfinite(scale)) return SAS_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAS_ERR_UNSUPPORTED;
  if (b != 16 && b != 32 && b != 64) return SAS_ERR_UNSUPPORTED;
  if (!dense && K > 256) return SAS_ERR_UNSUPPORTED;
  if ((long long)B * Hq * T * d >= (1ll << 40)) return SAS_ERR_UNSUPPORTED;
  const long long N = (T + (long long)b - 1) / b;
  // N <= 16384 bounds the reverse-index kernel's shared memory (8 bytes per block).
  if (N > 16384 || B > 65535 || Hq > 65535) return SAS_ERR_UNSUPPORTED;
  return SAS_OK;
}

AttnShape make_shape(int B, int Hq, int Hkv, int T, int d, int b, int K, float scale, bool dense) {
  AttnShape s;
  s.B = B;
  s.Hq = Hq;
  s.Hkv = Hkv;
  s.T = T;
  s.d = d;
  s.b = b;
  s.N = (T + b - 1) / b;
  s.K = dense ? 0 : K;
  s.scale = resolve_scale(scale, d);
  s.dense = dense;
  s.outer = false;
  s.phi = SAS_PHI_SOFTMAX;
  return s;
}

bool valid_phi(int phi) {
  return phi == SAS_PHI_SOFTMAX || phi == SAS_PHI_SIGMOID || phi == SAS_PHI_RAW;
}
bool valid_gating(int g) { return g == SAS_GATE_INNER || g == SAS_GATE_OUTER; }

sas_status_t gate_topk_impl(const float* scores, int B, int Hkv, int rows, int C, int causal,
                            int K, int phi, float* gates, int32_t* idx, cudaStream_t stream) {
  if (B < 0 || Hkv < 0 || rows < 0) return SAS_ERR_INVALID_ARG;
  if (C < 0 || K < 1 || (causal != 0 && causal != 1)) return SAS_ERR_INVALID_ARG;
  if (!valid_phi(phi)) return SAS_ERR_INVALID_ARG;
  if (causal && rows != C) return SAS_ERR_INVALID_ARG;
  if (C > 262144 || K > 256) return SAS_ERR_UNSUPPORTED;
  if ((long long)B * Hkv * rows == 0) return SAS_OK;
  if (!idx || (C > 0 && (!scores || !gates))) return SAS_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(gates, 4) || !aligned(idx, 4)) return SAS_ERR_INVALID_ARG;
  if ((long long)B * Hkv * rows > (1ll << 31) - 1) return SAS_ERR_UNSUPPORTED;
  return cuda_status(launch_gate_topk(scores, B, Hkv, rows, C, causal, K, phi, gates, idx, stream));
}

sas_status_t attn_fwd_impl(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                           const int32_t* idx, const float* gates, int B, int Hq, int Hkv, int T,
                           int d, int b, int K, float scale, int gating, void* o, void* o_res,
                           float* lse, cudaStream_t stream) {
  sas_status_t st = check_attn(dtype, B, Hq, Hkv, T, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (!valid_gating(gating)) return SAS_ERR_INVALID_ARG;
  if (B == 0) return SAS_OK;
  if (!q || !k || !v || !idx || !o || !lse) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(idx, 4) || (gates && !aligned(gates, 4)))
    return SAS_ERR_INVALID_ARG;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  AttnShape s = make_shape(B, Hq, Hkv, T, d, b, K, scale, false);
  s.outer = gating == SAS_GATE_OUTER;
  if (o_res) {  // the residual output: tensor-core forward, inner gating
    if (!aligned(o_res, 16)) return SAS_ERR_INVALID_ARG;
    if (!tc_fwd_supported(dtype, s) || s.outer) return SAS_ERR_UNSUPPORTED;
  }
  if (tc_fwd_supported(dtype, s))
    return cuda_status(launch_attn_fwd_tc(s, q, k, v, idx, gates, o, o_res, lse, ctx, stream));
  return cuda_status(launch_attn_fwd_simt(dtype, s, q, k, v, idx, gates, o, lse, ctx, stream));
}

sas_status_t attn_bwd_impl(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                           const void* o, const void* o_res, const float* lse, const void* dO,
                           const int32_t* idx,
                           const float* gates, int B, int Hq, int Hkv, int T, int d, int b, int K,
                           float scale, int phi, int gating, void* dq, void* dk, void* dv,
                           float* dscores, void* ws, size_t ws_bytes, cudaStream_t stream) {
  sas_status_t st = check_attn(dtype, B, Hq, Hkv, T, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (!valid_phi(phi) || !valid_gating(gating)) return SAS_ERR_INVALID_ARG;
  if (B == 0) return SAS_OK;
  if (!q || !k || !v || !o || !lse || !dO || !idx || !dq || !dk || !dv)
    return SAS_ERR_INVALID_ARG;
  if (!gates && dscores) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dO, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(idx, 4) || (gates && !aligned(gates, 4)) ||
      (dscores && !aligned(dscores, 4)))
    return SAS_ERR_INVALID_ARG;
  AttnShape s = make_shape(B, Hq, Hkv, T, d, b, K, scale, false);
  s.outer = gating == SAS_GATE_OUTER;
  s.phi = phi;
  if (o_res) {  // D from o and the forward's residual: tensor-core path, inner gating
    if (!aligned(o_res, 16)) return SAS_ERR_INVALID_ARG;
    if (!tc_bwd_supported(dtype, s) || s.outer) return SAS_ERR_UNSUPPORTED;
  }
  const size_t need = bwd_workspace_layout(s, tc_bwd_supported(dtype, s)).total;
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  if (tc_bwd_supported(dtype, s))
    return cuda_status(launch_attn_bwd_tc(s, q, k, v, o, o_res, lse, dO, idx, gates, dq, dk, dv,
                                          dscores, ws, ctx, stream));
  return cuda_status(launch_attn_bwd_simt(dtype, s, q, k, v, o, lse, dO, idx, gates, dq, dk, dv,
                                          dscores, ws, ctx, stream));
}

sas_status_t check_decode(sas_dtype_t dt, int B, int Hq, int Hkv, int L, int Lcap, int d, int b,
                          int K, bool dense, float scale) {
  if (!valid_dtype(dt)) return SAS_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || L < 1 || Lcap < L || d < 1 || b < 1)
    return SAS_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SAS_ERR_INVALID_ARG;
  if (!dense && K < 1) return SAS_ERR_INVALID_ARG;
  if (!isfinite(scale)) return SAS_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAS_ERR_UNSUPPORTED;
  if (b != 16 && b != 32 && b != 64) return SAS_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return SAS_ERR_UNSUPPORTED;
  if (!dense && K > 256) return SAS_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return SAS_ERR_UNSUPPORTED;
  return SAS_OK;
}

DecodeShape make_decode(int B, int Hq, int Hkv, int L, int Lcap, int d, int b, int K, float scale,
                        bool dense, int use_gates) {
  DecodeShape s;
  s.B = B;
  s.Hq = Hq;
  s.Hkv = Hkv;
  s.L = L;
  s.Lcap = Lcap;
  s.d = d;
  s.b = b;
  s.K = dense ? 0 : K;
  s.scale = resolve_scale(scale, d);
  s.C = (L - 1) / b;
  s.dense = dense;
  s.use_gates = dense ? 0 : (use_gates != 0);
  s.paged = false;
  decode_plan(s);
  return s;
}

__global__ void wait_selftest_kernel(DevCtx ctx) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(ctx, &bar, 0);  // nothing ever arrives
}

}  // namespace

void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

cudaError_t launch_wait_selftest(const DevCtx& ctx, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(ctx);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace sas

using namespace sas;

extern "C" {

const char* sas_status_string(sas_status_t s) {
  switch (s) {
    case SAS_OK: return "SAS_OK";
    case SAS_ERR_INVALID_ARG: return "SAS_ERR_INVALID_ARG";
    case SAS_ERR_UNSUPPORTED: return "SAS_ERR_UNSUPPORTED";
    case SAS_ERR_CUDA: return "SAS_ERR_CUDA";
    case SAS_ERR_TIMEOUT: return "SAS_ERR_TIMEOUT";
    case SAS_ERR_WORKSPACE: return "SAS_ERR_WORKSPACE";
    case SAS_ERR_DEVICE: return "SAS_ERR_DEVICE";
  }
  return "SAS_ERR_UNKNOWN";
}

int sas_version(void) { return 100; }

uint64_t sas_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void sas_set_wait_limit(uint64_t iterations) {
  g_wait_limit.store(iterations ? iterations : kDefaultWaitLimit, std::memory_order_relaxed);
}

sas_status_t sas_get_device_error(sas_stream_t stream, uint32_t* raw) {
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SAS_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ctx.err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAS_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpy(ctx.err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return SAS_ERR_CUDA;
  if (raw) *raw = v;
  if (v & kDevErrTimeout) return SAS_ERR_TIMEOUT;
  if (v) return SAS_ERR_DEVICE;
  return SAS_OK;
}

sas_status_t sas_selftest_wait_timeout(sas_stream_t stream) {
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  return cuda_status(launch_wait_selftest(ctx, stream));
}

sas_status_t sas_gate_topk(const float* scores, int B, int Hkv, int rows, int C, int causal,
                           int K, float* gates, int32_t* idx, sas_stream_t stream) {
  return gate_topk_impl(scores, B, Hkv, rows, C, causal, K, SAS_PHI_SOFTMAX, gates, idx, stream);
}

sas_status_t sas_gate_topk_phi(const float* scores, int B, int Hkv, int rows, int C, int causal,
                               int K, sas_phi_t phi, float* gates, int32_t* idx,
                               sas_stream_t stream) {
  return gate_topk_impl(scores, B, Hkv, rows, C, causal, K, (int)phi, gates, idx, stream);
}

sas_status_t sas_attn_fwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                          const int32_t* idx, const float* gates, int B, int Hq, int Hkv, int T,
                          int d, int b, int K, float scale, void* o, float* lse,
                          sas_stream_t stream) {
  return attn_fwd_impl(dtype, q, k, v, idx, gates, B, Hq, Hkv, T, d, b, K, scale, SAS_GATE_INNER,
                       o, nullptr, lse, stream);
}

sas_status_t sas_attn_fwd_gated(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                                int T, int d, int b, int K, float scale, sas_gating_t gating,
                                void* o, float* lse, sas_stream_t stream) {
  return attn_fwd_impl(dtype, q, k, v, idx, gates, B, Hq, Hkv, T, d, b, K, scale, (int)gating, o,
                       nullptr, lse, stream);
}

size_t sas_attn_bwd_workspace_size(sas_dtype_t dtype, int B, int Hq, int Hkv, int T, int d, int b,
                                   int K) {
  if (check_attn(dtype, B, Hq, Hkv, T, d, b, K, false, 1.f) != SAS_OK) return 0;
  const AttnShape s = make_shape(B, Hq, Hkv, T, d, b, K, 1.f, false);
  return bwd_workspace_layout(s, tc_bwd_supported(dtype, s)).total;
}

sas_status_t sas_attn_bwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dO, const int32_t* idx,
                          const float* gates, int B, int Hq, int Hkv, int T, int d, int b, int K,
                          float scale, void* dq, void* dk, void* dv, float* dscores, void* ws,
                          size_t ws_bytes, sas_stream_t stream) {
  return attn_bwd_impl(dtype, q, k, v, o, nullptr, lse, dO, idx, gates, B, Hq, Hkv, T, d, b, K,
                       scale, SAS_PHI_SOFTMAX, SAS_GATE_INNER, dq, dk, dv, dscores, ws, ws_bytes,
                       stream);
}

sas_status_t sas_attn_bwd_gated(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dO,
                                const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                                int T, int d, int b, int K, float scale, sas_phi_t phi,
                                sas_gating_t gating, void* dq, void* dk, void* dv,
                                float* dscores, void* ws, size_t ws_bytes, sas_stream_t stream) {
  return attn_bwd_impl(dtype, q, k, v, o, nullptr, lse, dO, idx, gates, B, Hq, Hkv, T, d, b, K,
                       scale, (int)phi, (int)gating, dq, dk, dv, dscores, ws, ws_bytes, stream);
}

sas_status_t sas_attn_fwd_res(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* gates, int B, int Hq, int Hkv, int T,
                              int d, int b, int K, float scale, void* o, void* o_res, float* lse,
                              sas_stream_t stream) {
  if (!o_res && B > 0) return SAS_ERR_INVALID_ARG;
  return attn_fwd_impl(dtype, q, k, v, idx, gates, B, Hq, Hkv, T, d, b, K, scale, SAS_GATE_INNER,
                       o, o_res, lse, stream);
}

sas_status_t sas_attn_bwd_res(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                              const void* o, const void* o_res, const float* lse, const void* dO,
                              const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                              int T, int d, int b, int K, float scale, void* dq, void* dk, void* dv,
                              float* dscores, void* ws, size_t ws_bytes, sas_stream_t stream) {
  if (!o_res && B > 0) return SAS_ERR_INVALID_ARG;
  return attn_bwd_impl(dtype, q, k, v, o, o_res, lse, dO, idx, gates, B, Hq, Hkv, T, d, b, K,
                       scale, SAS_PHI_SOFTMAX, SAS_GATE_INNER, dq, dk, dv, dscores, ws, ws_bytes,
                       stream);
}

size_t sas_decode_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K) {
  if (check_decode(SAS_BF16, B, Hq, Hkv, L, L, d, b, K, false, 1.f) != SAS_OK) return 0;
  return decode_workspace_bytes(make_decode(B, Hq, Hkv, L, L, d, b, K, 1.f, false, 0));
}

sas_status_t sas_decode(sas_dtype_t dtype, const void* q, const void* kcache, const void* vcache,
                        const int32_t* idx, const float* gates, int use_gates, int B, int Hq,
                        int Hkv, int L, int Lcap, int d, int b, int K, float scale, void* o,
                        void* ws, size_t ws_bytes, sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hq, Hkv, L, Lcap, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !kcache || !vcache || !idx || !o) return SAS_ERR_INVALID_ARG;
  if (use_gates && !gates && (L - 1) / b > 0) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16) ||
      !aligned(idx, 4) || (gates && !aligned(gates, 4)))
    return SAS_ERR_INVALID_ARG;
  const DecodeShape s = make_decode(B, Hq, Hkv, L, Lcap, d, b, K, scale, false, use_gates);
  if (s.splits > 1 && (!ws || ws_bytes < decode_workspace_bytes(s) || !aligned(ws, 256)))
    return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  return cuda_status(launch_decode(dtype, s, q, kcache, vcache, idx, gates, o, ws, ctx, stream));
}

// Workspace of sas_decode_select: the decode's, then room for the gates and
// the Top-K indices when the caller does not keep them and the selection
// runs as its own launch.
static size_t select_ws_parts(const DecodeShape& s, size_t* off_g, size_t* off_i) {
  const size_t a = (decode_workspace_bytes(s) + 255) & ~(size_t)255;
  const size_t g = ((size_t)s.B * s.Hkv * s.C * sizeof(float) + 255) & ~(size_t)255;
  const size_t i = ((size_t)s.B * s.Hkv * s.K * sizeof(int32_t) + 255) & ~(size_t)255;
  *off_g = a;
  *off_i = a + g;
  return a + g + i;
}

size_t sas_decode_select_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K) {
  if (check_decode(SAS_BF16, B, Hq, Hkv, L, L, d, b, K, false, 1.f) != SAS_OK) return 0;
  size_t og, oi;
  return select_ws_parts(make_decode(B, Hq, Hkv, L, L, d, b, K, 1.f, false, 0), &og, &oi);
}

// The fused step and its two-launch fallback. kbar (nullable): the scores
// are the pooled selector's, formed in the launch (or, on the fallback, by
// the selector kernel into the workspace's scores part at off_s).
static sas_status_t decode_select_impl(sas_dtype_t dtype, const void* q, const void* kcache,
                                       const void* vcache, const float* scores, const float* kbar,
                                       float sel_scale, size_t off_s, int use_gates, int B,
                                       int Hq, int Hkv, int L, int Lcap, int d, int b, int K,
                                       float scale, void* o, float* gates, int32_t* idx, void* ws,
                                       size_t ws_bytes, sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hq, Hkv, L, Lcap, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  const int C = (L - 1) / b;
  if (!q || !kcache || !vcache || !o || (!scores && !kbar && C > 0)) return SAS_ERR_INVALID_ARG;
  if (C > 262144) return SAS_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16) ||
      (scores && !aligned(scores, 4)) || (kbar && !aligned(kbar, 4)) ||
      (gates && !aligned(gates, 4)) || (idx && !aligned(idx, 4)))
    return SAS_ERR_INVALID_ARG;
  const DecodeShape s = make_decode(B, Hq, Hkv, L, Lcap, d, b, K, scale, false, use_gates);
  size_t og, oi;
  const size_t need = select_ws_parts(s, &og, &oi) +
                      (kbar ? (((size_t)B * Hkv * C * sizeof(float) + 255) & ~(size_t)255) : 0);
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  if (tc_decode_supported(dtype, s) && (!kbar || aligned(kbar, 16))) {
    const cudaError_t e = launch_decode_select_tc(s, q, kcache, vcache, scores, kbar, sel_scale,
                                                  gates, idx, o, ws, ctx, stream);
    if (e != cudaErrorNotSupported) return cuda_status(e);
  }
  // Two or three launches: the pooled selector's scores (when asked for),
  // the gates and Top-K of the rows, then the decode.
  if (kbar && C > 0) {
    float* sc = reinterpret_cast<float*>(static_cast<char*>(ws) + off_s);
    const cudaError_t e = launch_selector_scores_decode(dtype, q, kbar, B * Hkv, Hq / Hkv, C, d,
                                                        sel_scale, sc, stream);
    if (e != cudaSuccess) return cuda_status(e);
    scores = sc;
  }
  float* g = gates ? gates : reinterpret_cast<float*>(static_cast<char*>(ws) + og);
  int32_t* ix = idx ? idx : reinterpret_cast<int32_t*>(static_cast<char*>(ws) + oi);
  cudaError_t e = launch_gate_topk(scores, B, Hkv, 1, C, 0, K, SAS_PHI_SOFTMAX, g, ix, stream);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_decode(dtype, s, q, kcache, vcache, ix, g, o, ws, ctx, stream));
}

sas_status_t sas_decode_select(sas_dtype_t dtype, const void* q, const void* kcache,
                               const void* vcache, const float* scores, int use_gates, int B,
                               int Hq, int Hkv, int L, int Lcap, int d, int b, int K, float scale,
                               void* o, float* gates, int32_t* idx, void* ws, size_t ws_bytes,
                               sas_stream_t stream) {
  return decode_select_impl(dtype, q, kcache, vcache, scores, nullptr, 0.f, 0, use_gates, B, Hq,
                            Hkv, L, Lcap, d, b, K, scale, o, gates, idx, ws, ws_bytes, stream);
}

size_t sas_decode_select_pooled_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K) {
  if (check_decode(SAS_BF16, B, Hq, Hkv, L, L, d, b, K, false, 1.f) != SAS_OK) return 0;
  size_t og, oi;
  const DecodeShape s = make_decode(B, Hq, Hkv, L, L, d, b, K, 1.f, false, 0);
  return select_ws_parts(s, &og, &oi) +
         (((size_t)B * Hkv * s.C * sizeof(float) + 255) & ~(size_t)255);
}

sas_status_t sas_decode_select_pooled(sas_dtype_t dtype, const void* q, const void* kcache,
                                      const void* vcache, const float* kbar, float sel_scale,
                                      int use_gates, int B, int Hq, int Hkv, int L, int Lcap, int d,
                                      int b, int K, float scale, void* o, float* gates,
                                      int32_t* idx, void* ws, size_t ws_bytes,
                                      sas_stream_t stream) {
  const sas_status_t st = check_decode(dtype, B, Hq, Hkv, L, Lcap, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (!isfinite(sel_scale)) return SAS_ERR_INVALID_ARG;
  if (B == 0) return SAS_OK;
  if ((L - 1) / b > 0 && !kbar) return SAS_ERR_INVALID_ARG;
  if ((long long)B * Hkv > 65535) return SAS_ERR_UNSUPPORTED;  // the selector kernel's grid
  size_t og, oi;
  const size_t off_s = select_ws_parts(make_decode(B, Hq, Hkv, L, Lcap, d, b, K, 1.f, false, 0),
                                       &og, &oi);
  return decode_select_impl(dtype, q, kcache, vcache, nullptr, kbar, resolve_scale(sel_scale, d),
                            off_s, use_gates, B, Hq, Hkv, L, Lcap, d, b, K, scale, o, gates, idx,
                            ws, ws_bytes, stream);
}

sas_status_t sas_decode_noalloc(sas_dtype_t dtype, const void* q, const void* kcache,
                                const void* vcache, const int32_t* idx, const float* gates,
                                int use_gates, int B, int Hq, int Hkv, int L, int Lcap, int d,
                                int b, int K, float scale, void* o, sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hq, Hkv, L, Lcap, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !kcache || !vcache || !idx || !o) return SAS_ERR_INVALID_ARG;
  if (use_gates && !gates && (L - 1) / b > 0) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16) ||
      !aligned(idx, 4) || (gates && !aligned(gates, 4)))
    return SAS_ERR_INVALID_ARG;
  const DecodeShape s = make_decode(B, Hq, Hkv, L, Lcap, d, b, K, scale, false, use_gates);
  void* scratch = nullptr;
  if (s.splits > 1) {
    if (decode_workspace_bytes(s) > decode_noalloc_capacity()) return SAS_ERR_WORKSPACE;
    if (decode_noalloc_scratch(&scratch) != cudaSuccess) return SAS_ERR_CUDA;
  }
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  return cuda_status(
      launch_decode(dtype, s, q, kcache, vcache, idx, gates, o, scratch, ctx, stream));
}

size_t sas_decode_noalloc_max_scratch(void) { return decode_noalloc_capacity(); }

size_t sas_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_len, int d, int b, int K) {
  return sas_decode_workspace_size(B, Hq, Hkv, max_len, d, b, K);
}

sas_status_t sas_decode_paged(sas_dtype_t dtype, const void* q, const void* kpages,
                              const void* vpages, const int32_t* page_indptr,
                              const int32_t* page_indices, const int32_t* seq_lens,
                              const int32_t* idx, const float* gates, int use_gates, int B, int Hq,
                              int Hkv, int num_pages, int page_size, int max_len, int d, int b,
                              int K, float scale, void* o, void* ws, size_t ws_bytes,
                              sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hq, Hkv, max_len, max_len, d, b, K, false, scale);
  if (st != SAS_OK) return st;
  if (num_pages < 1 || page_size < 1) return SAS_ERR_INVALID_ARG;
  if (page_size < 16 || (page_size & (page_size - 1)) != 0 || page_size > (1 << 20))
    return SAS_ERR_UNSUPPORTED;
  if ((long long)num_pages * Hkv > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;
  if (dtype != SAS_BF16 || d != 128 || b != 64) return SAS_ERR_UNSUPPORTED;
  if (B == 0) return SAS_OK;
  if (!q || !kpages || !vpages || !page_indptr || !page_indices || !seq_lens || !idx || !o)
    return SAS_ERR_INVALID_ARG;
  if (use_gates && !gates && (max_len - 1) / b > 0) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kpages, 16) || !aligned(vpages, 16) || !aligned(o, 16) ||
      !aligned(idx, 4) || !aligned(page_indptr, 4) || !aligned(page_indices, 4) ||
      !aligned(seq_lens, 4) || (gates && !aligned(gates, 4)))
    return SAS_ERR_INVALID_ARG;
  DecodeShape s = make_decode(B, Hq, Hkv, max_len, max_len, d, b, K, scale, false, use_gates);
  s.paged = true;
  if (!tc_decode_supported(dtype, s)) return SAS_ERR_UNSUPPORTED;
  if (s.splits > 1 && (!ws || ws_bytes < decode_workspace_bytes(s) || !aligned(ws, 256)))
    return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  const PagedArgs pa = {page_indptr, page_indices, seq_lens, page_size, num_pages};
  return cuda_status(
      launch_decode_paged_tc(s, pa, q, kpages, vpages, idx, gates, o, ws, ctx, stream));
}

size_t sas_selector_workspace_size(int B, int Hkv, int T, int d, int b) {
  if (B < 0 || Hkv < 1 || T < 1 || (d != 64 && d != 128) || b < 1) return 0;
  const size_t N = ((size_t)T + b - 1) / b;
  return 2 * ((sizeof(float) * (size_t)B * Hkv * N * d + 255) & ~(size_t)255);
}

sas_status_t sas_selector_scores(sas_dtype_t dtype, const void* q, const void* k, int B, int Hq,
                                 int Hkv, int T, int d, int b, float scale, float* scores,
                                 void* ws, size_t ws_bytes, sas_stream_t stream) {
  sas_status_t st = check_attn(dtype, B, Hq, Hkv, T, d, b, 1, false, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !k || !scores) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(scores, 4)) return SAS_ERR_INVALID_ARG;
  if ((long long)B * Hkv > 65535) return SAS_ERR_UNSUPPORTED;  // grid dimension
  const size_t need = sas_selector_workspace_size(B, Hkv, T, d, b);
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  const int N = (T + b - 1) / b;
  float* qbar = static_cast<float*>(ws);
  float* kbar = reinterpret_cast<float*>(static_cast<char*>(ws) + need / 2);
  const int G = Hq / Hkv;
  cudaError_t e = launch_block_summaries(dtype, q, B * Hkv, G, T, T, b, N, d, qbar, stream);
  if (e == cudaSuccess)
    e = launch_block_summaries(dtype, k, B * Hkv, 1, T, T, b, N, d, kbar, stream);
  if (e == cudaSuccess)
    e = launch_selector_scores(qbar, kbar, B * Hkv, N, d, resolve_scale(scale, d), scores,
                               stream);
  return cuda_status(e);
}

sas_status_t sas_block_summaries(sas_dtype_t dtype, const void* kcache, int B, int Hkv, int L,
                                 int Lcap, int d, int b, float* kbar, sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hkv, Hkv, L, Lcap, d, b, 1, false, 1.f);
  if (st != SAS_OK) return st;
  const int C = (L - 1) / b;
  if (B == 0 || C == 0) return SAS_OK;
  if (!kcache || !kbar) return SAS_ERR_INVALID_ARG;
  if (!aligned(kcache, 16) || !aligned(kbar, 4)) return SAS_ERR_INVALID_ARG;
  if ((long long)B * Hkv > 65535) return SAS_ERR_UNSUPPORTED;  // grid dimension
  return cuda_status(
      launch_block_summaries(dtype, kcache, B * Hkv, 1, C * b, Lcap, b, C, d, kbar, stream));
}

sas_status_t sas_selector_scores_decode(sas_dtype_t dtype, const void* q, const float* kbar, int B,
                                        int Hq, int Hkv, int C, int d, float scale, float* scores,
                                        sas_stream_t stream) {
  if (!valid_dtype(dtype)) return SAS_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || C < 0 || Hq % Hkv != 0 || !isfinite(scale))
    return SAS_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAS_ERR_UNSUPPORTED;
  if (B > 65535 || (long long)B * Hkv > 65535) return SAS_ERR_UNSUPPORTED;
  if (B == 0 || C == 0) return SAS_OK;
  if (!q || !kbar || !scores) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kbar, 4) || !aligned(scores, 4)) return SAS_ERR_INVALID_ARG;
  return cuda_status(launch_selector_scores_decode(dtype, q, kbar, B * Hkv, Hq / Hkv, C, d,
                                                   resolve_scale(scale, d), scores, stream));
}

sas_status_t sas_dense_fwd(sas_dtype_t dtype, const void* q, const void* k, const void* v, int B,
                           int Hq, int Hkv, int T, int d, int b, float scale, void* o, float* lse,
                           sas_stream_t stream) {
  sas_status_t st = check_attn(dtype, B, Hq, Hkv, T, d, b, 0, true, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !k || !v || !o || !lse) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return SAS_ERR_INVALID_ARG;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  const AttnShape s = make_shape(B, Hq, Hkv, T, d, b, 0, scale, true);
  if (tc_fwd_supported(dtype, s))
    return cuda_status(launch_attn_fwd_tc(s, q, k, v, nullptr, nullptr, o, nullptr, lse, ctx,
                                          stream));
  return cuda_status(launch_attn_fwd_simt(dtype, s, q, k, v, nullptr, nullptr, o, lse, ctx, stream));
}

size_t sas_dense_bwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int b) {
  if (check_attn(SAS_BF16, B, Hq, Hkv, T, d, b, 0, true, 1.f) != SAS_OK) return 0;
  // The general layout covers the tensor-core one (D first, no dS tiles).
  return bwd_workspace_layout(make_shape(B, Hq, Hkv, T, d, b, 0, 1.f, true), false).total;
}

sas_status_t sas_dense_bwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                           const void* o, const float* lse, const void* dO, int B, int Hq, int Hkv,
                           int T, int d, int b, float scale, void* dq, void* dk, void* dv,
                           void* ws, size_t ws_bytes, sas_stream_t stream) {
  sas_status_t st = check_attn(dtype, B, Hq, Hkv, T, d, b, 0, true, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dO, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4))
    return SAS_ERR_INVALID_ARG;
  const AttnShape s = make_shape(B, Hq, Hkv, T, d, b, 0, scale, true);
  const size_t need = bwd_workspace_layout(s, false).total;
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  if (tc_bwd_supported(dtype, s))
    return cuda_status(launch_attn_bwd_tc(s, q, k, v, o, nullptr, lse, dO, nullptr, nullptr, dq, dk, dv,
                                          nullptr, ws, ctx, stream));
  return cuda_status(launch_attn_bwd_simt(dtype, s, q, k, v, o, lse, dO, nullptr, nullptr, dq, dk,
                                          dv, nullptr, ws, ctx, stream));
}

size_t sas_dense_decode_workspace_size(int B, int Hq, int Hkv, int L, int d) {
  if (check_decode(SAS_BF16, B, Hq, Hkv, L, L, d, 64, 0, true, 1.f) != SAS_OK) return 0;
  return decode_workspace_bytes(make_decode(B, Hq, Hkv, L, L, d, 64, 0, 1.f, true, 0));
}

sas_status_t sas_dense_decode(sas_dtype_t dtype, const void* q, const void* kcache,
                              const void* vcache, int B, int Hq, int Hkv, int L, int Lcap, int d,
                              float scale, void* o, void* ws, size_t ws_bytes,
                              sas_stream_t stream) {
  sas_status_t st = check_decode(dtype, B, Hq, Hkv, L, Lcap, d, 64, 0, true, scale);
  if (st != SAS_OK) return st;
  if (B == 0) return SAS_OK;
  if (!q || !kcache || !vcache || !o) return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16))
    return SAS_ERR_INVALID_ARG;
  const DecodeShape s = make_decode(B, Hq, Hkv, L, Lcap, d, 64, 0, scale, true, 0);
  if (s.splits > 1 && (!ws || ws_bytes < decode_workspace_bytes(s) || !aligned(ws, 256)))
    return SAS_ERR_WORKSPACE;
  DevCtx ctx;
  if (device_ctx(ctx) != cudaSuccess) return SAS_ERR_CUDA;
  return cuda_status(
      launch_decode(dtype, s, q, kcache, vcache, nullptr, nullptr, o, ws, ctx, stream));
}

}  // extern "C"
