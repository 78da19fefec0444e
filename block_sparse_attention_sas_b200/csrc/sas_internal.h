// Internal launchers of the SAS library. Each returns the CUDA error of its
// launches (cudaSuccess when everything was enqueued). Arguments are already
// validated by the C-ABI layer (sas_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sas.h"

namespace sas {

struct DevCtx;

// Adds n to the library's launch counter (sas_launch_count).
void note_launches(int n);

// phi: a sas_phi_t value.
cudaError_t launch_gate_topk(const float* scores, int B, int Hkv, int rows, int C, int causal,
                             int K, int phi, float* gates, int32_t* idx, cudaStream_t stream);

// Problem description shared by the attention launchers.
struct AttnShape {
  int B, Hq, Hkv, T, d, b, K;
  float scale;   // already resolved (> 0)
  int N;         // ceil(T / b)
  bool dense;    // every history block, no idx / gates
  bool outer;    // outer gating (gate after the softmax); inner otherwise
  int phi;       // gate activation (sas_phi_t) for the d scores Jacobian
};

// Workspace carve-up of the backward pass (byte offsets, 256-aligned).
struct BwdWorkspace {
  size_t off_D, off_da, off_csr_off, off_csr_list, off_order, off_ds, total;
};
// `tc`: the tensor-core backward runs (it adds the stored dS tiles and keeps
// da in four row chunks per head).
BwdWorkspace bwd_workspace_layout(const AttnShape& s, bool tc);

cudaError_t launch_attn_fwd_simt(sas_dtype_t dt, const AttnShape& s, const void* q, const void* k,
                                 const void* v, const int32_t* idx, const float* gates, void* o,
                                 float* lse, const DevCtx& ctx, cudaStream_t stream);
// Tensor-core (tcgen05) forward: bf16, d = 128, b = 64, G in {2, 4}.
bool tc_fwd_supported(sas_dtype_t dt, const AttnShape& s);
// o_res (nullable, inner gating only): the forward also writes o's bf16
// residual o_fp32 - o, with P split in two bf16 terms in the PV product.
cudaError_t launch_attn_fwd_tc(const AttnShape& s, const void* q, const void* k, const void* v,
                               const int32_t* idx, const float* gates, void* o, void* o_res,
                               float* lse, const DevCtx& ctx, cudaStream_t stream);

// Tensor-core (tcgen05) backward for the same shapes as the forward.
bool tc_bwd_supported(sas_dtype_t dt, const AttnShape& s);
// o / o_res (both or neither): D = dO . (o + o_res) in one memory-bound pass
// instead of the exact recomputation (inner gating).
cudaError_t launch_attn_bwd_tc(const AttnShape& s, const void* q, const void* k, const void* v,
                               const void* o, const void* o_res, const float* lse, const void* dO,
                               const int32_t* idx, const float* gates, void* dq, void* dk, void* dv,
                               float* dscores, void* ws, const DevCtx& ctx, cudaStream_t stream);
// Shared pieces of the backward (defined with the SIMT kernels).
cudaError_t launch_bwd_csr(const AttnShape& s, const int32_t* idx, int32_t* off, int32_t* list,
                           const DevCtx& ctx, cudaStream_t stream);
// da holds RC row chunks per (head, query block, slot); s.phi picks the
// Jacobian of the gate activation.
cudaError_t launch_bwd_jacobian(const AttnShape& s, const float* da, const int32_t* idx,
                                const float* gates, float* dscores, int RC, cudaStream_t stream);
// 3-D TMA map over a [planes][rows][128] bf16 tensor, 64x64 boxes, 128-byte swizzle.
cudaError_t make_tmap_bf16(void* map, const void* ptr, int rows, int planes);

cudaError_t launch_attn_bwd_simt(sas_dtype_t dt, const AttnShape& s, const void* q, const void* k,
                                 const void* v, const void* o, const float* lse, const void* dO,
                                 const int32_t* idx, const float* gates, void* dq, void* dk,
                                 void* dv, float* dscores, void* ws, const DevCtx& ctx,
                                 cudaStream_t stream);

// Decode (sparse and dense).
struct DecodeShape {
  int B, Hq, Hkv, L, Lcap, d, b, K;
  float scale;
  int C;        // (L - 1) / b history blocks
  bool dense;   // all blocks 0..C, no idx / gates
  int use_gates;
  int splits;   // CTAs per (batch, kv head)
  int bps;      // blocks per split
  bool cluster; // (tensor-core decode) a unit's splits form one cluster
  bool paged;   // the cache is paged (L = the longest sequence, C its history)
};

// Page table of a paged KV cache: sequence bi owns the pages
// indices[indptr[bi] .. indptr[bi + 1]) in logical order and has lens[bi]
// tokens; token t sits at row t % P of its (t / P)-th page.
struct PagedArgs {
  const int32_t* indptr;
  const int32_t* indices;
  const int32_t* lens;
  int P;          // tokens per page: a power of two, at least 16
  int num_pages;
};
void decode_plan(DecodeShape& s);  // fills splits / bps
size_t decode_workspace_bytes(const DecodeShape& s);
cudaError_t launch_decode(sas_dtype_t dt, const DecodeShape& s, const void* q, const void* kc,
                          const void* vc, const int32_t* idx, const float* gates, void* o,
                          void* ws, const DevCtx& ctx, cudaStream_t stream);

// Tensor-core (tcgen05) decode: bf16 cache, d = 128, b = 64, G <= 8.
bool tc_decode_supported(sas_dtype_t dt, const DecodeShape& s);
// The tensor-core decode with the gates and Top-K of the unit's selector
// scores [B * Hkv][C] computed in the same launch (softmax gates); gates_out /
// idx_out may be null. cudaErrorNotSupported when the shape does not allow
// it (a unit's row must fit its splits' cluster, 512 entries a split).
// kbar (nullable, with sel_scale): the scores come from the pooled selector
// in the same launch (scores is then unused).
cudaError_t launch_decode_select_tc(const DecodeShape& s, const void* q, const void* kc,
                                    const void* vc, const float* scores, const float* kbar,
                                    float sel_scale, float* gates_out, int32_t* idx_out, void* o,
                                    void* ws, const DevCtx& ctx, cudaStream_t st);
cudaError_t launch_decode_tc(const DecodeShape& s, const void* q, const void* kc, const void* vc,
                             const int32_t* idx, const float* gates, void* o, void* ws,
                             const DevCtx& ctx, cudaStream_t stream);
// The same over a paged cache (s.paged; kpages / vpages [num_pages, Hkv, P, d]).
cudaError_t launch_decode_paged_tc(const DecodeShape& s, const PagedArgs& pa, const void* q,
                                   const void* kpages, const void* vpages, const int32_t* idx,
                                   const float* gates, void* o, void* ws, const DevCtx& ctx,
                                   cudaStream_t stream);
// The same map with 64 x 64 x 2 boxes (two consecutive planes per box).
cudaError_t make_tmap_bf16_2planes(void* map, const void* ptr, int rows, int planes);
// 3-D TMA map over planes of `pitch_rows` rows, the first `rows` of each mapped.
cudaError_t make_tmap_bf16_rows8(void* map_out, const void* ptr, int rows);
cudaError_t make_tmap_bf16_pitched(void* map, const void* ptr, int rows, int pitch_rows,
                                   int planes);
// Map over [planes][rows][128] bf16 with 64 x box_rows x 1 boxes (pages).
cudaError_t make_tmap_bf16_box(void* map, const void* ptr, int rows, int planes, int box_rows);
// Fixed-size device scratch for sas_decode_noalloc (no allocation involved).
size_t decode_noalloc_capacity();
cudaError_t decode_noalloc_scratch(void** out);

cudaError_t launch_wait_selftest(const DevCtx& ctx, cudaStream_t stream);

// Block-selector scores (selector.cu). Summaries: mean over each block's rows
// of `group` consecutive planes ([planes_out * group][pitch rows][d], the
// first `rows` valid) into out [planes_out][N][d] fp32.
cudaError_t launch_block_summaries(sas_dtype_t dt, const void* x, int planes_out, int group,
                                   int rows, int pitch, int b, int N, int d, float* out,
                                   cudaStream_t st);
cudaError_t launch_selector_scores(const float* qbar, const float* kbar, int units, int N, int d,
                                   float scale, float* scores, cudaStream_t st);
cudaError_t launch_selector_scores_decode(sas_dtype_t dt, const void* q, const float* kbar,
                                          int units, int G, int C, int d, float scale,
                                          float* scores, cudaStream_t st);

}  // namespace sas
