/*
 * sas.h - C ABI of a CUDA library (NVIDIA B200, sm_100a) for SAS gated
 * block-sparse causal attention.
 *
 * Sources (by page and section; the pages print no code for this path):
 *   [picx]   picx.dev summary of "SAS: Simple Attention Sparsification via
 *            End-to-End Optimization of Context Ranking": Theoretical
 *            Foundation (Eq. 1-3), Methodology (Eq. 4, Eq. 9), Gradient
 *            Analysis (Eq. 5, Eq. 6), Kernel Design, Decode Efficiency (Fig. 7).
 *   [readme] "SAS: End-to-end learning of sparse attention rankings from
 *            language-model loss" (reproduction README): Core equations,
 *            the only statement of the 1/sqrt(d) scale.
 *   [review] evolve.pub review of the same paper: Summary (gates dropped at
 *            inference, hard selection kept).
 *
 * Notation. B batch, Hq query heads, Hkv KV heads, G = Hq/Hkv query heads per
 * KV head, T sequence length, d head dim, b block size (tokens per block),
 * N = ceil(T/b) blocks, K history budget in blocks. Query block j has the
 * history blocks 0..j-1; its "current block" is block j itself, always
 * attended with a causal mask and gate g0 = 1 ([picx] Eq. 4). Block j selects
 * n_j = min(K, j) history blocks.
 *
 * Conventions shared by every call:
 *   - Every tensor argument is a DEVICE pointer owned by the caller, dense
 *     row-major in the layout stated, 16-byte aligned. The library never
 *     allocates memory the caller can see; scratch comes from the caller's
 *     workspace (see the *_workspace_size calls).
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream) and returns after enqueueing its kernels.
 *   - Argument errors are detected on the host before any launch and return
 *     SAS_ERR_INVALID_ARG / SAS_ERR_UNSUPPORTED / SAS_ERR_WORKSPACE; nothing is
 *     launched in that case. A failed launch returns SAS_ERR_CUDA. Errors
 *     found on the device (a bounded wait that ran out, an index out of
 *     range) set a per-device error word that sas_get_device_error reports;
 *     the kernel that found them stops early and leaves its outputs undefined.
 *   - dtype: q, k, v, o, dO, dq, dk, dv, kcache, vcache share one dtype
 *     (SAS_F32 or SAS_BF16). scores, gates, lse, dscores are always fp32;
 *     idx is int32. bf16 paths accumulate in fp32.
 *   - scale <= 0 selects 1/sqrt(d) ([readme] Core equations). The scale
 *     multiplies q.k only; log g is added unscaled.
 *   - Limits: d in {64, 128}; b in {16, 32, 64}; 1 <= K <= 256;
 *     Hq % Hkv == 0; G = Hq/Hkv <= 8 for decode; N <= 16384; T, L >= 1.
 *     The entries of one idx
 *     row must be distinct (sas_gate_topk writes them so).
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* sas_stream_t; /* the same type as cudaStream_t */

typedef enum {
  SAS_F32 = 0,
  SAS_BF16 = 1
} sas_dtype_t;

typedef enum {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size, misaligned pointer */
  SAS_ERR_UNSUPPORTED = 2, /* well-formed but outside the limits above */
  SAS_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  SAS_ERR_TIMEOUT = 4,     /* (device) a bounded wait ran out of iterations */
  SAS_ERR_WORKSPACE = 5,   /* workspace missing, too small or misaligned */
  SAS_ERR_DEVICE = 6       /* (device) a device-side check failed, e.g. idx out of range */
} sas_status_t;

/*
 * Gate variants: the two ablation axes of the method. [picx] Methodology,
 * Eq. 4 leaves the activation phi open; the [review] Summary compares the
 * method's softmax with sigmoid and raw-logit gates, and inner with outer
 * gating; [picx] Gradient Analysis, Eq. 5 gives the gate gradient of both
 * gatings. The pages print no formula for the variants; this library reads
 * them as:
 *   SAS_PHI_SOFTMAX  g = softmax(s) over the valid history (Eq. 6; the method)
 *   SAS_PHI_SIGMOID  g_m = 1 / (1 + exp(-s_m)), elementwise, not normalised
 *   SAS_PHI_RAW      log g_m = s_m (stored as g_m = exp(s_m); needs s < 88)
 *   SAS_GATE_INNER   log g enters the logits: o = softmax(q K^T scale + log g) V
 *                    (Eq. 9; the method)
 *   SAS_GATE_OUTER   the gate scales the softmax weights after normalisation:
 *                    o_i = sum_t g_{m(t)} p_it v_t with p = softmax(q K^T scale)
 *                    over the same keys (g = 1 on the current block); lse is
 *                    that of the ungated logits
 * Top-K is over the scores for every phi (each is increasing).
 */
typedef enum {
  SAS_PHI_SOFTMAX = 0,
  SAS_PHI_SIGMOID = 1,
  SAS_PHI_RAW = 2
} sas_phi_t;

typedef enum {
  SAS_GATE_INNER = 0,
  SAS_GATE_OUTER = 1
} sas_gating_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char* sas_status_string(sas_status_t status);

/* Library version as an integer MAJOR*10000 + MINOR*100 + PATCH. */
int sas_version(void);

/* Number of kernels this process has launched through the library so far
 * (all devices, all threads). Lets a caller count the launches of a region. */
uint64_t sas_launch_count(void);

/*
 * sas_gate_topk - history gates and Top-K block selection.
 *   [picx] Eq. 4 with phi = softmax and Eq. 6: log g_m = s_m - LSE(s) over the
 *   valid history entries of a row, g_m = exp(log g_m) (so they sum to 1);
 *   [picx] Eq. 3 / [readme] Core equations: I = Top-K(s, K).
 *
 *   scores [B, Hkv, rows, C] fp32 (device, read). Must be finite.
 *   causal = 1 (training): rows == C == N and row j has j valid entries
 *            (the history of query block j; entries m >= j are ignored).
 *   causal = 0 (decode):   every row has C valid entries.
 *   gates  [B, Hkv, rows, C] fp32 (device, written): g_m for valid m, 0 past
 *            the valid length (row 0 of a causal call is all zero).
 *   idx    [B, Hkv, rows, K] int32 (device, written): the min(K, valid)
 *            largest scores' block indices in rank order (descending score,
 *            equal scores ordered by lower index; -0.0 equals +0.0), padded
 *            with -1.
 *   Limits: 0 <= C <= 262144 (C = 0: no history, idx all -1; scores and
 *   gates may then be NULL), 1 <= K <= 256.
 */
sas_status_t sas_gate_topk(const float* scores, int B, int Hkv, int rows, int C, int causal,
                           int K, float* gates, int32_t* idx, sas_stream_t stream);

/*
 * sas_attn_fwd - gated block-sparse causal attention, forward.
 *   [picx] Eq. 9 with the [readme] scale: for query row i of block j,
 *   o_i = softmax(q_i K_S^T * scale + log g_S) V_S over the keys of the
 *   selected blocks S = idx[.., j, :] (bias log g_m) and the keys t <= i of
 *   block j (bias 0). With gates == NULL the bias of selected blocks is 0
 *   ([picx] Eq. 2, gates dropped).
 *
 *   q [B, Hq, T, d]; k, v [B, Hkv, T, d] (dtype; read).
 *   idx [B, Hkv, N, K] int32: entries -1 are skipped; every other entry of
 *     row j must satisfy 0 <= m < j (checked on the device: an entry >= j or
 *     below -1 is skipped and reported as SAS_ERR_DEVICE).
 *   gates [B, Hkv, N, N] fp32 or NULL: row j holds g_{j,m} (as written by
 *     sas_gate_topk with causal = 1). A zero gate masks its block.
 *   o [B, Hq, T, d] (dtype; written); lse [B, Hq, T] fp32 (written): the
 *     natural-log normaliser of each row's softmax, needed by the backward.
 */
sas_status_t sas_attn_fwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                          const int32_t* idx, const float* gates, int B, int Hq, int Hkv, int T,
                          int d, int b, int K, float scale, void* o, float* lse,
                          sas_stream_t stream);

/*
 * sas_attn_bwd - backward of sas_attn_fwd for L = any loss with dL/do = dO.
 *   Recomputes the probabilities from lse and returns
 *     dq [B, Hq, T, d], dk, dv [B, Hkv, T, d]   (dtype; written);
 *     dscores [B, Hkv, N, N] fp32 (written; may be NULL): the gradient into
 *       the selector scores through the gate softmax. With da_{j,m} = the sum
 *       of dL/dlogit over the tile (all G heads, rows of block j, keys of
 *       block m) -- equal to g_m * dg_m of [picx] Eq. 5, inner form -- and the
 *       Jacobian of [picx] Eq. 6 (d log g_m / d s_k = delta_mk - g_k):
 *         dscores[j, k] = [k in I_j] da_{j,k} - g_{j,k} * sum_{m in I_j} da_{j,m}
 *       for k < j, and 0 for k >= j. No gradient flows through idx.
 *   q, k, v, idx, gates, scale as passed to sas_attn_fwd; o, lse its outputs;
 *   dO [B, Hq, T, d] (dtype). gates == NULL requires dscores == NULL.
 *   ws / ws_bytes: caller workspace of at least sas_attn_bwd_workspace_size()
 *   bytes for the same dtype and shape, 256-byte aligned; its contents on
 *   entry do not matter. (For bf16 with d = 128, b = 64 and G = 2 or 4 it
 *   holds the dS tiles of every attended block: B*Hkv*N*(G/2)*(K+1)*16 KB.)
 */
size_t sas_attn_bwd_workspace_size(sas_dtype_t dtype, int B, int Hq, int Hkv, int T, int d, int b,
                                   int K);
sas_status_t sas_attn_bwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dO, const int32_t* idx,
                          const float* gates, int B, int Hq, int Hkv, int T, int d, int b, int K,
                          float scale, void* dq, void* dk, void* dv, float* dscores, void* ws,
                          size_t ws_bytes, sas_stream_t stream);

/*
 * Gate-variant forms of the three training calls ([review] Summary; [picx]
 * Eq. 4 and Eq. 5; readings above). Arguments, layouts and errors are those
 * of the calls without the suffix, which are the (SAS_PHI_SOFTMAX,
 * SAS_GATE_INNER) case.
 *   sas_gate_topk_phi: gates g = phi(s) (the selection does not depend on phi).
 *   sas_attn_fwd_gated: gating selects inner (Eq. 9) or outer gating; gates
 *     as written by sas_gate_topk_phi with any phi (NULL: gates off, where
 *     both gatings are plain block-sparse attention).
 *   sas_attn_bwd_gated: the backward of sas_attn_fwd_gated with the same
 *     gating, o and lse; dscores through the Jacobian of phi:
 *       softmax: dscores[j,k] = [k in I_j] da_k - g_k sum_{m in I_j} da_m
 *       sigmoid: dscores[j,k] = [k in I_j] da_k (1 - g_k)
 *       raw:     dscores[j,k] = [k in I_j] da_k
 *     with da_m = dL/dlog g_m: the sum of dS over the tile for inner gating,
 *     the sum of g_m p dP (Eq. 5, outer form, times g_m) for outer gating.
 *     Workspace: sas_attn_bwd_workspace_size() of the same shape.
 */
sas_status_t sas_gate_topk_phi(const float* scores, int B, int Hkv, int rows, int C, int causal,
                               int K, sas_phi_t phi, float* gates, int32_t* idx,
                               sas_stream_t stream);
sas_status_t sas_attn_fwd_gated(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                                int T, int d, int b, int K, float scale, sas_gating_t gating,
                                void* o, float* lse, sas_stream_t stream);
sas_status_t sas_attn_bwd_gated(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dO,
                                const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                                int T, int d, int b, int K, float scale, sas_phi_t phi,
                                sas_gating_t gating, void* dq, void* dk, void* dv,
                                float* dscores, void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * The training pair with the forward's output residual: the same results as
 * sas_attn_fwd / sas_attn_bwd, with the backward's row sums
 * D_i = sum_t P_it dP_it taken in one pass over dO, o and o_res instead of a
 * recomputation of every attended tile. This is a library variant; the
 * method's pages fix no kernel split of the backward.
 *   sas_attn_fwd_res: also writes o_res [B, Hq, T, d] (dtype), the part of
 *     the fp32 output that rounding o to the dtype drops: o + o_res is the
 *     output to fp32 rounding. For this the probabilities enter the P.V
 *     product as two bf16 terms (P = P_hi + P_lo), so that product is the
 *     fp32 one; o itself is the same up to that rounding.
 *   sas_attn_bwd_res: the backward with D_i = dO_i . (o_i + o_res_i), which
 *     equals sum_t P_it dP_it to fp32 rounding. Taking D from the stored bf16
 *     o alone would move dq by more than the bf16 tolerance on rows that
 *     attend a few large-logit keys; with the residual it does not.
 *   Both: bf16, d = 128, b = 64, G = Hq / Hkv of 2 or 4 (the tensor-core
 *   path), inner gating; any other shape returns SAS_ERR_UNSUPPORTED. o_res
 *   is 16-byte aligned and not NULL (SAS_ERR_INVALID_ARG). Other arguments,
 *   layouts, the workspace and the errors are those of sas_attn_fwd /
 *   sas_attn_bwd.
 */
sas_status_t sas_attn_fwd_res(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* gates, int B, int Hq, int Hkv, int T,
                              int d, int b, int K, float scale, void* o, void* o_res, float* lse,
                              sas_stream_t stream);
sas_status_t sas_attn_bwd_res(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                              const void* o, const void* o_res, const float* lse, const void* dO,
                              const int32_t* idx, const float* gates, int B, int Hq, int Hkv,
                              int T, int d, int b, int K, float scale, void* dq, void* dk, void* dv,
                              float* dscores, void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * sas_decode - one query token per sequence over a KV cache, selected blocks
 * plus the current block ([picx] Eq. 2 with use_gates = 0, Eq. 9 with
 * use_gates = 1; [review] Summary: gates are dropped at inference while the
 * hard selection stays).
 *   The query of sequence bi sits at position L-1 and its key is already in
 *   the cache. The current block cb = floor((L-1)/b) covers positions
 *   cb*b .. L-1 (all visible, bias 0); the C = cb blocks before it are the
 *   history that idx selects from.
 *   q [B, Hq, d] (dtype). kcache, vcache [B, Hkv, Lcap, d] (dtype), positions
 *     0..L-1 valid, L <= Lcap.
 *   idx [B, Hkv, K] int32 over 0..C-1, -1 skipped (as written by
 *     sas_gate_topk with causal = 0, rows = 1); an entry >= C or below -1 is
 *     skipped and reported as SAS_ERR_DEVICE.
 *   gates [B, Hkv, C] fp32; read only when use_gates != 0 (may be NULL otherwise).
 *   o [B, Hq, d] (dtype; written).
 *   ws / ws_bytes: at least sas_decode_workspace_size() bytes, 256-byte
 *   aligned; its contents on entry do not matter (the call clears the part
 *   that must start at zero). Calls that share a workspace must not overlap
 *   on the device.
 */
size_t sas_decode_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K);
sas_status_t sas_decode(sas_dtype_t dtype, const void* q, const void* kcache, const void* vcache,
                        const int32_t* idx, const float* gates, int use_gates, int B, int Hq,
                        int Hkv, int L, int Lcap, int d, int b, int K, float scale, void* o,
                        void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * sas_decode_select - one decode step from the selector scores: the gates
 * and Top-K of each (batch, KV head) row of history blocks, then sas_decode
 * with them ([picx] Methodology Eq. 4-6 and Eq. 9; the selection the
 * evolve.pub review's Summary keeps at inference). Equal to sas_gate_topk on
 * scores viewed as [B][Hkv][1][C] (causal = 0, softmax gates) followed by
 * sas_decode with its idx and gates.
 *   scores   [B][Hkv][C] fp32, C = (L - 1) / b (may be NULL when C == 0).
 *   gates    [B][Hkv][C] fp32 output, or NULL (not stored).
 *   idx      [B][Hkv][K] int32 output, or NULL (not stored).
 *   The other arguments are those of sas_decode. ws: at least
 *   sas_decode_select_workspace_size(B, Hq, Hkv, L, d, b, K) bytes, 256-byte
 *   aligned, owned by the caller, free once the call's work on `stream` is
 *   done.
 * With the tensor-core decode (bf16, d = 128, b = 64, G <= 8) and each row
 * short enough for its splits (C <= 512 x splits, splits <= 16), the
 * selection runs in the decode's own launch: the splits of a (batch, KV head)
 * form one thread-block cluster that selects the row, and each split then
 * streams its share of the selected blocks. Otherwise it is two launches.
 * Errors: those of sas_gate_topk and sas_decode; a bad argument is reported
 * before any launch.
 */
size_t sas_decode_select_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K);
sas_status_t sas_decode_select(sas_dtype_t dtype, const void* q, const void* kcache,
                               const void* vcache, const float* scores, int use_gates, int B,
                               int Hq, int Hkv, int L, int Lcap, int d, int b, int K, float scale,
                               void* o, float* gates, int32_t* idx, void* ws, size_t ws_bytes,
                               sas_stream_t stream);

/*
 * sas_decode_select_pooled - sas_decode_select whose scores are the
 * weight-free pooled selector's (sas_selector_scores_decode below), formed
 * from the key summaries instead of being passed in:
 *   scores[b, kvh, m] = sel_scale * qbar . kbar[b, kvh, m],
 *   qbar = the mean of q over the group's G heads; sel_scale <= 0 selects
 *   1/sqrt(d).
 * Equal to sas_selector_scores_decode followed by sas_decode_select.
 *   kbar [B][Hkv][C][d] fp32 (sas_block_summaries' output; may be NULL when
 *   C == 0). The other arguments are those of sas_decode_select; ws: at
 *   least sas_decode_select_pooled_workspace_size(B, Hq, Hkv, L, d, b, K)
 *   bytes, 256-byte aligned, owned by the caller.
 * Where sas_decode_select runs in one launch and kbar is 16-byte aligned,
 * the scores are formed in that launch too: each split of the cluster scores
 * its own entries of the row before the selection. Otherwise the selector
 * kernel writes them into the workspace first.
 * Errors: those of sas_decode_select and sas_selector_scores_decode
 * (B x Hkv > 65535 is SAS_ERR_UNSUPPORTED).
 */
size_t sas_decode_select_pooled_workspace_size(int B, int Hq, int Hkv, int L, int d, int b, int K);
sas_status_t sas_decode_select_pooled(sas_dtype_t dtype, const void* q, const void* kcache,
                                      const void* vcache, const float* kbar, float sel_scale,
                                      int use_gates, int B, int Hq, int Hkv, int L, int Lcap, int d,
                                      int b, int K, float scale, void* o, float* gates,
                                      int32_t* idx, void* ws, size_t ws_bytes,
                                      sas_stream_t stream);

/*
 * sas_decode_noalloc - sas_decode for callers that cannot allocate device
 * memory. Some callers cannot call cudaMalloc or take a workspace from their
 * framework at the point where they decode: an inference server or plugin
 * whose host framework owns every device allocation and forbids new ones once
 * serving starts, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device synchronisation. This entry point takes the same inputs and
 * outputs as sas_decode but no workspace: its scratch (the split partials and
 * merge tickets) lives in a fixed 2 MiB array in device memory, which every
 * GPU that loads the library holds until the process exits. The paper has no
 * counterpart; it is a deployment convenience of this library.
 *   - The call itself allocates nothing: no cudaMalloc, cudaFree or
 *     allocating library routine. Its first call on a device looks up the
 *     array's device address (once per device, with that device current).
 *     That first call (like the first call of any entry point on a device)
 *     is also when the CUDA runtime loads the library's device code onto the
 *     device: the loader reserves the array and the code in device memory,
 *     an allocation the runtime makes, and may synchronise the device. Make
 *     one warm-up call per device at initialisation, before serving starts
 *     and before any stream capture, so that later calls do none of this.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents; the call clears the part that must start at zero.
 *     Calls that overlap on the GPU (other streams, other host threads) race
 *     on it: issue them one after another.
 *   - A problem whose scratch would exceed the array
 *     (sas_decode_noalloc_max_scratch() bytes; compare with
 *     sas_decode_workspace_size()) returns SAS_ERR_WORKSPACE before any launch.
 *   Arguments, layouts and results are those of sas_decode.
 */
sas_status_t sas_decode_noalloc(sas_dtype_t dtype, const void* q, const void* kcache,
                                const void* vcache, const int32_t* idx, const float* gates,
                                int use_gates, int B, int Hq, int Hkv, int L, int Lcap, int d,
                                int b, int K, float scale, void* o, sas_stream_t stream);
size_t sas_decode_noalloc_max_scratch(void);

/*
 * sas_decode_paged - sas_decode over a paged KV cache, the layout the pages'
 * deployment decodes from ([picx] Efficiency Benefits: an SGLang backend
 * with FlashInfer kernels, GQA with per-group selection). The pages fix no
 * layout; this call reads it as:
 *   kpages, vpages [num_pages, Hkv, P, d] (dtype), P = page_size tokens per
 *     page. Sequence bi owns the pages page_indices[page_indptr[bi] ..
 *     page_indptr[bi + 1]) in logical order; its token t sits at row t % P
 *     of its (t / P)-th page. Pages may be shared or in any order.
 *   seq_lens [B] int32: tokens of each sequence (1 <= L_bi <= max_len); the
 *     last page may be partly used (rows past L_bi are never read into o).
 *   The query of sequence bi sits at L_bi - 1; its current block is
 *   cb = floor((L_bi - 1)/b) and idx[bi] selects among its cb history blocks.
 *   gates [B, Hkv, Cmax] fp32 with Cmax = floor((max_len - 1)/b) (row bi
 *     valid for its first cb entries); read only when use_gates != 0.
 *   page_indptr [B + 1], page_indices, seq_lens, idx: device int32.
 *   The result equals sas_decode on each sequence's gathered contiguous cache.
 *   Limits: bf16, d = 128, b = 64, G <= 8, P a power of two >= 16
 *   (SAS_ERR_UNSUPPORTED otherwise). A length, page entry or idx entry out
 *   of range is skipped and reported as SAS_ERR_DEVICE.
 *   ws / ws_bytes: at least sas_decode_paged_workspace_size() bytes, as for
 *   sas_decode.
 */
size_t sas_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_len, int d, int b, int K);
sas_status_t sas_decode_paged(sas_dtype_t dtype, const void* q, const void* kpages,
                              const void* vpages, const int32_t* page_indptr,
                              const int32_t* page_indices, const int32_t* seq_lens,
                              const int32_t* idx, const float* gates, int use_gates, int B, int Hq,
                              int Hkv, int num_pages, int page_size, int max_len, int d, int b,
                              int K, float scale, void* o, void* ws, size_t ws_bytes,
                              sas_stream_t stream);

/*
 * Block-selector scores from pooled block summaries. [review] Frequently
 * asked questions: the selector (the AttnGate architecture) works from
 * pooling-based block summaries and scores history blocks per query block and
 * KV-head group; the pages give neither its layers nor its weights. These
 * calls compute the weight-free reading: a block's key summary is the mean of
 * its keys (a partial last block: of its valid rows), a query block's
 * summary the mean of its rows over the G heads of the group, and
 *   scores[b, kvh, j, m] = scale * qbar_j . kbar_m  for m < j, 0 for m >= j
 * (the mean of the attention logits over every row/head/key pair of the two
 * blocks), fp32, ready for sas_gate_topk. scale <= 0 selects 1/sqrt(d).
 *   sas_selector_scores: q [B, Hq, T, d], k [B, Hkv, T, d] (dtype) ->
 *     scores [B, Hkv, N, N]; workspace sas_selector_workspace_size() bytes
 *     (256-byte aligned; contents on entry do not matter).
 *   sas_block_summaries: the key summaries of the C = floor((L-1)/b) full
 *     history blocks of a cache [B, Hkv, Lcap, d] -> kbar [B, Hkv, C, d] fp32
 *     (a server keeps these and adds one whenever a block fills).
 *   sas_selector_scores_decode: q [B, Hq, d] (the token at L-1), kbar as
 *     above -> scores [B, Hkv, C]: qbar is the mean of the group's G heads.
 */
size_t sas_selector_workspace_size(int B, int Hkv, int T, int d, int b);
sas_status_t sas_selector_scores(sas_dtype_t dtype, const void* q, const void* k, int B, int Hq,
                                 int Hkv, int T, int d, int b, float scale, float* scores,
                                 void* ws, size_t ws_bytes, sas_stream_t stream);
sas_status_t sas_block_summaries(sas_dtype_t dtype, const void* kcache, int B, int Hkv, int L,
                                 int Lcap, int d, int b, float* kbar, sas_stream_t stream);
sas_status_t sas_selector_scores_decode(sas_dtype_t dtype, const void* q, const float* kbar, int B,
                                        int Hq, int Hkv, int C, int d, float scale, float* scores,
                                        sas_stream_t stream);

/*
 * Dense comparison kernels ([picx] Eq. 1 with a causal mask): every block is
 * attended, no gates. Same layouts and conventions as the sparse calls; the
 * block size b only sets the kernels' tiling (use 64 unless d or T call for
 * less) and does not change the result.
 */
sas_status_t sas_dense_fwd(sas_dtype_t dtype, const void* q, const void* k, const void* v, int B,
                           int Hq, int Hkv, int T, int d, int b, float scale, void* o, float* lse,
                           sas_stream_t stream);
size_t sas_dense_bwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int b);
sas_status_t sas_dense_bwd(sas_dtype_t dtype, const void* q, const void* k, const void* v,
                           const void* o, const float* lse, const void* dO, int B, int Hq, int Hkv,
                           int T, int d, int b, float scale, void* dq, void* dk, void* dv,
                           void* ws, size_t ws_bytes, sas_stream_t stream);
size_t sas_dense_decode_workspace_size(int B, int Hq, int Hkv, int L, int d);
sas_status_t sas_dense_decode(sas_dtype_t dtype, const void* q, const void* kcache,
                              const void* vcache, int B, int Hq, int Hkv, int L, int Lcap, int d,
                              float scale, void* o, void* ws, size_t ws_bytes,
                              sas_stream_t stream);

/*
 * Device-side error reporting. sas_get_device_error synchronises `stream`,
 * reads the current device's error word, clears it and returns SAS_OK,
 * SAS_ERR_TIMEOUT or SAS_ERR_DEVICE (SAS_ERR_CUDA if the read itself fails).
 * *raw (may be NULL) receives the raw bit mask.
 */
sas_status_t sas_get_device_error(sas_stream_t stream, uint32_t* raw);

/*
 * Iteration limit of every bounded device wait (mbarrier and flag spins);
 * 0 restores the default (about a second of spinning). Applies to calls
 * enqueued afterwards from any thread.
 */
void sas_set_wait_limit(uint64_t iterations);

/*
 * Failure-detection self test: launches one kernel that waits, with the
 * current wait limit, on a barrier that nothing ever completes; the wait
 * runs out, the kernel records SAS_ERR_TIMEOUT in the error word and
 * returns. Nothing hangs or faults. Use with a small limit.
 */
sas_status_t sas_selftest_wait_timeout(sas_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SAS_H_ */
