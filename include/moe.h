/*
 * moe.h - C ABI of the single-GPU MoE-layer forward for NVIDIA B200 (sm_100a).
 *
 * The layer (SonicMoE explainer, gitcode.csdn.net, sections 1 and 3):
 *     y_t = sum over the token's top-K experts e of  w_{t,e} * FFN_e(x_t),
 *     FFN_e(x) = (silu(x W_gate[e]) * (x W_up[e])) W_down[e],
 * computed as router GEMM -> softmax -> top-K -> per-expert count + exclusive
 * scan -> stable permutation into expert-major order -> grouped gate/up GEMM
 * with the token gather fused into the operand load and SwiGLU in the epilogue
 * -> grouped down GEMM -> weighted combine back to token order.
 *
 * Conventions shared by every entry point:
 *  - Ownership: the caller allocates and owns every buffer. Pointers named
 *    "device" must be device-accessible memory of the current CUDA device; the
 *    library never allocates, frees or synchronises, except moe_get_device_status
 *    and the profiling queries, which synchronise.
 *  - Layout: every tensor is dense row-major. Indices are int32.
 *  - Dtypes: MOE_F32 - x, weights, outputs and intermediates are fp32.
 *    MOE_BF16 - x, W_r, W_gate, W_up, W_down, x_perm, a_act, y_perm and out are
 *    bf16; logits, bias and top-k weights are fp32; all sums accumulate in fp32.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns at once.
 *  - Errors: argument errors (null required pointer, bad sizes, unsupported
 *    shape, short workspace) are returned synchronously and nothing is
 *    enqueued. A launch failure returns MOE_ERR_CUDA. Faults found on the
 *    device (an expert id out of range, a bounded wait that ran out) set a
 *    device status word that moe_get_device_status() reads and clears.
 *  - T = 0 is valid: nothing is read or written (moe_permute still zeroes counts
 *    and offsets) and data pointers may be NULL.
 *  - Thread safety: calls are reentrant; the only global state is the device
 *    status word, a per-device cache of SM counts and the opt-in profiler.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same handle as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, K > E, ...          */
  MOE_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. E > 256)      */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed            */
  MOE_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required   */
  MOE_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out               */
  MOE_ERR_DEVICE_INDEX = 6 /* device: an index read was out of range       */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Problem size. T tokens of width d, E experts, top-K per token, expert
 * intermediate width n. capacity_factor <= 0 means no limit; otherwise each
 * expert keeps at most C = ceil(capacity_factor * T * K / E) assignments,
 * the first C in token order ("Operators & compilers: MoE routing and sparse
 * kernels", section 4: capacity factor bounds the tokens per expert, the
 * overflow is dropped). renormalize != 0: top-K weights are the softmax
 * restricted to the K selected experts (they sum to 1); 0: plain softmax
 * over all E experts, read at the selected ones. Limits: 1 <= K <= E <= 256,
 * K <= 32, T >= 0, T * K < 2^31, d % 64 == 0 (router tiles, TMA boxes);
 * n % 64 == 0 for MOE_BF16 and n % 16 == 0 for MOE_F32.
 * tile_round = R > 0: tile-aware token rounding (SonicMoE explainer, section 6.5, names
 * it without a rule; this is the library's reading), in the direction tile_round_mode gives
 * (0 = down, 1 = up, 2 = nearest). For expert e with c routed assignments, r = c mod R != 0:
 *   down: with c >= R, e keeps R * floor(c / R) of them, the ones with the largest router
 *     logit for e (equal logits: the earlier token stays), and drops the rest like capacity
 *     overflow (assign_to_perm = -1, no re-normalisation); with c < R it keeps all;
 *   up: e gains the min(R - r, T - c) tokens that did not route to it with the largest
 *     router logit for it (equal logits: the earlier token), each such token gaining one
 *     more slot; a token's weights are then computed over its enlarged selection
 *     (renormalised: they still sum to 1; plain softmax: unchanged for its routed experts);
 *   nearest: down when r <= R - r, else up.
 * Added assignments follow the routed ones in the flat numbering, a = T*K + j for the j-th
 * added (listed by expert, then ascending token), so that assign_to_perm / perm_to_assign
 * span T*K + E*(R-1) entries with rounding up or to the nearest tile. Needs the router
 * logits, so rounding applies in moe_forward (every direction) and moe_dispatch (down only;
 * the other directions return MOE_ERR_UNSUPPORTED there, as moe_permute does for any
 * rounding, and moe_forward_h); exclusive with capacity_factor > 0. 0 = off. Up and nearest
 * need T <= 131072 (one bit a token in shared memory) and T*K + E*(R-1) < 2^31, else
 * MOE_ERR_UNSUPPORTED. */
typedef struct {
  int32_t T, d, E, K, n;
  float capacity_factor;
  int32_t renormalize;
  int32_t dtype;      /* moe_dtype */
  int32_t tile_round; /* 0, or the row tile R that each expert's kept count is rounded to */
  int32_t tile_round_mode; /* 0 = round down, 1 = up, 2 = to the nearest tile (see above) */
  int32_t ffn_variant; /* tiles of the bf16 grouped GEMMs (a deployment choice; the pages have
                        * no counterpart): 0 = automatic, 1 = single-CTA 128 x 256 tiles,
                        * 2 = CTA pairs (256 x 256 tiles on two SMs, tcgen05 cta_group::2)
                        * with the gate/up rows gathered inside the GEMM, 3 = CTA pairs with
                        * the gate/up rows first copied expert-major into the y_perm buffer
                        * by one gather kernel. All compute the same result; other values
                        * return MOE_ERR_INVALID_ARG. A per-call field: calls on different
                        * streams or threads may choose differently. */
  int32_t route_topk;  /* top-K form of the warp-per-token routers (fp32 x, given logits, the
                        * one-launch route + permute of moe_dispatch), a per-call field:
                        * 0 = automatic (currently form 1, measured faster), 1 = K rounds of a
                        * warp arg-max, 2 = bitonic merges ("How AI chips support MoE",
                        * chapter 4, section 4.3: a bitonic network for few experts): lane l
                        * holds experts l and l + 32 as a sorted pair and five shuffle merges
                        * give every lane the token's top-K; applies for E <= 64 and K <= 8,
                        * otherwise form 1 runs. Both give the same ids and weights. The bf16
                        * tensor-core router keeps its per-thread insertion lists. Other values
                        * return MOE_ERR_INVALID_ARG. */
} moe_shape;

/* ----------------------------------------------------------------------------
 * Workspace sizes (bytes). The caller passes a device buffer at least this big
 * (256-byte aligned) to moe_permute / moe_forward. Returns 0 on a bad shape.
 * moe_permute_workspace_size: scratch of the histogram / scan / scatter
 *   kernels (per-chunk expert counts and rank bases), plus, when tile_round > 0,
 *   the rounded copy of the ids and the kept counts (used by moe_dispatch).
 * moe_forward_workspace_size: everything moe_forward keeps between kernels:
 *   logits, top-K ids and weights, counts, offsets, both permutation indices,
 *   the permute scratch, a_act[n_assign, n] and y_perm[n_assign, d] (n_assign = T*K, or
 *   T*K + E*(R-1) with rounding up or to the nearest tile) and the rounding buffers.
 */
size_t moe_permute_workspace_size(const moe_shape* shape);
size_t moe_forward_workspace_size(const moe_shape* shape);

/* ----------------------------------------------------------------------------
 * moe_route - router logits, softmax and top-K.
 * "Two upstream innovations of MoE: Routing-Free and OmniMoE"
 * (chatdocs.ruinique.com), section 1.1: x -> Router(x) -> Softmax -> TopK;
 * "How AI chips support MoE", chapter 4, sections 4.2-4.3: the gate is a
 * small dense linear map followed by softmax and a top-K selection.
 *
 *   x          [T, d]  device, dtype; ignored when logits_in != NULL
 *   w_r        [d, E]  device, dtype; ignored when logits_in != NULL
 *   bias       [E]     device fp32 or NULL; added to every token's x W_r
 *                      (not to logits_in)
 *   logits_in  [T, E]  device fp32 or NULL: use these logits instead of x W_r
 *   logits_out [T, E]  device fp32 or NULL: receives the logits the top-K saw
 *                      (x W_r + bias, or a copy of logits_in)
 *   topk_ids   [T, K]  device int32 out: slot 0 = largest logit; ties go to
 *                      the lower expert id (+0 and -0 are equal)
 *   topk_w     [T, K]  device fp32 out: weights (see renormalize)
 * Selection compares the fp32 logits; NaN logits give unspecified ids.
 */
moe_status moe_route(const moe_shape* shape, const void* x, const void* w_r, const float* bias,
                     const float* logits_in, float* logits_out, int32_t* topk_ids,
                     float* topk_w, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_permute - per-expert counts, exclusive scan and the stable permutation.
 * "Operators & compilers: MoE routing and sparse kernels"
 * (charles2530.github.io), section 3: regrouping tokens by expert is an
 * index/scatter/gather problem solved with counting and a prefix sum;
 * "Two upstream innovations of MoE: Routing-Free and OmniMoE", section 2.3:
 * the (token, expert) tasks sorted by (expert, token);
 * SonicMoE explainer, section 11: the expert-major metadata.
 * Atomic-free and deterministic: flat assignment a = t*K + k; inside an expert
 * the assignments keep ascending a (= token) order.
 *
 *   topk_ids        [T, K]   device int32 in, each in [0, E) (an id out of range
 *                            is skipped and flags MOE_ERR_DEVICE_INDEX)
 *   counts          [E]      device int32 out: raw assignments per expert
 *   offsets         [E + 1]  device int32 out: exclusive scan of min(counts, C);
 *                            offsets[E] = kept assignments
 *   assign_to_perm  [T * K]  device int32 out: a -> expert-major slot, -1 if dropped
 *   perm_to_assign  [T * K]  device int32 out: slot -> a for slots < offsets[E];
 *                            the tail is left unwritten
 *   x               [T, d]   device dtype or NULL  \ both non-NULL: also write the
 *   x_perm          [T*K, d] device dtype or NULL  / gathered rows x_perm[p] =
 *                            x[perm_to_assign[p] / K] for p < offsets[E]
 *   workspace, ws_bytes      >= moe_permute_workspace_size(shape)
 */
moe_status moe_permute(const moe_shape* shape, const int32_t* topk_ids, int32_t* counts,
                       int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                       const void* x, void* x_perm, void* workspace, size_t ws_bytes,
                       moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_permute_static - moe_permute for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant, not part of the method.
 * Some callers may not call cudaMalloc while they run: a serving engine that plans its
 * whole memory budget at start-up and forbids allocation on the request path, an embedded
 * runtime with a fixed arena, or code that runs where an allocation would synchronise the
 * device. This entry point takes the same arguments as moe_permute minus the workspace:
 * its scratch (per-chunk expert counts and rank bases) lives in a file-scope device array
 * of MOE_PERMUTE_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. It allocates nothing and calls no allocating
 * routine. Results are identical to moe_permute.
 *  - Limit: needs 2 * ceil(T*K / 1024) * E * 4 bytes of scratch (= moe_permute_workspace_size
 *    minus its 256-byte slack) when T*K > 32768; smaller problems run in one CTA or one
 *    cluster and use none of it. Problems beyond the limit return MOE_ERR_UNSUPPORTED and
 *    enqueue nothing. With the 1 MiB array: T*K up to about 0.5 million assignments at
 *    E = 256, 2 million at E = 64.
 *  - Set-up: the first call on each device (with that device current) resolves the array's
 *    device address with cudaGetSymbolAddress. That call, or any earlier call into the
 *    library on the device, may also be when the CUDA driver loads the library's module
 *    and places the array in device memory (lazy module loading), which can allocate and
 *    synchronise. So make the first call on each device at start-up, before any stream
 *    capture and before the allocation-free part of the program. The resolved address is
 *    kept for the life of the process; after cudaDeviceReset on a device it is stale and
 *    the library must not be used on that device again.
 *  - Sharing: every call uses the same array, which keeps the last call's contents (the
 *    kernels overwrite every entry they read, so nothing must start at zero). Calls whose
 *    kernels overlap on the GPU (other streams, other host threads) race on it: serialise
 *    them.
 */
#define MOE_PERMUTE_STATIC_SCRATCH_BYTES (1u << 20) /* fixed when the library is built */
moe_status moe_permute_static(const moe_shape* shape, const int32_t* topk_ids, int32_t* counts,
                              int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                              const void* x, void* x_perm, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_dispatch - moe_route followed by moe_permute, in one call.
 * The steps are those of the two calls ("How AI chips support MoE", chapter 4,
 * sections 4.2-4.3; "Operators & compilers: MoE routing and sparse kernels", section 3);
 * the pages describe no separate dispatch operation, this is a launch-count saving for
 * the decode regime. Arguments are the union of both calls' (x serves the router and
 * the optional gather); every output equals what moe_route then moe_permute write.
 * When logits_in is given, T <= 128, T*K <= 2048, E <= 256 and K <= 32, one kernel (one
 * CTA) routes and permutes without a round trip of the ids through global memory;
 * otherwise the two calls' kernels run in turn. A requested x_perm is then copied by
 * the gather kernel of moe_permute, over the whole GPU. bias is added only to x W_r, as
 * in moe_route.
 *   workspace, ws_bytes  >= moe_permute_workspace_size(shape)
 * Errors: those of moe_route and moe_permute.
 */
moe_status moe_dispatch(const moe_shape* shape, const void* x, const void* w_r, const float* bias,
                        const float* logits_in, float* logits_out, int32_t* topk_ids,
                        float* topk_w, int32_t* counts, int32_t* offsets,
                        int32_t* assign_to_perm, int32_t* perm_to_assign, void* x_perm,
                        void* workspace, size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_grouped_ffn - the grouped SwiGLU expert FFN on the expert-major rows.
 * SonicMoE explainer, section 3 items 3-5 (grouped GEMM with a different M
 * per expert, SwiGLU, second grouped GEMM), section 6.2 (the gather of x is
 * fused into the GEMM's operand load: no [T*K, d] gathered copy of x is made)
 * and section 6.3 (SwiGLU runs in the epilogue while the accumulator is on chip).
 * For expert e, rows p in [offsets[e], offsets[e+1]) hold token
 * t = perm_to_assign[p] / K:
 *     a_act[p]  = silu(x[t] W_gate[e]) * (x[t] W_up[e])     (n wide)
 *     y_perm[p] = a_act[p] W_down[e]                        (d wide)
 *
 *   x               [T, d]      device dtype
 *   offsets         [E + 1]     device int32 (from moe_permute)
 *   perm_to_assign  [T * K]     device int32 (from moe_permute)
 *   w_gate, w_up    [E, d, n]   device dtype
 *   w_down          [E, n, d]   device dtype
 *   a_act           [T * K, n]  device dtype out (rows >= offsets[E] unwritten)
 *   y_perm          [T * K, d]  device dtype out (rows >= offsets[E] unwritten)
 * MOE_BF16 runs on the tcgen05 tensor cores (fp32 accumulation in TMEM);
 * MOE_F32 runs an fp32 FMA path.
 */
moe_status moe_grouped_ffn(const moe_shape* shape, const void* x, const int32_t* offsets,
                           const int32_t* perm_to_assign, const void* w_gate, const void* w_up,
                           const void* w_down, void* a_act, void* y_perm, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_combine - weighted scatter-combine back to token order.
 * SonicMoE explainer, section 3 item 6 (scatter/combine to token-major) and
 * section 6.1 (the aggregation fuses the scatter and the weighted sum).
 *     out[t] = sum_{k=0..K-1, assign_to_perm[t*K+k] >= 0} topk_w[t,k] * y_perm[assign_to_perm[t*K+k]]
 * summed in fp32 in k order (deterministic); dropped slots add nothing and the
 * remaining weights are not rescaled; a token with every slot dropped gets 0.
 *
 *   y_perm          [T * K, d]  device dtype
 *   assign_to_perm  [T * K]     device int32 (values >= T*K flag MOE_ERR_DEVICE_INDEX)
 *   topk_w          [T, K]      device fp32
 *   out             [T, d]      device dtype out
 */
moe_status moe_combine(const moe_shape* shape, const void* y_perm, const int32_t* assign_to_perm,
                       const float* topk_w, void* out, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_forward - the whole layer: moe_route, moe_permute (no x_perm),
 * moe_grouped_ffn and moe_combine chained on `stream` with no host sync.
 *
 *   x [T, d], w_r [d, E], bias [E] or NULL, logits_in [T, E] or NULL,
 *   w_gate/w_up [E, d, n], w_down [E, n, d]: as above
 *   out        [T, d]  device dtype out
 *   workspace, ws_bytes >= moe_forward_workspace_size(shape)
 *   layout of the workspace (byte offsets from moe_forward_workspace_layout)
 *   lets a caller read the intermediates after the call.
 */
moe_status moe_forward(const moe_shape* shape, const void* x, const void* w_r, const float* bias,
                       const float* logits_in, const void* w_gate, const void* w_up,
                       const void* w_down, void* out, void* workspace, size_t ws_bytes,
                       moe_stream_t stream);

/* Byte offsets of the intermediates inside moe_forward's workspace. */
typedef struct {
  size_t logits, topk_ids, topk_w, counts, offsets, assign_to_perm, perm_to_assign,
      permute_scratch, a_act, y_perm, round_ids, round_counts;
  /* rounding up or to the nearest tile (else equal to total, zero-sized): the added
   * assignments' tokens add_tok [E*(R-1)] int32 (-1 past the last one), their weights
   * add_w [E*(R-1)] fp32, each token's added assignments add_ptr [T+1] / add_idx
   * [E*(R-1)] (indices j into add_tok, ascending per token), a per-token cursor
   * add_cursor [T], and the token of every expert-major slot slot_token [T*K + E*(R-1)]. */
  size_t add_tok, add_w, add_ptr, add_idx, add_cursor, slot_token;
  size_t n_assign; /* entries of assign_to_perm / perm_to_assign: T*K, or T*K + E*(R-1) */
  size_t total;
} moe_workspace_layout;
moe_status moe_forward_workspace_layout(const moe_shape* shape, moe_workspace_layout* layout);

/* ----------------------------------------------------------------------------
 * moe_forward_h - moe_forward that also keeps, for the backward, the gate/up
 * pre-activations of every kept slot: h [T*K, 2n] bf16, row p = (g | u) with
 * g = x[tok(p)] W_gate[e], u = x[tok(p)] W_up[e] (rows past offsets[E] unwritten).
 * The routing outputs stay in the workspace (moe_forward_workspace_layout).
 * bf16 only (MOE_ERR_UNSUPPORTED otherwise); h 16-byte aligned.
 *
 * moe_backward - the backward of the expert half of the layer without caching
 * Y or dY (SonicMoE explainer, section 6.4; the gather of dO by routing index
 * fused into the GEMM's operand load, section 6.2; the SwiGLU backward in the
 * epilogue, section 6.3), routing held fixed. For the kept slot p of expert e
 * holding token t's slot k (a = perm_to_assign[p] = t*K + k):
 *   dA'[p] = d_out[t] W_down[e]^T          (tensor cores, fp32 accumulate)
 *   d_w[t, k] = <dA'[p], silu(g) * u>      (the routing-weight gradient; 0 if dropped)
 *   dA = topk_w[t, k] dA',  s = 1 / (1 + e^-g)
 *   d_h[p] = (dA u s (1 + g (1 - s)) | dA silu(g))   (dG | dU, bf16)
 * and, when d_x is not NULL, the input gradient through the experts:
 *   dX_perm[p] = dG[p] W_gate[e]^T + dU[p] W_up[e]^T  (tensor cores, K = 2n)
 *   d_x[t] = sum over t's kept slots of dX_perm      (fp32 sum in slot order, bf16)
 *   d_out  [T, d] bf16; topk_w [T, K] fp32; offsets, perm_to_assign,
 *   assign_to_perm as moe_permute wrote them; w_gate, w_up [E, d, n] and
 *   w_down [E, n, d] bf16 (w_gate, w_up may be NULL when d_x is NULL);
 *   h [T*K, 2n] from moe_forward_h; d_h [T*K, 2n] bf16 out; d_w [T, K] fp32 out;
 *   d_x [T, d] bf16 out or NULL;
 *   workspace >= moe_backward_workspace_size(shape), 256-byte aligned (per-slot partial
 *   sums, and one [T*K, d] row buffer: the dO rows copied expert-major for the dA' GEMM
 *   when shape.ffn_variant is 3, or 0 with n >= 4096 (1 and 2 gather them inside the
 *   GEMM), then the dX_perm rows).
 * d_w sums each slot's 256-column parts in a fixed order (deterministic). The router's
 * own backward (through the softmax and top-K to the logits, W_r and x) and the weight
 * gradients are not computed. bf16 only; d_out, w_*, h, d_h, d_x 16-byte aligned.
 */
moe_status moe_forward_h(const moe_shape* shape, const void* x, const void* w_r,
                         const float* bias, const float* logits_in, const void* w_gate,
                         const void* w_up, const void* w_down, void* out, void* h,
                         void* workspace, size_t ws_bytes, moe_stream_t stream);
size_t moe_backward_workspace_size(const moe_shape* shape);
moe_status moe_backward(const moe_shape* shape, const void* d_out, const float* topk_w,
                        const int32_t* offsets, const int32_t* perm_to_assign,
                        const int32_t* assign_to_perm, const void* w_gate, const void* w_up,
                        const void* w_down, const void* h, void* d_h, float* d_w, void* d_x,
                        void* workspace, size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * moe_backward_router - the router's backward with the top-K selection held fixed
 * ("Routing-Free and OmniMoE", section 1.1, Router -> Softmax -> TopK, and "How AI
 * chips support MoE", chapter 4, section 4.2, the gate x W_r + bias, read backwards).
 * With s_t = sum_k topk_w[t, k] d_w[t, k]:
 *   renormalize != 0: d_logits[t, e] = topk_w[t, k] (d_w[t, k] - s_t) at e = topk_ids[t, k],
 *                     0 at the experts not selected;
 *   renormalize == 0: d_logits[t, e] = p[t, e] (g - s_t), p = softmax(logits[t]) over all E,
 *                     g = d_w[t, k] at e = topk_ids[t, k], 0 elsewhere;
 *   d_w_r = x^T d_logits, d_bias = sum over tokens of d_logits, and (d_x not NULL)
 *   d_x += d_logits W_r^T (the router's term of the input gradient, added in fp32 to the
 *   bf16 d_x, e.g. the experts' term from moe_backward).
 *   x [T, d], w_r [d, E] bf16; logits [T, E] fp32 (read only when renormalize == 0);
 *   topk_ids, topk_w [T, K] from the forward; d_w [T, K] from moe_backward;
 *   d_logits [T, E] fp32 out (also the intermediate); d_w_r [d, E] fp32 out;
 *   d_bias [E] fp32 out or NULL; d_x [T, d] bf16 in/out or NULL (16-byte aligned); with
 *   E > 16, x 16-byte aligned too.
 * Sums over tokens run in a fixed order (deterministic). bf16 only. With 17..256 experts,
 * E % 8 == 0 and w_r, d_logits 16-byte aligned, both contractions run on the tensor cores
 * with each d_logits value split into two bf16 terms (hi = bf16(v), lo = bf16(v - hi):
 * |v - hi - lo| <= 2^-16 |v|), so the sums keep fp32 accuracy.
 */
moe_status moe_backward_router(const moe_shape* shape, const void* x, const void* w_r,
                               const float* logits, const int32_t* topk_ids, const float* topk_w,
                               const float* d_w, float* d_logits, float* d_w_r, float* d_bias,
                               void* d_x, moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * Atomic (rank-1) experts behind a Cartesian-product router, run expert-centric
 * ("Two upstream innovations of MoE: Routing-Free and OmniMoE", chatdocs.ruinique.com,
 * sections 2.1-2.3 and 3.2).
 * N = n_rows * n_cols experts; expert i = (i_r, i_c), i = i_r * n_cols + i_c, is a pair of
 * d-vectors w_in[i], w_out[i] (two [N, d] bf16 tables, section 2.1). Per token t:
 *   p_r = x_t W_row, p_c = x_t W_col   (W_row [d, n_rows], W_col [d, n_cols] bf16; the
 *       logits are one [T, n_rows + n_cols] fp32 array, row axis first; section 2.2);
 *   selection: the K experts with the largest fl32(p_r[i_r] + p_c[i_c]), descending, ties
 *       to the lower id. The pair's score LogSoftmax(p_r)_{i_r} + LogSoftmax(p_c)_{i_c}
 *       differs from that sum by a per-token constant, so the ranking is the same;
 *   weights: renormalize != 0: softmax of the scores over the K selected; renormalize == 0:
 *       softmax(p_r)_{i_r} * softmax(p_c)_{i_c}, the factorised probability over all N;
 *   y_t = sum_k w_{t,k} silu(x_t . w_in[i_k]) w_out[i_k]   (bf16 out, fp32 sums).
 * Reading: the page instantiates the expert's nonlinearity as "SwiGLU"; an atomic expert has
 * one input vector, so it is read as SiLU, the gating nonlinearity of SwiGLU.
 * Limits: T >= 0, T * K < 2^31; 1 <= n_rows, n_cols <= 1024, N <= 2^20; 1 <= K <=
 * min(N, 4096); d % 256 == 0 with d / 256 in 1..8 or 16. The router GEMM (logits_in NULL)
 * also needs n_rows % 8 == 0, n_cols % 8 == 0. Tables, x, out and logits_out 16-byte aligned.
 */
typedef struct {
  int32_t T, d, n_rows, n_cols, K;
  int32_t renormalize; /* != 0: weights renormalised over the K selected */
  int32_t output_mode; /* output side of moe_omni_forward (moe_omni_experts always gathers,
                        * having no workspace for the fp32 sums): 0 = token-centric
                        * gather, y_t = sum_k h w_out[i_k] summed per token in slot order
                        * (deterministic); 1 = the page's expert-centric scatter-add (section
                        * 2.3): each expert's w_out row is read once and h * w_out[e] is added
                        * into its tokens' fp32 rows with atomic vector reductions, then
                        * rounded to bf16 (the fp32 sum order, and so the last bits, vary from
                        * run to run). Other values return MOE_ERR_INVALID_ARG. */
} moe_omni_shape;

/* Byte offsets inside the workspace of moe_omni_forward (each 256-byte aligned). */
typedef struct {
  size_t logits;         /* fp32 [T, n_rows + n_cols] */
  size_t topk_ids;       /* int32 [T, K] */
  size_t topk_w;         /* fp32 [T, K] */
  size_t counts;         /* int32 [N] tasks per expert */
  size_t offsets;        /* int32 [N + 1] */
  size_t assign_to_perm; /* int32 [T * K] (not written by moe_omni_forward) */
  size_t perm_to_assign; /* int32 [T * K], grouped by expert */
  size_t h;              /* fp32 [T * K] per-task scalar w_{t,k} silu(x_t . w_in[i_k]) */
  size_t scratch;        /* the schedule's scratch */
  size_t y32;            /* fp32 [T, d] output accumulator (scatter-add output mode) */
  size_t total;
} moe_omni_layout;

/* Workspace bytes of moe_omni_forward and moe_omni_schedule (0 for an invalid shape). */
size_t moe_omni_workspace_size(const moe_omni_shape* shape);
moe_status moe_omni_workspace_layout(const moe_omni_shape* shape, moe_omni_layout* layout);

/* moe_omni_route - router GEMM (tcgen05), then the K best experts of each token over the
 * whole grid and their weights (section 2.2).
 *   logits_in [T, n_rows + n_cols] fp32 or NULL; when NULL, x [T, d], w_row and w_col are
 *   read and the logits written to logits_out (required then); otherwise x, w_row, w_col
 *   and logits_out are ignored. topk_ids [T, K] int32, topk_w [T, K] fp32 out, slot 0 best.
 * The selection equals a brute-force sort of all N pair sums (ties to the lower id). */
moe_status moe_omni_route(const moe_omni_shape* shape, const void* x, const void* w_row,
                          const void* w_col, const float* logits_in, float* logits_out,
                          int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* moe_omni_schedule - the task list in (expert, token) order (section 2.3): counts [N]
 * (tasks per expert), offsets [N + 1] (exclusive scan), perm_to_assign [T * K] (slot ->
 * flat assignment t * K + k, ascending token inside an expert), assign_to_perm [T * K] (the
 * inverse). Deterministic. workspace: moe_omni_workspace_size bytes (its scratch part is
 * used). An expert id outside [0, N) is skipped and reported as MOE_ERR_DEVICE_INDEX. */
moe_status moe_omni_schedule(const moe_omni_shape* shape, const int32_t* topk_ids, int32_t* counts,
                             int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                             void* workspace, size_t ws_bytes, moe_stream_t stream);

/* moe_omni_experts - the experts, given the routing and the schedule:
 *   h[t * K + k] = topk_w[t, k] * silu(x_t . w_in[i_{t,k}])   computed expert-centric: each
 *       expert's w_in row is read once and meets all of its tokens' rows (section 2.3);
 *   out[t] = sum_k h[t * K + k] * w_out[i_{t,k}]   gathered per token, k in order.
 * x [T, d], w_in/w_out [N, d] bf16; h [T * K] fp32 out; out [T, d] bf16 out. */
moe_status moe_omni_experts(const moe_omni_shape* shape, const void* x, const void* w_in,
                            const void* w_out, const int32_t* topk_ids, const float* topk_w,
                            const int32_t* offsets, const int32_t* perm_to_assign, float* h,
                            void* out, moe_stream_t stream);

/* moe_omni_forward - route + schedule + experts with every intermediate in `workspace`
 * (layout from moe_omni_workspace_layout). logits_in as in moe_omni_route. The experts need
 * the tasks grouped by expert only, so inside the workspace perm_to_assign is grouped by
 * expert with the order inside an expert unspecified, and assign_to_perm is not written
 * (moe_omni_schedule gives the stable order); the output does not depend on that order. */
moe_status moe_omni_forward(const moe_omni_shape* shape, const void* x, const void* w_row,
                            const void* w_col, const float* logits_in, const void* w_in,
                            const void* w_out, void* out, void* workspace, size_t ws_bytes,
                            moe_stream_t stream);

/* ----------------------------------------------------------------------------
 * Device status: synchronises `stream`, returns the first device-side fault
 * recorded since the last call (MOE_OK if none) and clears it.
 */
moe_status moe_get_device_status(moe_stream_t stream);
const char* moe_status_string(moe_status status);

/* ----------------------------------------------------------------------------
 * Opt-in per-kernel timing (host state, not thread safe). While enabled,
 * every kernel launch the library makes is bracketed by CUDA events on its
 * stream. moe_profile_query synchronises on the recorded events and returns,
 * for kernel `id` in [0, moe_kernel_count()), its launch count and total
 * device milliseconds since the last reset; moe_kernel_name names it.
 * moe_launch_count counts every kernel launch made by the library (always on).
 */
moe_status moe_profile_enable(int on);
moe_status moe_profile_reset(void);
int moe_kernel_count(void);
const char* moe_kernel_name(int id);
moe_status moe_profile_query(int id, int64_t* launches, double* total_ms);
int64_t moe_launch_count(void);

/* Test hook for the failure-detection path: launches one block that waits on
 * an mbarrier nothing will complete, bounded by `limit_ns` nanoseconds, then
 * records MOE_ERR_TIMEOUT in the device status word and returns (no trap, no
 * hang). Read the result with moe_get_device_status. */
moe_status moe_selftest_timeout(uint64_t limit_ns, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
