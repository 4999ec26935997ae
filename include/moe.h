/*
 * moe.h -- C ABI of the B200 (sm_100a) token-routed Mixture-of-Experts FFN layer.
 *
 * One layer, forward and backward, on one GPU: router logits with fused
 * softmax/top-k, on-device expert counts and offsets, a rowwise permute into
 * contiguous per-expert buffers, a device-scheduled grouped SwiGLU GEMM,
 * a gate-weighted combine, and the backward of each step; plus MXFP8 block
 * quantisation.  Besides the steps themselves: a dispatch that writes the MXFP8
 * operands directly (moe_permute_mx), a backward that recomputes the expert
 * activations (moe_grouped_ffn_bwd_recompute), weight-gradient accumulation
 * (MOE_DW_ACCUMULATE), routing-balance statistics (moe_routing_stats), an
 * optional renormalised gate rule (moe_renorm_gates, moe_renorm_gates_bwd),
 * and the padded-capacity comparison layout (moe_padded_dispatch).
 *
 * Sources (news pages about the Olmo-core 3 release; they describe the method
 * in prose only):
 *   [kongchang]  "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀", sections
 *                容量税 (capacity tax), 路由不只是模型问题，更是系统问题 (routing
 *                is a systems problem), 吞吐量数字的边界条件 (boundary conditions).
 *   [bytechap]   "Olmo-core 3 mở rộng quy mô đào tạo mixture-of-experts lên hàng
 *                nghìn tỷ tham số", section "Cách thức hoạt động" (how it works).
 *   [aikraft]    "Прорыв в масштабируемости и производительности", section
 *                "Технические оптимизации: от MXFP8 до маршрутизации".
 *
 * Conventions for every entry point
 *   - Notation: T tokens, d = d_model, E experts, k = top_k, f = d_ff,
 *     R = T*k permuted rows.  All matrices are row-major and dense.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     the argument is documented as host memory.  The library keeps no
 *     pointer after a call returns and allocates no device memory: scratch
 *     comes from the caller's workspace (see moe_workspace_size).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = the legacy default stream), makes no host synchronisation and
 *     no device-to-host copy: routing metadata never returns to the host
 *     ([kongchang] routing section: metadata stays on the GPU; [bytechap] how
 *     it works: the CPU queues work without waiting).  Calls can be captured
 *     in a CUDA graph.
 *   - Device pointers must be 16-byte aligned; the workspace of the MXFP8
 *     grouped FFN calls and act_saved of the bf16 and MXFP8 backward 32-byte
 *     aligned (cudaMalloc and PyTorch allocations are 256-byte aligned).  Row
 *     counts and offsets are int32.
 *   - Errors: a call validates its arguments on the host before it launches
 *     anything and returns MOE_ERR_INVALID_ARG (bad sizes, null or misaligned
 *     pointers, too small workspace) or MOE_ERR_UNSUPPORTED (valid but not
 *     implemented, e.g. a shape the tensor-core tiles do not cover); nothing
 *     is launched in that case.  MOE_ERR_CUDA reports a failed launch.
 *     A kernel that gives up a bounded wait records MOE_ERR_TIMEOUT in the
 *     workspace status word; read it with moe_get_device_status.  No C++
 *     exception crosses this interface.
 *   - dtype: MOE_F32 (fp32 everywhere, CUDA-core GEMMs), MOE_BF16 (bf16
 *     activations and weights, fp32 accumulation, tcgen05 tensor cores),
 *     MOE_MXFP8 (grouped FFN calls only: bf16 activations, MXFP8 GEMM operands
 *     with block-scaled tcgen05 MMAs, fp32 accumulation and weight gradients;
 *     the route, permute and combine calls of such a layer take MOE_BF16, and
 *     its workspace is sized with MOE_MXFP8).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_CUDA = 3,
  MOE_ERR_TIMEOUT = 4
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1, MOE_MXFP8 = 2 } moe_dtype;

/* Flag OR-ed into the dw_dtype of moe_grouped_ffn_bwd / _recompute and into the dtype of
 * moe_route_bwd: the weight gradients (dW1, dW2; dW_router) are ADDED to what the output
 * buffers hold instead of overwriting them, for gradient accumulation over micro-batches
 * before the one all-reduce of an optimizer step (kongchang, capacity-tax section: one
 * gradient synchronisation per optimizer step).  fp32 outputs: each element gets exactly
 * one fp32 addition, old + new, where new is the value the overwriting call would write
 * (bit-identical to adding the two results afterwards); bf16 dW: old + new in fp32,
 * rounded once to bf16. */
#define MOE_DW_ACCUMULATE 0x100

/* The problem as the pages state it: T tokens of width d_model, E experts,
 * each token routed to top_k of them, expert hidden width d_ff.
 * Limits: 1 <= top_k <= min(E, 32), E <= 1024, d_model % 8 == 0,
 * d_ff % 8 == 0, T >= 0, T * top_k < 2^31. */
typedef struct moe_shape {
  int32_t T;
  int32_t d_model;
  int32_t E;
  int32_t top_k;
  int32_t d_ff;
} moe_shape;

/* Library version string (static storage). */
const char* moe_version(void);

/* Bytes of device workspace that the calls taking `ws` need for this shape.
 * `rows` is the largest row count passed to moe_grouped_ffn_bwd (T*top_k
 * for the dropless layout, E*capacity for the padded one); 0 means T*top_k.
 * The first 256 bytes hold the status word; it must be zeroed once by the
 * caller (cudaMemset) before the first call. */
size_t moe_workspace_size(moe_shape shape, int dtype, int64_t rows);

/* Read and clear the workspace status word (MOE_OK or MOE_ERR_TIMEOUT).
 * Diagnostic only: this call SYNCHRONISES `stream` and copies 4 bytes to
 * the host, unlike every other call. */
moe_status moe_get_device_status(void* ws, void* stream, int32_t* status_out);

/* ---- per-launch device timing (diagnostic) --------------------------------
 * Between moe_profile_begin and moe_profile_end, on the calling host thread, every
 * kernel launch made by this library's entry points is bracketed by two CUDA
 * events recorded on the launch's stream: launch i records events[2i] right before
 * and events[2i+1] right after it, and names[i] receives a static string naming the
 * kernel (the expert-FFN GEMMs start with "gemm_", the router's with "router_").
 * events: host array of 2*capacity cudaEvent_t created by the caller (timing
 * enabled, on the device of the launches); names: host array of capacity entries.
 * Launches beyond capacity run unrecorded; moe_profile_end writes the number of
 * launches made (recorded or not).  Not for use while a stream is being captured
 * (the event records would be captured too).  begin while a profile is open, or
 * null arguments: MOE_ERR_INVALID_ARG; end without begin: MOE_ERR_INVALID_ARG. */
moe_status moe_profile_begin(void* const* events, const char** names, int capacity);
moe_status moe_profile_end(int32_t* count);

/* ---- a1 + a2: route ------------------------------------------------------
 * [kongchang] capacity tax: each token is routed to a few of the experts;
 * routing section: routing metadata (split sizes and expert GEMM group sizes)
 * stays on the GPU.
 *   logits[t,e]  = sum_c x[t,c] * w_router[e,c] + bias[e]      (fp32 [T,E])
 *   p            = softmax over e of logits[t,:]
 *   topk_idx[t,j]: experts ordered by (-logits, e), first k     (int32 [T,k])
 *                  -- the lowest index wins ties
 *   topk_gate[t,j] = p[t, topk_idx[t,j]], not renormalised      (fp32 [T,k])
 *   counts[e]     = #{(t,j): topk_idx[t,j] == e}               (int32 [E])
 *   offsets       = exclusive prefix sum of counts             (int32 [E+1])
 *   slot_row[t,j] = offsets[e] + #{t' < t : e in topk_idx[t']}  (int32 [T,k])
 * x: [T,d] (fp32 for MOE_F32, bf16 for MOE_BF16); w_router: [E,d] same type;
 * bias: fp32 [E] or NULL.  ws/ws_bytes: workspace (moe_workspace_size).
 * The discrete steps are exact given the fp32 logits: indices, counts,
 * offsets and rows are deterministic. */
moe_status moe_route(moe_shape shape, int dtype, const void* x, const void* w_router,
                     const float* bias, float* logits, int32_t* topk_idx, float* topk_gate,
                     int32_t* counts, int32_t* offsets, int32_t* slot_row, void* ws,
                     size_t ws_bytes, void* stream);

/* ---- moe_route without a caller workspace --------------------------------
 * The pages have no counterpart for this call.  It exists for callers that
 * cannot allocate device memory: for example a plugin hosted by a framework
 * that owns all device memory and offers no allocation hook, code on a
 * latency-critical path where cudaMalloc/cudaFree could synchronise the
 * device and stall queued work, or a deployment whose device-memory footprint
 * is fixed at start-up.  It computes exactly what moe_route computes, from the
 * same arguments minus the workspace.
 *   Scratch: the per-block expert counts, their scan and the in-block ranks
 *   live in one fixed array inside this library, MOE_ROUTE_NOALLOC_MAX_SCRATCH
 *   bytes of device memory that every GPU loading the library holds until the
 *   process exits.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 *   allocating library routine).
 *   Limit: the array's first 256 bytes hold a status word (below); the shape
 *   needs 2*r(4*E*nb) + r(4*T*top_k) bytes of scratch besides, where r() rounds
 *   up to a multiple of 256, nb = ceil(T / tb) and tb = 32 for E <= 256, 16 for
 *   E <= 512, else 8; above MOE_ROUTE_NOALLOC_MAX_SCRATCH - 256 bytes the call
 *   returns MOE_ERR_UNSUPPORTED and runs nothing (use moe_route then).
 *   Device address: every call looks up the array's device address with the
 *   caller's device current (no allocation); the first call on a device also
 *   loads the array, so make that first call before any stream capture.
 *   Sharing: all calls on a device use the same array, which keeps whatever
 *   the last call left in it; nothing in the scratch part has to start at zero
 *   because each call writes every scratch byte before reading it.  Calls whose
 *   kernels can overlap on the GPU (different streams without ordering between
 *   them) race on the array and produce wrong results: order them on one stream.
 *   Errors on the device: the array's status word works like the workspace
 *   status word of moe_route.  It is zero when the library is loaded; a kernel
 *   that gives up a bounded wait sets it to MOE_ERR_TIMEOUT (its outputs are then
 *   incomplete) and it keeps that value until moe_route_noalloc_status reads and
 *   clears it. */
#define MOE_ROUTE_NOALLOC_MAX_SCRATCH (4u << 20)
moe_status moe_route_noalloc(moe_shape shape, int dtype, const void* x, const void* w_router,
                             const float* bias, float* logits, int32_t* topk_idx,
                             float* topk_gate, int32_t* counts, int32_t* offsets,
                             int32_t* slot_row, void* stream);

/* Read and clear the status word of moe_route_noalloc's array on the current
 * device: *status_out = MOE_OK or MOE_ERR_TIMEOUT (a bounded wait of a call since
 * the last read gave up).  Diagnostic only: like moe_get_device_status it
 * SYNCHRONISES `stream` and copies 4 bytes to the host; it allocates nothing.
 * Order it after the calls it reports on (same stream). */
moe_status moe_route_noalloc_status(void* stream, int32_t* status_out);

/* ---- a3: rowwise permute -------------------------------------------------
 * [bytechap] how it works: rowwise dispatch places routed rows directly in
 * the experts' input buffers.
 *   x_perm[slot_row[t,j], :] = x[t, :];  perm_src[slot_row[t,j]] = t
 * x: [T,d]; x_perm: [T*k, d] same type; perm_src: int32 [T*k]. */
moe_status moe_permute(moe_shape shape, int dtype, const void* x, const int32_t* slot_row,
                       void* x_perm, int32_t* perm_src, void* stream);

/* MXFP8 copies of the expert weights for dtype MOE_MXFP8, made from their FP32
 * masters by moe_mx_quantize_weights (once per optimizer step).  Every member is a
 * device pointer to a buffer of the size given; d % 128 == 0 and f % 128 == 0.
 * Element codes (E4M3, row-major, one byte per weight):
 *   w1_q, w1t_q [E*2f, d]    W1 quantised in blocks of 32 along d / along 2f
 *   w2_q, w2t_q [E*d, f]     W2 quantised in blocks of 32 along f / along d
 * Scales (E8M0, E*2f*d/32 bytes for W1, E*d*f/32 for W2) are stored as the
 * block-scaled MMA consumes them: 512-byte atoms covering 128 rows r (of the GEMM's
 * M or N) x 4 consecutive 32-blocks kb along its K, the scale of (r, kb) at byte
 *   (r % 32) * 16 + (r / 32) * 4 + kb.
 * Atom order, with j a 128-wide K stage:
 *   w1_s   atom (e * 2f/128 + r / 128) * d/128 + j, rows r = rows of W1[e]
 *   w1t_s  atom (e * 2f/128 + j) * d/128 + n / 128, rows n = columns of W1[e],
 *          K = its 2f rows
 *   w2_s   atom (e * d/128 + r / 128) * f/128 + j, rows r = rows of W2[e]
 *   w2t_s  atom (e * d/128 + j) * f/128 + n / 128, rows n = columns of W2[e], K = its
 *          d rows
 * The forward GEMMs use w1 and w2, the input-gradient GEMMs w2t and w1t. */
typedef struct moe_mx_weights {
  const uint8_t* w1_q;
  const uint8_t* w1_s;
  const uint8_t* w1t_q;
  const uint8_t* w1t_s;
  const uint8_t* w2_q;
  const uint8_t* w2_s;
  const uint8_t* w2t_q;
  const uint8_t* w2t_s;
} moe_mx_weights;

/* ---- MXFP8 weight copies ---------------------------------------------------
 * [kongchang] boundary-conditions section: MXFP8 operands with an authoritative FP32
 * master weight.  Writes all eight buffers of *out (a HOST struct whose members are
 * device pointers; the call writes through them) from the FP32 masters
 * w1 [E, 2f, d] and w2 [E, d, f], each element quantised as mxfp8_quantize does
 * (OCP floor rule), in one pass over each master.  d % 128 == 0, f % 128 == 0. */
moe_status moe_mx_quantize_weights(moe_shape shape, const float* w1, const float* w2,
                                   const moe_mx_weights* out, void* stream);

/* ---- f1: MXFP8 dispatch (permute fused with the quantisation of x) --------
 * [kongchang] boundary-conditions section: MXFP8 cuts the bytes the dispatch
 * moves.  Instead of copying bf16 rows into x_perm for the MXFP8 grouped FFN to
 * quantise, this call reads each routed row of x once where it lies and writes
 * only the two MXFP8 copies the GEMMs use: along d (E4M3 rows, 1 byte per
 * element + one E8M0 byte per 32) and in 32-row token blocks restarting at every
 * expert (for the dW1 GEMM of the backward).  Both go to `ws`, with the row maps,
 * where moe_grouped_ffn_fwd (dtype MOE_MXFP8, x_perm = NULL) reads them; no
 * call may use `ws` in between.  The result is bit-identical to moe_permute
 * followed by the forward's own quantisation.
 * x: bf16 [T, d]; slot_row, offsets: from moe_route (dropless, rows = T*k);
 * perm_src: int32 [T*k] written as in moe_permute (row r came from token
 * perm_src[r]).  Needs d % 128 == 0 and f % 128 == 0 (else MOE_ERR_UNSUPPORTED);
 * ws_bytes >= moe_workspace_size(shape, MOE_MXFP8, T*k). */
moe_status moe_permute_mx(moe_shape shape, const void* x, const int32_t* slot_row,
                          const int32_t* offsets, int32_t* perm_src, void* ws, size_t ws_bytes,
                          void* stream);

/* ---- MXFP8 operand copies in the workspace (diagnostic) ------------------
 * The MXFP8 grouped FFN calls keep each quantised activation in `ws`: a row copy
 * (E4M3 codes [rows, K] row-major, blocks of 32 along each row; E8M0 scales as
 * 512-byte MMA atoms per 128-row tile of the row-grouped GEMMs) and a token-block
 * copy (codes [K][Rp], blocks of 32 rows within each column restarting at every
 * expert offset, stored column by column; scales as atoms per 128-row stage of the
 * token axis).  This call
 * writes the byte offsets, from the start of `ws`, of the 20 regions below into
 * offsets_out[0..19] (n >= 20), for a workspace sized by moe_workspace_size(shape,
 * MOE_MXFP8, rows) (rows <= 0 means T*top_k), so that tests and debuggers can read
 * the bytes the layer produced.  No launch and no device access.  Token-block codes are
 * column-major over a stage-padded token axis of Rp = (rows/128 + E) * 128 positions:
 * every expert's tokens start a 128-row stage (stage numbering as for the atoms), column
 * c's code of the token at position p is at byte c * Rp + p, and the positions past an
 * expert's last token up to the end of its last stage hold code 0.
 *   0 x token-block codes [d][Rp]        1 x token-block scale atoms
 *   2 h token-block codes [f][Rp]        3 h token-block scale atoms
 *   4 row_tile int32 [rows]: row r -> 128 * tile + row within the tile (-1 outside)
 *   5 token blocks int4 [rows/32 + E]: {first row, rows (1..32), stage,
 *     block in stage | 4 if last of its expert}, then the stage table int32
 *     [rows/128 + E + 1]: first token block of each stage (entry nstages = nblocks)
 *   6 int32 [2]: number of token blocks, number of stages
 *   7 x row codes [rows, d]   8 x row-tile scale atoms
 *   9 h row codes [rows, f]  10 h row-tile scale atoms
 *  11 [da | du] bf16 [rows, 2f] (the SwiGLU-backward epilogue writes [da | du] straight
 *     into 14-15 and 18-19; this region holds bf16 [da | du] only in the library's
 *     diagnostic forms, and each routed row's gate (fp32 [rows]) during
 *     moe_combine_bwd_mx)
 *  12 dy row codes [rows, d]  13 dy row-tile atoms  14 [da|du] row codes [rows, 2f]
 *  15 [da|du] row-tile atoms  16 dy token-block codes [d][Rp]  17 dy token-block atoms
 *  18 [da|du] token-block codes [2f][Rp]  19 [da|du] token-block atoms
 * Regions 0-6 hold from the forward (moe_permute_mx writes 0, 1 and 4-8) to the
 * backward; 7-10 from the forward until the backward starts (they share memory
 * with 11-19); 11-19 after the backward (moe_combine_bwd_mx writes 12, 13, 16 and 17,
 * which the backward then reads).  Atom byte of (row r, block kb) within a
 * 128 x 4-block atom: (r % 32) * 16 + (r / 32) * 4 + kb; row-tile atom index
 * tile * (K/128) + K/128-column block; token-block atom index stage * (K/128) +
 * column block, with the blocks of a stage as kb (blocks past an expert's last one
 * hold 0x7F, the scale 2^0).  d % 128 == 0 and f % 128 == 0 (else
 * MOE_ERR_UNSUPPORTED); a bad shape or pointer: MOE_ERR_INVALID_ARG. */
moe_status moe_mx_workspace_layout(moe_shape shape, int64_t rows, int64_t* offsets_out, int n);

/* ---- a4: grouped SwiGLU FFN, forward -------------------------------------
 * [kongchang] routing section: a device-scheduled grouped GEMM handles the
 * uneven per-expert shapes; the tile scheduler reads `offsets` from device
 * memory (no host round trip for group sizes).
 * For expert e and rows r in [offsets[e], offsets[e+1]):
 *   a = X W1[e,0:f]^T, u = X W1[e,f:2f]^T, h = silu(a)*u, y = h W2[e]^T
 * rows:     number of rows of x_perm / y_perm / act_saved (T*k dropless;
 *           E*capacity padded).  offsets[E] <= rows.
 * x_perm:   [rows, d];  w1: [E, 2f, d] (gate rows then up rows);
 * w2:       [E, d, f];  act_saved: [rows, 3f] = a | u | h (saved for bwd);
 * y_perm:   [rows, d].  Rows outside every expert segment are not written.
 * MOE_BF16 needs d % 256 == 0 and f % 256 == 0 (tensor-core tiles); mx is NULL.
 * MOE_MXFP8 (kongchang, boundary-conditions section: MXFP8 cuts GEMM time and
 * saved-activation bytes): x_perm, act_saved and y_perm stay bf16; mx is a HOST
 * pointer to a moe_mx_weights whose members are device pointers (w1, w2 are not
 * read and may be NULL); x (in one pass) and h (in the gate/up GEMM's epilogue) are
 * quantised along their rows (for this call's GEMMs) and in 32-row token blocks (kept in
 * `ws` for the backward), and the GEMMs run block-scaled E4M3 x E4M3 with fp32
 * accumulation.  Needs d % 128 == 0 and f % 128 == 0, and `ws` 32-byte aligned.  x_perm
 * may be NULL when moe_permute_mx has just filled `ws` for the same offsets (the x
 * quantisation is then skipped). */
moe_status moe_grouped_ffn_fwd(moe_shape shape, int dtype, int64_t rows, const void* x_perm,
                               const int32_t* offsets, const void* w1, const void* w2,
                               const void* mx, void* act_saved, void* y_perm, void* ws,
                               size_t ws_bytes, void* stream);

/* ---- a5: gate-weighted combine -------------------------------------------
 *   out[t,:] = sum_{j ascending, slot_row[t,j] >= 0} topk_gate[t,j] * y_perm[slot_row[t,j],:]
 * fp32 accumulation, rounded once to the output type.  A row index of -1
 * (a pair dropped by the padded layout) contributes nothing.
 * y_perm: [rows, d]; out: [T, d]. */
moe_status moe_combine(moe_shape shape, int dtype, const void* y_perm, const int32_t* slot_row,
                       const float* topk_gate, void* out, void* stream);

/* ---- a6: combine backward ------------------------------------------------
 *   dgate[t,j]            = <dout[t,:], y_perm[slot_row[t,j],:]>   (fp32 [T,k])
 *   dy_perm[slot_row[t,j]] = topk_gate[t,j] * dout[t,:]           ([rows, d])
 * Pairs with slot_row -1 get dgate 0 and write no row.  Rows of dy_perm not
 * named by slot_row are not written (zero them once for the padded layout). */
moe_status moe_combine_bwd(moe_shape shape, int dtype, const void* dout, const void* y_perm,
                           const int32_t* slot_row, const float* topk_gate, void* dy_perm,
                           float* dgate, void* stream);

/* ---- f1 (backward): MXFP8 combine backward --------------------------------
 * [kongchang] boundary-conditions section: MXFP8 cuts the bytes the rows move.  In the
 * MXFP8 layer the rows dy_perm[slot_row[t,j]] = topk_gate[t,j] * dout[t,:] are read only
 * as their two MXFP8 copies (along d for the dh GEMM, in 32-row token blocks for the dW2
 * GEMM).  This call writes dgate exactly as moe_combine_bwd does (fp32 [T, k]) and those
 * two copies into `ws`, each operand row r taken from dout[perm_src[r],:] times its gate,
 * rounded to bf16 first as moe_combine_bwd rounds dy_perm, without writing dy_perm; then
 * moe_grouped_ffn_bwd (MOE_MXFP8, dy_perm = NULL) reads them.  The result is bit-identical
 * to moe_combine_bwd followed by that backward's own quantisation of dy_perm.
 * dout, y_perm: bf16 [T, d] / [T*k, d]; slot_row, perm_src: from the dropless route and
 * dispatch (perm_src[r] = the token of row r); topk_gate: the gates the combine used.
 * `ws` must be the workspace of this step's MXFP8 forward (moe_grouped_ffn_fwd, which
 * leaves the row and block maps there), sized for rows = T*top_k, with no call using it
 * in between.  Not with moe_grouped_ffn_bwd_recompute, whose forward half reuses that
 * memory.  d % 128 == 0 and f % 128 == 0 (else MOE_ERR_UNSUPPORTED). */
moe_status moe_combine_bwd_mx(moe_shape shape, const void* dout, const void* y_perm,
                              const int32_t* slot_row, const float* topk_gate,
                              const int32_t* perm_src, float* dgate, void* ws, size_t ws_bytes,
                              void* stream);

/* ---- a7 + a8: grouped SwiGLU FFN, backward -------------------------------
 * Per expert e on its rows: dh = dy W2[e]; s = sigmoid(a);
 *   da = dh*u*s*(1 + a*(1-s)); du = dh*silu(a);
 *   dx_perm = da W1[e,0:f] + du W1[e,f:2f];
 *   dW2[e] = dy^T h; dW1[e,0:f] = da^T x; dW1[e,f:2f] = du^T x.
 * An expert with no rows gets dW1[e] = dW2[e] = 0 (dW is overwritten; with
 * MOE_DW_ACCUMULATE in dw_dtype it is added to, and such an expert's dW is unchanged).
 * dy_perm, x_perm: [rows, d]; act_saved: [rows, 3f] from the forward, 32-byte
 * aligned for MOE_BF16 and MOE_MXFP8 (a and u are read in 32-byte pieces; a
 * buffer aligned only to 16 bytes gets MOE_ERR_INVALID_ARG);
 * dx_perm: [rows, d]; dw1: [E, 2f, d]; dw2: [E, d, f] of type dw_dtype
 * (MOE_F32 or MOE_BF16; MOE_F32 only when dtype is MOE_F32 or MOE_MXFP8).
 * Uses 2*f*rows elements of scratch in `ws` for [da | du].
 * MOE_MXFP8: dy_perm, x_perm, act_saved, dx_perm bf16; mx as for the forward; `ws`
 * 32-byte aligned; dy (in one pass) and [da | du] (in the SwiGLU-backward GEMM's
 * epilogue) are quantised along their rows for the dgrad GEMMs, and dy, h, [da | du], x
 * in 32-row blocks restarting at every expert for the wgrad GEMMs.  The
 * token-block copies of x and h (and the row/block maps) are the ones the forward of the
 * same step wrote into `ws`: pass the same workspace, with no call using it in between
 * (moe_combine and moe_combine_bwd take none), and the same offsets.  x_perm is not
 * read and may be NULL.  dy_perm may be NULL when moe_combine_bwd_mx has just written
 * dy's copies into `ws` (its quantisation is then skipped). */
moe_status moe_grouped_ffn_bwd(moe_shape shape, int dtype, int64_t rows, const void* dy_perm,
                               const void* x_perm, const void* act_saved,
                               const int32_t* offsets, const void* w1, const void* w2,
                               const void* mx, void* dx_perm, void* dw1, void* dw2,
                               int dw_dtype, void* ws, size_t ws_bytes, void* stream);

/* ---- f3: grouped FFN backward with recompute ------------------------------
 * [kongchang] boundary-conditions section: keeping only the layer input and
 * recomputing the expert activations in the backward trades about a fifth of
 * the throughput for two thirds of the activation memory.
 * Same arguments and results as moe_grouped_ffn_bwd, except that act_scratch
 * ([rows, 3f], same type as act_saved) need not hold anything: the call first
 * recomputes a | u | h into it from x_perm with the gate/up GEMM of the
 * forward (for MOE_MXFP8 also the token-block copies of x and h in `ws`, so the
 * workspace may have served other calls since the forward), then runs the
 * backward.  One act_scratch can serve every layer of a model.  act_scratch
 * is overwritten; its contents afterwards are this layer's a | u | h.  x_perm
 * and dy_perm are required here, for every dtype. */
moe_status moe_grouped_ffn_bwd_recompute(moe_shape shape, int dtype, int64_t rows,
                                         const void* dy_perm, const void* x_perm,
                                         void* act_scratch, const int32_t* offsets,
                                         const void* w1, const void* w2, const void* mx,
                                         void* dx_perm, void* dw1, void* dw2, int dw_dtype,
                                         void* ws, size_t ws_bytes, void* stream);

/* ---- a9: unpermute-grad + router grad ------------------------------------
 *   dx[t,:]  = sum_{j, slot_row[t,j] >= 0} dx_perm[slot_row[t,j],:] + sum_e dl[t,e] w_router[e,:]
 *   dl[t,:]  = p * (dp - <p, dp>),  p = softmax(logits[t,:]),
 *              dp[e] = dgate[t,j] where e = topk_idx[t,j], else 0
 *   dw_router = dl^T x                                   (fp32 [E, d], overwritten;
 *               added to instead with MOE_DW_ACCUMULATE OR-ed into dtype)
 * x, dx: [T, d]; w_router: [E, d]; logits fp32 [T,E]; dgate fp32 [T,k].
 * slot_row may be NULL: dx_perm is then [T, d] and its row t, the sum of token t's
 * expert-row gradients (as moe_ep_combine gathers them under expert parallelism), is
 * what is added to dx[t].
 * Deterministic: fixed summation order, no floating-point atomics. */
moe_status moe_route_bwd(moe_shape shape, int dtype, const void* x, const void* w_router,
                         const float* logits, const int32_t* topk_idx, const float* dgate,
                         const void* dx_perm, const int32_t* slot_row, void* dx,
                         float* dw_router, void* ws, size_t ws_bytes, void* stream);

/* ---- f2: expert parallelism across ranks -----------------------------------
 * [kongchang] capacity-tax section: expert parallelism spreads the routed experts over
 * the ranks and writes only the selected token rows directly into the target rank's
 * buffer; routing section: the exchange's split sizes never go to the host.
 * [bytechap] how it works: each device holds a fraction of the experts, and routed rows
 * are placed directly in the experts' input buffers.
 * Setting: n_ranks ranks (one GPU each; n_ranks <= 64), each with its own T tokens
 * routed over all E experts (shape.E = the total; E % n_ranks == 0).  Rank o owns the
 * E_loc = E / n_ranks experts [o E_loc, (o + 1) E_loc).  An owner's receive buffer
 * holds its experts' rows expert by expert, within an expert by source rank, within a
 * source in token order: the rows one device would permute from the ranks' batches
 * concatenated (rank 0's tokens first), in the same order.
 * Peer buffers (peer_x, peer_y, peer_dy): a HOST array of n_ranks device pointers, entry
 * o = rank o's buffer as mapped on the calling device (a peer mapping over NVLink, e.g.
 * a symmetric-memory allocation, or this rank's own memory for o == rank), each with room
 * for every row the owner can receive (n_ranks * T * top_k rows of d_model at most).  The
 * kernels use plain loads and stores on them.  Ordering between ranks is the caller's:
 * the rows a call writes into other ranks' memory are visible to work the owner starts
 * after a collective (e.g. an NCCL all-reduce of one word) that follows the call on the
 * writer's stream; a reader must likewise wait until the owner's writes are done. */

/* Layout of the exchange.  counts_all: device int32 [n_ranks, E], row s = moe_route's
 * counts on rank s (gathered by the caller, e.g. an all-gather on the device).
 *   recv_offsets: int32 [E_loc + 1], this rank's receive-buffer segments (the last entry
 *                 = rows received), ready for moe_grouped_ffn_fwd / _bwd with E_loc experts;
 *   send_base:    int32 [E], for every expert e, the row of e's owner's buffer where this
 *                 rank's rows of e begin.
 * One launch of one block.  Bad sizes or pointers: MOE_ERR_INVALID_ARG. */
moe_status moe_ep_layout(moe_shape shape, int n_ranks, int rank, const int32_t* counts_all,
                         int32_t* recv_offsets, int32_t* send_base, void* stream);

/* Dispatch: for every pair (t, j), x[t] is written to row
 *   ep_row[t, j] = send_base[e] + slot_row[t, j] - offsets[e],   e = topk_idx[t, j]
 * of peer_x[e / E_loc] (each row of x read once, 16-byte stores through the peer
 * pointers); ep_row (int32 [T, k]) is written here for the combine steps.  x: [T, d] of
 * dtype (MOE_F32 or MOE_BF16); topk_idx, slot_row, offsets: this rank's moe_route results;
 * send_base: from moe_ep_layout.  A pair left unrouted by a routing pass that gave up a
 * wait (slot_row -1) gets ep_row -1 and moves nothing. */
moe_status moe_ep_dispatch(moe_shape shape, int dtype, int n_ranks, const void* x,
                           const int32_t* topk_idx, const int32_t* slot_row,
                           const int32_t* offsets, const int32_t* send_base, void* const* peer_x,
                           int32_t* ep_row, void* stream);

/* Combine from the owners' rows:
 *   out[t] = sum_{j ascending} gate[t, j] * peer_y[e / E_loc][ep_row[t, j]]
 * in fp32, rounded once to dtype; gate == NULL gives the plain sum (the gather of the
 * input-gradient rows after the owners' backward, then moe_route_bwd with slot_row NULL).
 * Rows with ep_row -1 contribute nothing.  out: [T, d]. */
moe_status moe_ep_combine(moe_shape shape, int dtype, int n_ranks, const void* const* peer_y,
                          const int32_t* topk_idx, const int32_t* ep_row, const float* gate,
                          void* out, void* stream);

/* Combine backward across ranks:
 *   dgate[t, j] = <dout[t], peer_y[o][ep_row[t, j]]>,  peer_dy[o][ep_row[t, j]] = gate[t, j] dout[t]
 * with o = topk_idx[t, j] / E_loc (fp32 dot products; dy rows written to the owners). */
moe_status moe_ep_combine_bwd(moe_shape shape, int dtype, int n_ranks, const void* dout,
                              const void* const* peer_y, const int32_t* topk_idx,
                              const int32_t* ep_row, const float* gate, void* const* peer_dy,
                              float* dgate, void* stream);

/* ---- a10: MXFP8 quantisation ---------------------------------------------
 * [kongchang] boundary-conditions section: MXFP8 shares one scale among every
 * 32 elements; an FP32 master weight is kept.  Rule (OCP MX reading):
 *   per block V of 32: amax = max|V_i|; e = floor(log2 amax) - 8, clamped to
 *   [-127, 127] (amax == 0 -> -127); scale byte = e + 127 (E8M0);
 *   q_i = E4M3 round-to-nearest-even of V_i / 2^e, saturated to +-448, the
 *   sign bit taken from V_i.
 * src: [rows, K] of src_dtype (MOE_F32 or MOE_BF16).
 * axis 0: blocks of 32 along each row (K % 32 == 0); scale: u8 [rows, K/32].
 * axis 1: blocks of 32 consecutive rows within each column, restarting at
 *   every segment start seg_offsets[g] (device int32 [nseg+1], or NULL for one
 *   segment [0, rows)); a segment's last partial block is zero-padded.
 *   scale: u8 [S, K] with S = sum_g ceil(len_g / 32), segment by segment
 *   (S <= rows/32 + nseg, a bound that needs no device data); K % 16 == 0.
 * q: u8 [rows, K].  Bytes are exact (bit-for-bit with the rule above). */
moe_status mxfp8_quantize(int64_t rows, int64_t K, int src_dtype, const void* src, int axis,
                          const int32_t* seg_offsets, int nseg, uint8_t* q, uint8_t* scale,
                          void* stream);

/* ---- a11: padded-capacity comparison layout ------------------------------
 * [kongchang] routing section: the report compares the device-scheduled
 * grouped GEMM with padding every expert batch to one uniform capacity.
 * With capacity C (e.g. ceil(1.25 * T*k / E)): a pair (t,j) with rank
 * q = slot_row[t,j] - offsets[topk_idx[t,j]] is kept iff q < C and then
 *   x_pad[e*C + q, :] = x[t, :],  pad_row[t,j] = e*C + q;  else pad_row = -1.
 * Unused rows of x_pad are zeroed; offsets_pad[e] = e*C (int32 [E+1]).
 * The grouped FFN, combine, combine-bwd and route-bwd calls then take
 * rows = E*C, offsets_pad and pad_row in place of offsets and slot_row.
 * x_pad: [E*C, d]; pad_row: int32 [T,k]. */
/* Capacity of the padded layout for capacity factor cf = cf_num / cf_den:
 *   C = ceil(cf * T*top_k / E), computed in exact integer arithmetic
 * ([kongchang] routing section: every expert batch padded to one uniform capacity;
 * the comparison uses cf = 5/4).  Returns -1 for a bad shape, cf_num <= 0,
 * cf_den <= 0, or a C above INT32_MAX.  Host only: no launch. */
int32_t moe_capacity(moe_shape shape, int32_t cf_num, int32_t cf_den);

moe_status moe_padded_dispatch(moe_shape shape, int dtype, int32_t capacity, const void* x,
                               const int32_t* topk_idx, const int32_t* slot_row,
                               const int32_t* offsets, void* x_pad, int32_t* pad_row,
                               int32_t* offsets_pad, void* stream);

/* ---- f4: load balance of a routing --------------------------------------
 * [kongchang] routing section: how evenly the rows spread over the experts
 * sets the grouped GEMM's speed, more than the auxiliary loss value does.
 * From counts (device int32 [E], as moe_route writes them), with R = sum c,
 * mean = R / E, writes device fp32 stats[8]:
 *   [0] R   [1] mean   [2] max(c)/mean   [3] min(c)/mean
 *   [4] coefficient of variation sqrt(sum (c - mean)^2 / E) / mean
 *   [5] number of experts with c == 0
 *   [6] dropped fraction sum max(0, c - C) / R  of a capacity-C layout
 *   [7] used fraction (R - dropped) / (E*C)     of its E*C slots
 * Ratios are 0 when R == 0; [6] and [7] are 0 when capacity == 0 (no padded
 * layout).  Totals are exact integers, the deviations are summed in double in
 * a fixed order, each entry rounded once to fp32.  One kernel; nothing goes
 * to the host.  capacity < 0 or a bad pointer: MOE_ERR_INVALID_ARG. */
moe_status moe_routing_stats(moe_shape shape, const int32_t* counts, int32_t capacity,
                             float* stats, void* stream);

/* ---- f4: renormalised gates (an optional gate rule) ----------------------
 * The pages fix no gate rule; moe_route's gates are the softmax values of the
 * selected experts as they are.  These two calls offer the other usual rule,
 * the selected values rescaled to sum to one over each token's k experts:
 *   S[t] = sum_j topk_gate[t,j] (in index order),  gate_out[t,j] = topk_gate[t,j] / S[t]
 * Use gate_out in place of topk_gate in moe_combine and moe_combine_bwd; the
 * gate gradient that moe_combine_bwd then writes (dgate_out) goes through
 *   dgate[t,j] = (dgate_out[t,j] - sum_i gate_out[t,i] dgate_out[t,i]) / S[t]
 * before moe_route_bwd, which takes dgate.  topk_gate is the un-renormalised
 * output of moe_route (fp32 [T,k]); gate_out, dgate_out, dgate: fp32 [T,k].
 * gate_out may be topk_gate itself (in place) only when no backward follows;
 * dgate may be dgate_out.  T == 0 is a no-op. */
moe_status moe_renorm_gates(moe_shape shape, const float* topk_gate, float* gate_out, void* stream);
moe_status moe_renorm_gates_bwd(moe_shape shape, const float* topk_gate, const float* dgate_out,
                                float* dgate, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
