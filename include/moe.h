/*
 * moe.h — C ABI of the B200 (sm_100a) dropless sparse-MoE expert-MLP forward.
 *
 * The operation, as the pages state it:
 *  - router: H(X) = Softmax(TopK(X W_gate, k))
 *      ("ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs",
 *       "1. The Dynamic Routing Imbalance Dilemma", router equation);
 *  - sparse map: Histogram(e), Offsets(e) and an expert-sorted route index I
 *      (same page, "2. Grouped Coordinate Indexing Without Padding"; and "Add scalable sparse map
 *       kernel for large MoE models (128+ experts)", "Pass 1", "Pass 2" and "Usage");
 *  - ParallelLinear(X, W, I, G): gather rows on load, multiply by W[expert], scale by the router
 *    weight and scatter-add into token order (ScatterMoE guide, "1. The Anatomy of ParallelLinear"
 *    and "The ParallelLinear Core Abstraction" figure, Steps 1-3);
 *  - SwiGLU expert MLP y = sum_j w_j (silu(x W_gate_e[e_j]) * (x W_up[e_j])) W_down[e_j]
 *    (ScatterMoE guide, "3. Assembling the ScatterMoE FFN Block"; fused gate+up as in the
 *     abstract of "Cross-Platform Fused MoE Dispatch in Triton").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major and contiguous.
 *    Tensors read by the tensor cores (x, weights, X, Y, out) must be 16-byte aligned; int32 and
 *    float32 side arrays must be 4-byte aligned. The library never allocates device memory in
 *    these calls: scratch space comes from the caller's workspace `ws` (size from
 *    moe_workspace_size, alignment 256 bytes).
 *  - Environment: MOE_GEMM_2SM=1 (or 0) forces the grouped GEMMs onto CTA pairs (or single CTAs)
 *    instead of the library's choice by rows per expert; MOE_PREGATHER=0 keeps moe_mlp_forward's
 *    first GEMM gathering x rows on load where it would copy them to slot order first. Results
 *    are the same either way (the parity tests run both). No other environment variable is read.
 *  - One device per process: the first call that launches a kernel needing more than 48 KB of
 *    shared memory raises that kernel's limit (cudaFuncSetAttribute) once, for the device current
 *    at that call. A process that then calls on another device gets MOE_ERR_CUDA from those
 *    launches. Run one process per GPU, as the bench and the expert-parallel path do.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *    never synchronise the host. Argument errors are detected on the host and returned before any
 *    launch. Errors the device detects (an expert id outside [0,E), a bounded wait that ran out)
 *    set a status word inside `ws`; moe_check_device_status() synchronises the stream and reports
 *    it. Every call that takes `ws` clears that word first.
 *  - Return value: MOE_OK (0) or a negative moe_status; moe_last_error() gives a message for the
 *    last failing call on the calling host thread.
 *  - Limits checked on the host: 1 <= k <= min(E, 8); E <= 256; 0 <= S and S*k < 2^31;
 *    D, F, Din, Dout multiples of 8 and > 0; all dims < 2^31.
 *  - Floating point: bf16 inputs multiply on the tensor cores with fp32 accumulation; fp32 inputs
 *    multiply as tf32 with fp32 accumulation; the router accumulates in fp32 on the CUDA cores.
 *    Scatter outputs are fp32 and use fp32 atomic adds, so their last bits may differ between
 *    runs. The sparse map is exact and deterministic.
 *  - Requires a device of compute capability 10.0 (B200, sm_100a); other devices get
 *    MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,    /* null / misaligned pointer, bad size or limit */
    MOE_ERR_UNSUPPORTED = -2,    /* device is not sm_100, or dtype not supported */
    MOE_ERR_WORKSPACE = -3,      /* ws is null, misaligned or smaller than moe_workspace_size */
    MOE_ERR_CUDA = -4,           /* a CUDA runtime / driver call failed */
    MOE_ERR_BAD_EXPERT_ID = -5,  /* device saw an expert id outside [0, E) */
    MOE_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait ran out; the kernel returned */
    MOE_ERR_BAD_INDEX = -7       /* debug build only: a device bounds check skipped an index */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/*
 * Router: per token s, logits l = x[s] . W_gate (+ logit_bias), then the k largest logits in
 * descending order (equal logits: smaller expert id first) and their softmax weights
 * w_j = exp(l_{e_j} - l_{e_0}) / sum_j' exp(l_{e_j'} - l_{e_0}).
 *   x           [S, D]  dt        token activations
 *   w_gate      [D, E]  dt        router weight (x . W_gate, E contiguous)
 *   logit_bias  [E]     float32   nullable; added to the logits before selection and softmax
 *   top_experts [S, k]  int32     out
 *   top_weights [S, k]  float32   out
 * Cites: ScatterMoE guide, "1. The Dynamic Routing Imbalance Dilemma" (router equation) and
 * "3. Assembling the ScatterMoE FFN Block" (softmax, top-k, renormalise).
 */
int moe_route_topk(const void *x, const void *w_gate, const float *logit_bias, int64_t S,
                   int64_t D, int32_t E, int32_t k, moe_dtype dt, int32_t *top_experts,
                   float *top_weights, moe_stream_t stream);

/*
 * Sparse map of the flat route list i = s*k + j, expert(i) = top_experts[i]:
 *   expert_counts  [E]    int32  out  Histogram(e) = #{i : expert(i) = e}
 *   expert_offsets [E+1]  int32  out  Offsets(e) = sum_{e'<e} Histogram(e'); offsets[E] = S*k.
 *                                     expert_offsets[1..E] are the "expert_ends" of the Fast-LLM
 *                                     API; with zero padding the "pad begins" equal the ends.
 *   sparse_rows    [S*k]  int32  out  slot of route i: offsets[e] + #{i' < i : expert(i') = e}
 *   sorted_rows    [S*k]  int32  out  inverse permutation: sorted_rows[sparse_rows[i]] = i
 * Slots inside an expert follow increasing i (stable), so the result is unique and bit-exact.
 * An id outside [0,E) is not counted, gets sparse_rows[i] = -1, and sets MOE_ERR_BAD_EXPERT_ID in
 * the device status.  ws: moe_workspace_size("sparse_map", S, 0, 0, E, k, dt) bytes.
 * Cites: ScatterMoE guide, "2. Grouped Coordinate Indexing Without Padding"; "Add scalable sparse
 * map kernel for large MoE models (128+ experts)", "Pass 1: Histogram with Atomics", "Pass 2: Two
 * Assignment Variants", "4. Correctness Validation" and "Usage".
 */
int moe_sparse_map(const int32_t *top_experts, int64_t S, int32_t k, int32_t E,
                   int32_t *expert_counts, int32_t *expert_offsets, int32_t *sparse_rows,
                   int32_t *sorted_rows, void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Sparse map without any workspace: the same outputs as moe_sparse_map (bit-identical), for
 * callers that can pass their input and output buffers but cannot obtain extra device memory at
 * call time, such as plugin-style interfaces that hand over only fixed input/output bindings, or
 * runtimes that keep all device memory in their own pool, where a cudaMalloc for scratch would
 * fail or stall the device. The pages have no counterpart of this entry point.
 * The scratch is a fixed array inside the library: 1 MiB of counters plus a 256-byte status area,
 * held on every device that loads the library until the process exits. Sizes must satisfy
 * (ceil(S*k / 4096) + 1) * E * 4 <= 1 MiB (for example S*k <= 4190208 routes at E = 256); larger
 * sizes are rejected with MOE_ERR_INVALID_ARG before any launch. The call allocates nothing.
 * The first call on a device looks up the array's device address (with that device current);
 * make that first call before any stream capture. Under CUDA's lazy module loading (the default)
 * that first call may also be what loads this library's device code on the device, and with it
 * what reserves the fixed array in device memory: make it before a memory pool takes the rest
 * of the device. All calls share the array, which keeps the
 * last call's contents; calls whose kernels overlap on the GPU (e.g. on two streams) race on it
 * and must be serialised by the caller. An expert id outside [0,E) is not counted and gets
 * sparse_rows[i] = -1; this call reports no device status, so such ids show as
 * expert_offsets[E] < S*k.
 */
int moe_sparse_map_noalloc(const int32_t *top_experts, int64_t S, int32_t k, int32_t E,
                           int32_t *expert_counts, int32_t *expert_offsets, int32_t *sparse_rows,
                           int32_t *sorted_rows, moe_stream_t stream);

/*
 * ParallelLinear(X, W, I, G): for each slot p of expert e (offsets[e] <= p < offsets[e+1]),
 * route i = sorted_rows[p], token s = i / k:
 *   v_p = src_p . W[e]   with src_p = X[s] (gather_in = 1, X is [S, Din] in token order)
 *                        or   src_p = X[p] (gather_in = 0, X is [S*k, Din] in slot order)
 *   c_p = top_weights[i] * v_p   (top_weights nullable: no scaling)
 *   scatter_out = 1: Y[s] += c_p  (Y is [S, Dout] float32; the caller zeroes it first)
 *   scatter_out = 0: Y[p]  = c_p  (Y is [S*k, Dout] in dt, slot order)
 *   W [E, Din, Dout] dt; sorted_rows [S*k], expert_offsets [E+1] as from moe_sparse_map.
 * ws: moe_workspace_size("scatter_linear", ...) bytes (holds the device status word).
 * Cites: ScatterMoE guide, "1. The Anatomy of ParallelLinear", "The ParallelLinear Core
 * Abstraction" figure (Steps 1-3) and "2. Grouped Coordinate Indexing Without Padding" (tiles of
 * an expert's rows, last tile masked, no padding in memory).
 */
int moe_scatter_linear(const void *X, const void *W, int64_t S, int64_t Din, int64_t Dout,
                       int32_t E, int32_t k, const int32_t *sorted_rows,
                       const int32_t *expert_offsets, const float *top_weights, int gather_in,
                       int scatter_out, moe_dtype dt, void *Y, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/*
 * Backward of moe_scatter_linear (ScatterMoE guide, "3. Fused Backward Pass Dynamics"): with the
 * forward's X, W, sorted_rows, expert_offsets, top_weights, gather_in and scatter_out, and dY
 * shaped like the forward's Y, for every slot p of expert e (route i, token s):
 *   dc_p = dY[s] (scatter_out) or dY[p];  dv_p = top_weights[i] * dc_p (1 without top_weights)
 *   dX[s] += dv_p . W[e]^T  (gather_in: dX [S, Din] float32, overwritten)
 *   dX[p]  = dv_p . W[e]^T  (else:      dX [S*k, Din] bf16)
 *   dW[e]  = sum over e's slots of src_p^T (x) dv_p, src_p = X[s] or X[p]  ([E, Din, Dout] f32)
 *   dgates[i] = dc_p . (src_p . W[e])   ([S*k] float32; needs top_weights)
 * dY: float32 [S, Dout] when scatter_out, else bf16 [S*k, Dout]. dX, dW and dgates are each
 * nullable (not computed) and 16-byte aligned; every output is overwritten (dW is zero for an
 * expert without slots; dgates is zero for a route whose expert id was out of range).
 * bf16 only (dt = MOE_BF16; MOE_ERR_UNSUPPORTED otherwise). The input gradient runs the forward's
 * grouped GEMM with the gather and scatter roles exchanged and W read transposed (K-major, no
 * copy); the weight gradient is a grouped GEMM whose reduction runs over each expert's slots
 * (fp32 accumulation in TMEM, bf16 operands: dY is rounded to bf16 once).
 * ws: moe_workspace_size("scatter_linear_backward", S, Din, Dout, E, k, dt) bytes.
 */
int moe_scatter_linear_backward(const void *X, const void *W, const void *dY, int64_t S,
                                int64_t Din, int64_t Dout, int32_t E, int32_t k,
                                const int32_t *sorted_rows, const int32_t *expert_offsets,
                                const float *top_weights, int gather_in, int scatter_out,
                                moe_dtype dt, void *dX, float *dW, float *dgates, void *ws,
                                size_t ws_bytes, moe_stream_t stream);

/*
 * Whole MoE expert-MLP forward:
 *   out[s] = sum_j w_j * ( silu(x[s] W_gate_e[e_j]) * (x[s] W_up[e_j]) ) W_down[e_j]
 * with (e_j, w_j) from moe_route_topk. Steps on `stream`: zero out, route, sparse map, GEMM1
 * (gathered x rows, fused gate+up, SwiGLU in registers, h in slot order), GEMM2 (h rows,
 * W_down, router weight, scatter-add into out). No host synchronisation.
 *   For bf16 with experts of 384 or more rows on average (S*k / E >= 384) and F >= 2048, GEMM1
 *   does not gather on load: one more kernel first copies the x rows to slot order inside the
 *   workspace ("x_sorted"), and GEMM1 reads them by TMA (set the environment variable
 *   MOE_PREGATHER=0 to gather on load instead; the workspace size does not change).
 *   x [S,D], w_gate [D,E], w_gate_e [E,D,F], w_up [E,D,F], w_down [E,F,D]: dt
 *   logit_bias [E] float32 nullable;  out [S,D] float32 (overwritten).
 *   ws: moe_workspace_size("mlp_forward", S, D, F, E, k, dt) bytes; after the call it holds the
 *   routing (see moe_workspace_view) until the next call that uses it.
 * Cites: ScatterMoE guide, "3. Assembling the ScatterMoE FFN Block" and "Enter ScatterMoE" pipeline
 * figure; fused gate+up from the abstract of "Cross-Platform Fused MoE Dispatch in Triton".
 */
int moe_mlp_forward(const void *x, const void *w_gate, const float *logit_bias,
                    const void *w_gate_e, const void *w_up, const void *w_down, int64_t S,
                    int64_t D, int64_t F, int32_t E, int32_t k, moe_dtype dt, float *out, void *ws,
                    size_t ws_bytes, moe_stream_t stream);

/*
 * Backward of moe_mlp_forward (bf16): given dout [S, D] float32 (the gradient of out) and the
 * workspace of the forward call on the same inputs (fwd_ws: its routing, sparse map and h), the
 * float32 gradients (all overwritten, all required):
 *   dx [S, D], dw_gate [D, E], dw_gate_e [E, D, F], dw_up [E, D, F], dw_down [E, F, D].
 * The selection of the top-k experts has no derivative; the weights are the softmax over the
 * selected logits, differentiated through it. Steps on `stream`:
 *   1. dout rows (bf16) and x rows copied to slot order.
 *   2. dh = dout[s] . W_down[e]^T per slot (the forward's grouped GEMM, W_down read K-major).
 *   3. The fused gate+up GEMM recomputed on the slot-ordered x rows, with the SwiGLU backward in
 *      its epilogue: the route-weight gradient dh . h, then da and db.
 *   4. dW_down (weight-gradient GEMM over each expert's slots).
 *   5. dx += [da | db] . [W_gate_e ; W_up]^T (scatter-added into tokens).
 *   6. dW_gate_e and dW_up.
 *   7. Router backward: the softmax Jacobian, then dx += dl W_gate^T and dW_gate = x^T dl.
 * ScatterMoE guide, "3. Fused Backward Pass Dynamics" (each ParallelLinear's input and weight
 * gradients). Constraints beyond the forward's: bf16 only, E a multiple of 8, F a multiple of 64.
 * ws: moe_workspace_size("mlp_backward", S, D, F, E, k, dt) bytes.
 */
int moe_mlp_backward(const void *x, const void *w_gate, const void *w_gate_e, const void *w_up,
                     const void *w_down, const float *dout, int64_t S, int64_t D, int64_t F,
                     int32_t E, int32_t k, moe_dtype dt, const void *fwd_ws, size_t fwd_ws_bytes,
                     float *dx, float *dw_gate, float *dw_gate_e, float *dw_up, float *dw_down,
                     void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Mixture of Attention forward (ScatterMoE guide, "2. Generalization to Mixture of Attention
 * (MoA)"; the ScatterMoE abstract's MoA demonstration), bf16. The router of moe_route_topk picks
 * k of E attention experts per token; expert e owns a query projection W_q[e] and an output
 * projection W_o[e]; keys and values are shared by all experts. For token s, selected expert
 * e_j with router weight w_j, and head h (H heads of dh columns, HD = H * dh):
 *   q = x[s] W_q[e_j];  K = x W_kv[:, :HD];  V = x W_kv[:, HD:]
 *   o_h = sum_{t <= s} softmax_t(q_h . K[t, h] / sqrt(dh)) V[t, h]   (causal, one sequence)
 *   out[s] = sum_j w_j * (o W_o[e_j])
 * Steps on `stream`: route, sparse map, the shared key/value projection (one group of all S
 * tokens, [S, D] x [D, 2 HD]; its epilogue warps zero `out`), the routed query projection
 * (ParallelLinear with gathered x rows, q in slot order), the attention core over the slot-ordered
 * query rows (tensor cores, running-max softmax, each row masked at its own token position), and
 * the routed output projection (ParallelLinear from slot order, router weight, scatter-add into
 * tokens). No host synchronisation.
 *   x [S, D], w_gate [D, E], w_q [E, D, HD], w_kv [D, 2 HD], w_o [E, HD, D]: bf16;
 *   logit_bias [E] float32 nullable; out [S, D] float32 (overwritten). dh is 64 or 128.
 *   ws: moe_workspace_size("moa_forward", S, D, HD, E, k, MOE_BF16) bytes; the routing views of
 *   moe_workspace_view (top_experts ... sorted_rows, any F) apply to it.
 * MOE_ERR_UNSUPPORTED for another dtype or head size.
 */
int moe_moa_forward(const void *x, const void *w_gate, const float *logit_bias, const void *w_q,
                    const void *w_kv, const void *w_o, int64_t S, int64_t D, int32_t H, int32_t dh,
                    int32_t E, int32_t k, moe_dtype dt, float *out, void *ws, size_t ws_bytes,
                    moe_stream_t stream);

/*
 * Expert parallelism (ScatterMoE guide, "Combine with Tensor and Pipeline Parallelism": expert
 * weights spread over expert-parallel ranks, ParallelLinear running each rank's local experts).
 * The E experts are split into contiguous ranges, one per rank. A forward is:
 *   route (moe_route_topk) -> moe_ep_dispatch -> all-to-all of the rows (caller, e.g. NCCL)
 *   -> moe_expert_mlp_forward on the received rows -> all-to-all back -> moe_ep_combine.
 * The library does no communication; these calls prepare and consume the exchanged buffers.
 *
 * moe_ep_dispatch: the sparse map of top_experts (outputs as moe_sparse_map) plus the send
 * buffer in slot order: send_x[p] = x[sorted_rows[p] / k] ([S*k, D], dt) and
 * send_e[p] = top_experts[sorted_rows[p]] (the global expert id of row p). Slots are grouped by
 * expert, so rank r's rows are the contiguous range [expert_offsets[r*E/n], expert_offsets[(r+1)*E/n])
 * for n ranks of E/n experts each. Slots at or past expert_offsets[E] (routes with an id outside
 * [0,E)) are not written.
 *   ws: moe_workspace_size("ep_dispatch", S, D, 0, E, k, dt) bytes (status word + map scratch).
 */
int moe_ep_dispatch(const void *x, const int32_t *top_experts, int64_t S, int64_t D, int32_t E,
                    int32_t k, moe_dtype dt, int32_t *expert_counts, int32_t *expert_offsets,
                    int32_t *sparse_rows, int32_t *sorted_rows, void *send_x, int32_t *send_e,
                    void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The expert MLP on rows that arrive with their expert ids (the receiving side of expert
 * parallelism): for row i with local expert e = expert_ids[i] - expert_base (0 <= e < E),
 *   y[i] = (silu(x_rows[i] W_gate_e[e]) * (x_rows[i] W_up[e])) W_down[e]   (unweighted, fp32)
 * Steps: local ids, sparse map over the rows, GEMM1 (rows gathered on load, fused gate+up, SwiGLU),
 * GEMM2 (scatter-add into row order). A row whose id is out of range is reported through the
 * status word (MOE_ERR_BAD_EXPERT_ID) and its y row stays zero.
 *   x_rows [R, D], w_gate_e / w_up [E, D, F], w_down [E, F, D]: dt; expert_ids [R] int32;
 *   y [R, D] float32 (overwritten).
 *   ws: moe_workspace_size("expert_mlp_forward", R, D, F, E, 1, dt) bytes.
 */
int moe_expert_mlp_forward(const void *x_rows, const int32_t *expert_ids, int32_t expert_base,
                           int64_t R, int64_t D, int64_t F, int32_t E, const void *w_gate_e,
                           const void *w_up, const void *w_down, moe_dtype dt, float *y, void *ws,
                           size_t ws_bytes, moe_stream_t stream);

/*
 * Expert-parallel combine: out[s] = sum_j top_weights[s*k + j] * y_ret[sparse_rows[s*k + j]],
 * with y_ret [S*k, D] float32 the expert outputs returned into the send buffer's slot order and
 * sparse_rows the dispatch's map. Routes with sparse_rows outside [0, S*k) add nothing. out
 * [S, D] float32 is overwritten; every token sums its k rows in order (deterministic, no atomics).
 */
int moe_ep_combine(const float *y_ret, const int32_t *sparse_rows, const float *top_weights,
                   int64_t S, int64_t D, int32_t k, float *out, moe_stream_t stream);

/*
 * The optional last step of the forward: an fp32 output (e.g. moe_mlp_forward's `out`) rounded to
 * bf16, round-to-nearest-even, for callers whose activations are bf16 (the ScatterMoE guide's
 * forward returns the input's dtype). src [n] float32, dst [n] bf16, n a multiple of 8, both
 * 16-byte aligned; no workspace.
 */
int moe_cast_bf16(const float *src, int64_t n, void *dst, moe_stream_t stream);

/*
 * Workspace bytes for op = "sparse_map", "scatter_linear", "scatter_linear_backward" (D = Din,
 * F = Dout), "mlp_forward", "mlp_backward", "moa_forward" (F = H * dh), "ep_dispatch" or
 * "expert_mlp_forward" (S = rows, k = 1) (unused sizes may be 0). Returns 0 for an unknown op or sizes
 * outside the limits.
 */
size_t moe_workspace_size(const char *op, int64_t S, int64_t D, int64_t F, int32_t E, int32_t k,
                          moe_dtype dt);

/*
 * Byte offsets inside an "mlp_forward" workspace of the intermediate results the forward leaves
 * there (for inspection and tests): which = "top_experts" [S*k] int32, "top_weights" [S*k] f32,
 * "expert_counts" [E], "expert_offsets" [E+1], "sparse_rows" [S*k], "sorted_rows" [S*k] int32,
 * "h" [S*k, F] (bf16 for bf16, f32 for f32), "x_sorted" [S*k, D] (the x rows in slot order, only
 * in workspaces of shapes whose forward copies them, see moe_mlp_forward; -1 otherwise). Returns
 * -1 for an unknown name.
 */
int64_t moe_workspace_view(const char *which, int64_t S, int64_t D, int64_t F, int32_t E,
                           int32_t k, moe_dtype dt);

/* Message for the last failing call on this host thread ("" if none). */
const char *moe_last_error(void);

/*
 * Synchronises `stream`, reads the status word in `ws` and returns MOE_OK,
 * MOE_ERR_BAD_EXPERT_ID, MOE_ERR_DEVICE_TIMEOUT or, from the debug build, MOE_ERR_BAD_INDEX
 * (or MOE_ERR_CUDA). Off the hot path.
 */
int moe_check_device_status(void *ws, moe_stream_t stream);

/*
 * 1 in the debug build of this library (libmoe_b200_debug.so, compiled with MOE_DEBUG=1), 0 in
 * the release build. The debug build has the same entry points and results; in addition every
 * index a kernel takes from its inputs before addressing memory with it (a gathered token row
 * sorted_rows[p] / k, a slot, a route, the expert offsets behind a tile schedule) is checked
 * against its range. An index outside it skips that access (the row is not read or written;
 * out-of-range expert offsets empty the schedule) and sets MOE_ERR_BAD_INDEX in the status word
 * read by moe_check_device_status. Nothing traps. This stands in for a memory sanitizer, which
 * is not available where this library was measured. Not an operation of the pages.
 */
int moe_debug_build(void);

/*
 * Optional per-stage timing on the calling host thread: when `events` holds n cudaEvent_t
 * handles (n <= 8), the next moe_mlp_forward, moe_mlp_backward or moe_moa_forward records the
 * first n of its stage events on its stream; then the registration clears.
 *   moe_mlp_forward (6): start, after route, after the sparse map, after the copy of the x rows
 *     to slot order (recorded at once when the forward makes none), after GEMM1, after GEMM2.
 *   moe_mlp_backward (7): start, after dh, after the recomputed GEMM1 with the SwiGLU backward,
 *     after dW_down, after dx, after dW_gate_e and dW_up, after the router backward.
 *   moe_moa_forward (7): start, after route, after the sparse map, after the key/value
 *     projection, after the query projection, after the attention core, after the output
 *     projection.
 * Pass n = 0 to clear. Returns MOE_OK or MOE_ERR_INVALID_ARG.
 */
int moe_profile_events(void *const *events, int n);

/*
 * Self-test of the bounded device wait: launches one block that waits on a barrier nothing
 * arrives at, with a limit of `limit_ns` nanoseconds (1 .. 10^9), then returns. The status word in
 * `ws` then reads MOE_ERR_DEVICE_TIMEOUT through moe_check_device_status. ws >= 256 bytes.
 */
int moe_debug_wait_timeout(int64_t limit_ns, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Number of kernels the last successful call on this host thread launched. */
int moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
