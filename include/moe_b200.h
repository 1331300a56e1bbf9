/*
 * moe_b200.h - C ABI of the single-GPU MoE dispatch-compute-combine hot path on B200.
 *
 * The layer (one GPU, no inter-GPU exchange):
 *
 *   moe_permute            route top-k copies into expert-contiguous order
 *   moe_grouped_ffn        y = Down_e(SwiGLU(Up_e x, Gate_e x)) for every expert's rows
 *   moe_unpermute_combine  out[t] = sum_k w[t,k] * y[row of (t,k)]
 *   moe_maxvio             max_e(T_e / T_bar) - 1
 *
 * Further calls, each documented where it is declared: the permutation without a workspace
 * argument (moe_permute_no_alloc); the layer's backward (moe_combine_backward,
 * moe_grouped_ffn_*_backward, moe_grouped_ffn_weight_grad, moe_permute_backward); the SwiGLU
 * pass reading token rows in place (moe_grouped_ffn_gather); shared experts
 * (moe_append_shared); and experts in MXFP8 (moe_mx_quantize_weights,
 * moe_mx_permute_quantize, moe_grouped_ffn_*mxfp8; "Mixture of Kittens" digest, Step 8).
 *
 * Sources (page title, section):
 *   "Distributed expert parallelism" (open-llm-engineering): "The dispatch-compute-combine
 *     lifecycle" (copy each token k times, sort copies by expert, grouped expert FFNs,
 *     restore token order, scale by route weight, sum the k results); "Token permutation
 *     and metadata" (expert-contiguous order plus the metadata that reverses it);
 *     "Failure modes ..." (empty experts, scatter-add rather than assign).
 *   "Mixture of Kittens" teaching digest, Step 1, The Math: Expert_i(x) =
 *     Down_i(SwiGLU(Up_i(x), Gate_i(x))).
 *   MoonEP README: "Integration" and "Weight buffer" (one contiguous weight tensor per
 *     projection, experts addressed by row index, cu_seqlens selects each expert's rows);
 *     "API walkthrough" (bf16 hidden states, fp32 route weights, int32 expert ids and
 *     counts); "Performance" (the maxvio formula).
 *
 * Conventions shared by every call:
 *   - All tensors are dense, row-major, caller-allocated device memory. The library never
 *     allocates, frees or keeps pointers across calls. bf16 tensors are passed as void*.
 *   - S tokens, K experts per token (slots), E experts, H hidden size, Hp = H' (expert
 *     intermediate size), M = S*K routed rows. Flat slot f = t*K + k.
 *   - Every call is asynchronous on `cuda_stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronises the host. The returned status covers argument checks
 *     and launch errors only; on any error nothing has been launched. Errors that depend
 *     on device data are OR-ed into *d_status (a device int32 the caller zeroes and reads
 *     when it chooses; may be NULL to skip reporting).
 *   - Preconditions, checked on the host: pointers non-NULL and 16-byte aligned (unless
 *     documented nullable), H and Hp multiples of 8 (of 128 for the grouped FFN calls),
 *     1 <= K <= E <= MOE_MAX_EXPERTS (E <= MOE_MAX_FFN_EXPERTS for the grouped FFN calls),
 *     S*K < 2^31. S = 0 (M = 0 rows) is legal: a call returns MOE_OK after its shape
 *     checks, reads and writes no row buffer (those may then be NULL, as a zero-size
 *     tensor's data pointer is), and only moe_permute's counts/offsets/maxvio and the
 *     weight gradients (zero when writing) are produced.
 *   - Results are deterministic: no floating-point atomics; every sum has a fixed order.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status;

#define MOE_OK 0
#define MOE_ERR_INVALID_ARGUMENT 1  /* null/misaligned pointer, negative size, K > E ... */
#define MOE_ERR_UNSUPPORTED_SHAPE 2 /* legal but outside what the kernels handle       */
#define MOE_ERR_CUDA 3              /* a CUDA runtime/driver call failed                 */
#define MOE_ERR_BAD_ROUTING 4       /* device: an expert id outside [0, E)               */
#define MOE_ERR_DEVICE_TIMEOUT 8    /* device: a bounded wait in a kernel ran out        */

/* Largest E of the routing calls (moe_permute, moe_permute_no_alloc, moe_maxvio,
 * moe_append_shared): expert ids fit in 16 bits. */
#define MOE_MAX_EXPERTS 65535

/* Largest E of the grouped FFN calls (forward, backward, MXFP8): every CTA of their
 * persistent grids keeps the per-expert row offsets and work-unit offsets in shared memory
 * (2 x 4 KiB at 1024 experts, next to 192 KiB of operand pipeline). */
#define MOE_MAX_FFN_EXPERTS 1024

/* Static description of a status code. Never NULL. */
const char* moe_status_string(moe_status s);

/* Version of this ABI, (major << 16) | minor. */
int32_t moe_abi_version(void);

/*
 * Bytes of device workspace moe_permute needs for (S, K, E). 0 when S*K <= 2^17 or
 * E > 1024: the metadata is then computed in one thread-block cluster's shared memory.
 * Otherwise the per-expert counts of every 512-slot chunk of the flat routing table,
 * rounded up to 256 bytes.
 */
size_t moe_permute_workspace_bytes(int64_t S, int32_t K, int32_t E);

/*
 * moe_permute - top-k route permutation into expert-contiguous order ("Distributed expert
 * parallelism", "Token permutation and metadata"; MoonEP README, "dispatch fwd").
 *
 *   x          [S, H] bf16 token states. May be NULL together with x_perm, or when S == 0
 *              (then topk_ids, row_id_map and perm_src may be NULL too).
 *   topk_ids   [S, K] int32 expert of every slot; K distinct ids per token are not required
 *              (a repeated id gives two rows that the combine adds).
 *   x_perm     [S*K, H] bf16 out: row row_id_map[f] = x[f / K]. NULL: metadata only.
 *   counts     [E] int32 out: rows per expert.
 *   cu_seqlens [E+1] int32 out: cu[0] = 0, cu[e+1] = cu[e] + counts[e], cu[E] = S*K. Expert e
 *              owns rows [cu[e], cu[e+1]). (MoonEP's end-offset array is cu_seqlens + 1.)
 *   row_id_map [S*K] int32 out: flat slot -> row. Inside one expert rows follow increasing
 *              f, i.e. (token, slot) order; the permutation is a bijection of [0, S*K).
 *   perm_src   [S*K] int32 out, nullable: row -> flat slot (inverse of row_id_map).
 *   maxvio     device double out, nullable: as moe_maxvio on the counts.
 *   max_count  device int32 out, nullable: max_e counts[e].
 *   workspace  device scratch of moe_permute_workspace_bytes(S, K, E) bytes (contents
 *              ignored on entry, undefined on exit); may be NULL when that size is 0.
 *   d_status   nullable device int32: MOE_ERR_BAD_ROUTING is OR-ed in if any id is outside
 *              [0, E); such slots are dropped (row_id_map[f] = -1) and counts no longer sum
 *              to S*K.
 */
moe_status moe_permute(const void* x, const int32_t* topk_ids, int64_t S, int64_t H, int32_t K,
                       int32_t E, void* x_perm, int32_t* counts, int32_t* cu_seqlens,
                       int32_t* row_id_map, int32_t* perm_src, double* maxvio, int32_t* max_count,
                       void* workspace, size_t workspace_bytes, int32_t* d_status,
                       void* cuda_stream);

/*
 * moe_permute_no_alloc - moe_permute for callers that cannot allocate device memory.
 *
 * This entry point has no counterpart in the pages this library follows; it exists for
 * callers that cannot hand moe_permute a workspace because they may not allocate device
 * memory at the point of the call: for example a plugin inside an inference engine whose
 * memory was planned up front, or a host framework that owns the whole device memory pool
 * and forbids cudaMalloc while it runs. It behaves exactly like moe_permute (same arguments
 * without workspace/workspace_bytes, same outputs bit for bit) but takes its scratch from
 * a fixed array inside this library's own device memory instead of from the caller.
 *
 *   - Limit: moe_permute_workspace_bytes(S, K, E) must be at most MOE_NO_ALLOC_SCRATCH_BYTES
 *     (4 MiB: every table of up to 2^17 routed slots, or with E > 1024, needs none; above
 *     that e.g. S*K up to 524288 routed slots with E up to 1024); larger problems return
 *     MOE_ERR_UNSUPPORTED_SHAPE and launch nothing. Use moe_permute with a workspace then.
 *   - Every GPU that loads the library holds this array until the process exits.
 *   - The first call in each CUDA context looks up the array's device address (with the
 *     device current) and keeps it for that context; a second context on the device, or the
 *     primary context re-created after cudaDeviceReset, does its own lookup on its first
 *     call. Make that first call before any stream capture.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - All calls on a device share the one array, and it keeps the last call's contents.
 *     Nothing in it has to start at zero (each call writes every entry it reads), but calls
 *     whose work overlaps on the GPU (e.g. on two streams at once) race on it: order them.
 */
#define MOE_NO_ALLOC_SCRATCH_BYTES (4u << 20)

moe_status moe_permute_no_alloc(const void* x, const int32_t* topk_ids, int64_t S, int64_t H,
                                int32_t K, int32_t E, void* x_perm, int32_t* counts,
                                int32_t* cu_seqlens, int32_t* row_id_map, int32_t* perm_src,
                                double* maxvio, int32_t* max_count, int32_t* d_status,
                                void* cuda_stream);

/*
 * moe_grouped_ffn - grouped expert SwiGLU FFN over expert-contiguous rows ("Mixture of
 * Kittens" digest, Step 1; MoonEP README, "Integration" and "Weight buffer"; "Distributed
 * expert parallelism", "Grouped expert computation").
 *
 * For every expert e and row r in [cu_seqlens[e], cu_seqlens[e+1]):
 *   g = x_perm[r] . W_gate[e],  u = x_perm[r] . W_up[e]     (fp32 accumulate)
 *   h[r] = bf16(silu(g) * u),   silu(z) = z / (1 + exp(-z))
 *   y[r] = bf16(h[r] . W_down[e])                            (fp32 accumulate)
 *
 *   x_perm      [M, H] bf16, e.g. from moe_permute.
 *   w_gate      [E, H, Hp] bf16, w_up [E, H, Hp] bf16, w_down [E, Hp, H] bf16: one contiguous
 *               tensor per projection; expert e is addressed by row index only.
 *   cu_seqlens  device [E+1] int32 as produced by moe_permute (read on the device: the host
 *               never learns the counts). Must be non-decreasing with cu[E] <= M; rows outside
 *               [0, M) are never written.
 *   h_scratch   [M, Hp] bf16 out: the SwiGLU activations (kept: the backward pass needs them).
 *   y           [M, H] bf16 out: expert outputs, row-aligned with x_perm.
 *   Requires H % 128 == 0, Hp % 128 == 0, 1 <= E <= MOE_MAX_FFN_EXPERTS, M < 2^31.
 *   d_status    nullable: MOE_ERR_DEVICE_TIMEOUT is OR-ed in if a pipeline wait in the kernel
 *               exceeded its bound (outputs are then incomplete).
 */
moe_status moe_grouped_ffn(const void* x_perm, const void* w_gate, const void* w_up,
                           const void* w_down, const int32_t* cu_seqlens, int64_t M, int64_t H,
                           int64_t Hp, int32_t E, void* h_scratch, void* y, int32_t* d_status,
                           void* cuda_stream);

/*
 * The two passes of moe_grouped_ffn, callable on their own (same arguments, conventions and
 * requirements; moe_grouped_ffn is exactly moe_grouped_ffn_up_gate then
 * moe_grouped_ffn_down on the same stream):
 *   moe_grouped_ffn_up_gate  h[r] = bf16(silu(x_perm[r] . W_gate[e]) * (x_perm[r] . W_up[e]))
 *   moe_grouped_ffn_down     y[r] = bf16(h[r] . W_down[e])
 */
moe_status moe_grouped_ffn_up_gate(const void* x_perm, const void* w_gate, const void* w_up,
                                   const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                   int32_t E, void* h_scratch, int32_t* d_status,
                                   void* cuda_stream);

moe_status moe_grouped_ffn_down(const void* h_scratch, const void* w_down,
                                const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                int32_t E, void* y, int32_t* d_status, void* cuda_stream);

/*
 * moe_append_shared - routing for a layer with shared experts ("Mixture of Kittens" digest,
 * Step 1: MoE(x) = SharedExpert(x) + sum_k w_k RoutedExpert_k(x)). A shared expert is an
 * expert every token visits with weight 1; appended to the routing it runs in the same
 * moe_permute / moe_grouped_ffn / moe_unpermute_combine launches as the routed experts.
 *   ids_out[t, k] = topk_ids[t, k], w_out[t, k] = route_w[t, k]          for k < K
 *   ids_out[t, K+j] = E + j,        w_out[t, K+j] = 1.0f                 for j < n_shared
 *   topk_ids [S, K] int32, route_w [S, K] fp32 in; ids_out [S, K+n_shared] int32,
 *   w_out [S, K+n_shared] fp32 out (caller-owned, device). The layer then runs with
 *   E + n_shared experts (weights [E+n_shared, ...], the shared ones last) and
 *   K + n_shared slots. A shared expert n times as wide as a routed one is n such experts
 *   holding its column slices (SwiGLU is element-wise over H', so the slices' down
 *   projections add up to the full one). The routed imbalance is moe_maxvio on the first E
 *   counts with the routed K; moe_permute's own maxvio covers all E + n_shared experts.
 * Requires E + n_shared <= MOE_MAX_EXPERTS (<= MOE_MAX_FFN_EXPERTS to run the grouped FFN on
 * the result), S*(K+n_shared) < 2^31.
 */
moe_status moe_append_shared(const int32_t* topk_ids, const float* route_w, int64_t S, int32_t K,
                             int32_t E, int32_t n_shared, int32_t* ids_out, float* w_out,
                             void* cuda_stream);

/*
 * moe_grouped_ffn_gather - moe_grouped_ffn without the permuted copy x_perm: the SwiGLU pass
 * reads each row's token straight from the token-major x (the zero-copy fusion of the MoonEP
 * README, "Zero-copy": experts read the dispatched rows in place). Row r of the
 * expert-grouped order is token perm_src[r] / K, so with perm_src and cu_seqlens from
 * moe_permute (which may then be called with x_perm = NULL) the results h and y equal those
 * of moe_grouped_ffn on the x_perm that moe_permute would have written, bit for bit.
 *   x         [S, H] bf16, token-major (16-byte aligned).
 *   perm_src  device [S*K] int32 from moe_permute; M = S*K rows.
 * Other arguments, requirements and errors as moe_grouped_ffn.
 *
 * moe_grouped_ffn_up_gate_gather is its first pass alone; gate_pre and up_pre (both NULL or
 * both [M, Hp] bf16) also store the pre-activations as moe_grouped_ffn_up_gate_train does.
 */
moe_status moe_grouped_ffn_gather(const void* x, const int32_t* perm_src, int64_t S, int32_t K,
                                  const void* w_gate, const void* w_up, const void* w_down,
                                  const int32_t* cu_seqlens, int64_t H, int64_t Hp, int32_t E,
                                  void* h_scratch, void* y, int32_t* d_status,
                                  void* cuda_stream);

moe_status moe_grouped_ffn_up_gate_gather(const void* x, const int32_t* perm_src, int64_t S,
                                          int32_t K, const void* w_gate, const void* w_up,
                                          const int32_t* cu_seqlens, int64_t H, int64_t Hp,
                                          int32_t E, void* h_scratch, void* gate_pre,
                                          void* up_pre, int32_t* d_status, void* cuda_stream);

/*
 * moe_grouped_ffn_up_gate_train - moe_grouped_ffn_up_gate for training: the same h, plus the
 * pre-activations the backward differentiates SwiGLU at, each rounded once to bf16 from the
 * fp32 accumulator:
 *   gate_pre[r] = bf16(x_perm[r] . W_gate[e]),   up_pre[r] = bf16(x_perm[r] . W_up[e])
 *   gate_pre, up_pre  [M, Hp] bf16 out (caller-owned, 16-byte aligned).
 * Other arguments, requirements and errors as moe_grouped_ffn_up_gate.
 */
moe_status moe_grouped_ffn_up_gate_train(const void* x_perm, const void* w_gate,
                                         const void* w_up, const int32_t* cu_seqlens, int64_t M,
                                         int64_t H, int64_t Hp, int32_t E, void* h_scratch,
                                         void* gate_pre, void* up_pre, int32_t* d_status,
                                         void* cuda_stream);

/*
 * moe_grouped_ffn_backward - backward of the grouped expert FFN: the chain rule of
 * Down(SwiGLU(Up x, Gate x)) ("Mixture of Kittens" digest, Step 1) per expert over the rows
 * cu_seqlens selects, with fp32 weight-gradient buffers laid out like the weights (MoonEP
 * README, "Gradient buffers"). With g = gate_pre[r], u = up_pre[r], s = sigmoid(g):
 *   grad_h       = grad_y[r] . W_down[e]^T                      (fp32, not stored)
 *   d_gate[r]    = bf16(grad_h * u * s * (1 + g * (1 - s)))
 *   d_up[r]      = bf16(grad_h * g * s)
 *   grad_x_perm[r] = bf16(d_gate[r] . W_gate[e]^T + d_up[r] . W_up[e]^T)   (one fp32 sum)
 *   grad_w_gate[e] (+)= sum_r x_perm[r]^T d_gate[r]     [E, H, Hp] fp32
 *   grad_w_up[e]   (+)= sum_r x_perm[r]^T d_up[r]       [E, H, Hp] fp32
 *   grad_w_down[e] (+)= sum_r h[r]^T grad_y[r]          [E, Hp, H] fp32
 * It runs the three calls below on one stream, in this order.
 *   x_perm [M, H], h [M, Hp], gate_pre, up_pre [M, Hp]: bf16 from the training forward.
 *   w_gate, w_up [E, H, Hp], w_down [E, Hp, H]: bf16 weights of the forward.
 *   grad_y [M, H] bf16: gradient of the expert outputs (e.g. from moe_combine_backward).
 *   d_gate, d_up [M, Hp] bf16 out (kept: the weight gradients read them); grad_x_perm [M, H]
 *   bf16 out (e.g. into moe_permute_backward).
 *   accumulate: 0 = the weight gradients are written; 1 = added into the buffers' contents.
 *   An expert without rows gets a zero gradient (left unchanged when accumulating).
 * Requirements, d_status and errors as moe_grouped_ffn; every pointer 16-byte aligned.
 */
moe_status moe_grouped_ffn_backward(const void* x_perm, const void* h, const void* gate_pre,
                                    const void* up_pre, const void* w_gate, const void* w_up,
                                    const void* w_down, const int32_t* cu_seqlens, int64_t M,
                                    int64_t H, int64_t Hp, int32_t E, const void* grad_y,
                                    void* d_gate, void* d_up, void* grad_x_perm,
                                    float* grad_w_gate, float* grad_w_up, float* grad_w_down,
                                    int32_t accumulate, int32_t* d_status, void* cuda_stream);

/*
 * The three passes of moe_grouped_ffn_backward, callable on their own (same arguments and
 * conventions):
 *   moe_grouped_ffn_down_backward     d_gate, d_up from grad_y, W_down, gate_pre, up_pre
 *   moe_grouped_ffn_up_gate_backward  grad_x_perm from d_gate, d_up, W_gate, W_up
 *   moe_grouped_ffn_weight_grad       grad_w_gate, grad_w_up, grad_w_down
 */
moe_status moe_grouped_ffn_down_backward(const void* grad_y, const void* w_down,
                                         const void* gate_pre, const void* up_pre,
                                         const int32_t* cu_seqlens, int64_t M, int64_t H,
                                         int64_t Hp, int32_t E, void* d_gate, void* d_up,
                                         int32_t* d_status, void* cuda_stream);

moe_status moe_grouped_ffn_up_gate_backward(const void* d_gate, const void* d_up,
                                            const void* w_gate, const void* w_up,
                                            const int32_t* cu_seqlens, int64_t M, int64_t H,
                                            int64_t Hp, int32_t E, void* grad_x_perm,
                                            int32_t* d_status, void* cuda_stream);

moe_status moe_grouped_ffn_weight_grad(const void* x_perm, const void* h, const void* d_gate,
                                       const void* d_up, const void* grad_y,
                                       const int32_t* cu_seqlens, int64_t M, int64_t H,
                                       int64_t Hp, int32_t E, float* grad_w_gate,
                                       float* grad_w_up, float* grad_w_down, int32_t accumulate,
                                       int32_t* d_status, void* cuda_stream);

/*
 * moe_unpermute_combine - restore token order, scale by route weight, sum the K results
 * ("Distributed expert parallelism", lifecycle step 8 and "Duplicate route accumulation";
 * MoonEP README, "combine fwd").
 *
 *   out[t] = bf16( sum_{k=0..K-1} route_w[t,k] * float(y[row_id_map[t*K+k]]) )
 *
 * with an fp32 accumulator, k ascending. Slots whose row_id_map entry is negative are
 * skipped.
 *   y          [M, H] bf16, M = S*K.    row_id_map [S*K] int32 (from moe_permute).
 *   route_w    [S, K] fp32.             out [S, H] bf16.
 */
moe_status moe_unpermute_combine(const void* y, const int32_t* row_id_map, const float* route_w,
                                 int64_t S, int64_t H, int32_t K, void* out, void* cuda_stream);

/*
 * moe_combine_backward - backward of moe_unpermute_combine (MoonEP README, "combine bwd":
 * the output gradient is scattered back to the expert-grouped rows by re-dispatching with the
 * saved plan; "Distributed expert parallelism", lifecycle step 8). For every slot f = t*K+k
 * with r = row_id_map[f] >= 0:
 *   grad_y[r]    = bf16(route_w[t,k] * grad_out[t])                 (fp32 product, one rounding)
 *   grad_w[t,k]  = sum_n grad_out[t,n] * y[r,n]                      (fp32, fixed order)
 *   grad_out [S, H] bf16; y [M, H] bf16 (the expert outputs of the forward; may be NULL when
 *   grad_w is NULL); row_id_map [S*K] int32; route_w [S, K] fp32; grad_y [M, H] bf16 out (rows
 *   no slot maps to are not written); grad_w [S, K] fp32 out, nullable.
 */
moe_status moe_combine_backward(const void* grad_out, const void* y, const int32_t* row_id_map,
                                const float* route_w, int64_t S, int64_t H, int32_t K,
                                void* grad_y, float* grad_w, void* cuda_stream);

/*
 * moe_permute_backward - backward of moe_permute's row copy (MoonEP README, "dispatch bwd":
 * each token's K dispatched gradient copies are summed back to token-major, i.e. a combine):
 *   grad_x[t] = bf16( sum_{k ascending} grad_x_perm[row_id_map[t*K+k]] )   (fp32 accumulate)
 *   grad_x_perm [M, H] bf16; row_id_map [S*K] int32; grad_x [S, H] bf16 out.
 */
moe_status moe_permute_backward(const void* grad_x_perm, const int32_t* row_id_map, int64_t S,
                                int64_t H, int32_t K, void* grad_x, void* cuda_stream);

/*
 * moe_maxvio - routing imbalance (MoonEP README, "Performance"):
 *   maxvio = max_e(T_e / T_bar) - 1,  T_e = counts[e],  T_bar = S*K/E,
 * evaluated in IEEE double as ((double)max_count * E) / ((double)S * K) - 1.
 *   counts     device [E] int32.   maxvio device double out.   max_count device int32 out
 *   (nullable). S*K must be > 0.
 */
moe_status moe_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                      int32_t* max_count, void* cuda_stream);

/*
 * MXFP8 expert FFN ("Mixture of Kittens" digest, Step 8: the expert GEMMs run in MXFP8). The
 * format is that of the OCP Microscaling Formats v1.0: blocks of 32 consecutive elements along
 * the reduction dimension share one E8M0 scale 2^s, s = floor(log2(amax of the block)) - 8
 * (at least -127; s = -127 for an all-zero block), stored as the byte s + 127; each element is
 * v / 2^s rounded to FP8 E4M3, nearest-even, magnitudes above 448 saturating to 448.
 *
 * moe_mx_quantize_weights - quantise one projection's weights once, ahead of the layer:
 *   w     [E, R, C] bf16, device, C contiguous, R the reduction dimension (R = H, C = H' for
 *         W_gate and W_up; R = H', C = H for W_down).
 *   w_q   [E, R, C] uint8 out: E4M3 codes, same layout as w.
 *   w_sf  uint8 out, moe_mx_weight_scale_bytes(E, R, C) = E*R*C/32 bytes: the scale of rows
 *         32b..32b+31 of column c of expert e is the byte
 *           ((e*(C/128) + c/128)*(R/128) + b/4)*512 + (c%128 % 32)*16 + (c%128 / 32)*4 + b%4,
 *         i.e. one 512-byte chunk per 128 columns x 128 rows, in the order the block-scaled
 *         tensor-core MMA takes its scales.
 *   Requires R % 128 == 0, C % 128 == 0; w, w_q, w_sf 16-byte aligned; caller-owned buffers.
 */
size_t moe_mx_weight_scale_bytes(int32_t E, int64_t R, int64_t C);

moe_status moe_mx_quantize_weights(const void* w, int32_t E, int64_t R, int64_t C, void* w_q,
                                   void* w_sf, void* cuda_stream);

/*
 * moe_mx_permute_quantize - moe_permute's row copy fused with the activations' quantisation:
 * each token row of x is quantised once (blocks of 32 along H) and its codes and scales are
 * written to the K rows row_id_map[t*K+k] of the expert-grouped order (rows of -1 skipped):
 *   x      [S, H] bf16 in.   row_id_map [S*K] int32 from moe_permute (which may be called with
 *   x_perm = NULL to produce the routing only).
 *   x_q    [S*K, H] uint8 out (E4M3);  x_sf [S*K, H/32] uint8 out (E8M0, row-major).
 *   Requires H % 128 == 0; x, x_q, x_sf 16-byte aligned. Launched as a dependent of the
 *   preceding kernel on the stream (programmatic dependent launch).
 */
moe_status moe_mx_permute_quantize(const void* x, const int32_t* row_id_map, int64_t S, int64_t H,
                                   int32_t K, void* x_q, void* x_sf, void* cuda_stream);

/*
 * moe_grouped_ffn_mxfp8 - moe_grouped_ffn in MXFP8 on block-scaled tcgen05 MMAs (fp32
 * accumulation):
 *   h[r] = silu(x[r] . Wg[e]) * (x[r] . Wu[e])   with x, Wg, Wu the dequantised MXFP8 values,
 *          stored quantised to MXFP8 along H' (h_q [M, Hp] uint8, h_sf [M, Hp/32] uint8) --
 *          the quantisation runs in the SwiGLU epilogue on the fp32 values;
 *   y[r] = bf16(h[r] . Wd[e])                   (dequantised h_q and W_down).
 *   x_q, x_sf  [M, H], [M, H/32] from moe_mx_permute_quantize.
 *   *_q, *_sf  weights from moe_mx_quantize_weights (W_gate, W_up: R = H, C = Hp; W_down:
 *              R = Hp, C = H).
 *   cu_seqlens, M, H, Hp, E, d_status and the requirements as moe_grouped_ffn; y [M, H] bf16.
 *
 * moe_grouped_ffn_up_gate_mxfp8 and moe_grouped_ffn_down_mxfp8 are its two passes alone.
 */
moe_status moe_grouped_ffn_mxfp8(const void* x_q, const void* x_sf, const void* w_gate_q,
                                 const void* w_gate_sf, const void* w_up_q, const void* w_up_sf,
                                 const void* w_down_q, const void* w_down_sf,
                                 const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                 int32_t E, void* h_q, void* h_sf, void* y, int32_t* d_status,
                                 void* cuda_stream);

moe_status moe_grouped_ffn_up_gate_mxfp8(const void* x_q, const void* x_sf, const void* w_gate_q,
                                         const void* w_gate_sf, const void* w_up_q,
                                         const void* w_up_sf, const int32_t* cu_seqlens, int64_t M,
                                         int64_t H, int64_t Hp, int32_t E, void* h_q, void* h_sf,
                                         int32_t* d_status, void* cuda_stream);

moe_status moe_grouped_ffn_down_mxfp8(const void* h_q, const void* h_sf, const void* w_down_q,
                                      const void* w_down_sf, const int32_t* cu_seqlens, int64_t M,
                                      int64_t H, int64_t Hp, int32_t E, void* y, int32_t* d_status,
                                      void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
