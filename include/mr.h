/*
 * mr.h -- C ABI of libmr.so: the MoE routing hot path on NVIDIA B200 (sm_100a).
 *
 * The path, as the pages define it:
 *
 *   router    logits L = x . W^T in fp32, scores s = sigmoid(L), selection
 *             scores c = s + bias, grouped selection (group score = sum of
 *             the two largest c of the group, keep topk_group groups, mask
 *             the rest), token top-k, weights = route_scale * s / (sum s +
 *             1e-20) over the chosen experts.
 *             (Kimi K2 "Normalize weights" page: formula G_i and the
 *             MoEGate.forward excerpt; DeepSeek-V3.2-Exp "Normalize weights"
 *             page: Gate.forward excerpt; DeepSeek-V3 "MoE Router" note:
 *             affinity equation, bias, grouped routing, route_scale.)
 *   dispatch  per-expert counts, expert offsets and the expert-sorted
 *             permutation idxs = argsort(topk_idx.view(-1)) (stable).
 *   gather    sorted_tokens = x[idxs // k].
 *   combine   new_x[idxs] = expert outputs; y = sum_k w * new_x cast back to
 *             the row dtype; y + shared-expert output.
 *             (Kimi K2 "Add shared output" page: DeepseekV3MoE.forward and
 *             moe_infer excerpts, formula Delta_ffn = y_routed + y_shared.)
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are caller-owned DEVICE pointers on the current
 *    device, row-major and densely packed.  The library never allocates
 *    device memory, frees or synchronises (except mr_get_error, which must
 *    read the device, and the mr_ipc_* calls, which map and unmap buffers of
 *    other processes); its only device memory is a few fixed arrays in its
 *    own image, named below where they are used.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy stream) and
 *    runs asynchronously.  Arguments are validated on the host before any
 *    launch; an invalid call launches nothing and returns a negative status.
 *  - Index tensors are int32 (T*k < 2^31 is required and checked).
 *  - T == 0 is valid and launches nothing.
 *  - Device-side faults in the data (an expert id out of [0, N_r)) do not
 *    trap: the kernel skips the entry and raises the sticky device flag that
 *    mr_get_error() reports and clears.
 *  - No exceptions cross the ABI.  Calls on different streams are
 *    independent, except for the per-device state named where it is used:
 *    the error flag, the split-K array of mr_router_forward (ordered across
 *    streams by the library) and the scratch array of mr_dispatch_noalloc
 *    (ordered by the caller).
 */
#ifndef MR_H
#define MR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA runtime headers. */
typedef struct CUstream_st *mr_stream_t;

/* ---- status codes ------------------------------------------------------ */
#define MR_OK 0
#define MR_ERR_INVALID_ARG (-1) /* bad size, null pointer, inconsistent args  */
#define MR_ERR_UNSUPPORTED (-2) /* valid but outside what the kernels support */
#define MR_ERR_CUDA (-3)        /* a CUDA launch or query failed              */
#define MR_ERR_DEVICE (-4)      /* device flag: bad expert id seen            */
#define MR_ERR_TIMEOUT (-5)     /* device flag: a bounded wait gave up        */
#define MR_ERR_OVERFLOW (-6)    /* device flag: rows past a buffer's capacity */

/* ---- element types of row tensors --------------------------------------- */
#define MR_F32 0
#define MR_BF16 1

/* ---- mask value for the experts of dropped groups ------------------------
 * MR_MASK_NEG_INF: -inf (DeepSeek-V3.2-Exp Gate.forward, masked_fill_ -inf);
 * MR_MASK_ZERO:    0.0  (Kimi K2 / HF MoEGate.forward, masked_fill 0.0).   */
#define MR_MASK_NEG_INF 0
#define MR_MASK_ZERO 1

/* ---- router arithmetic ----------------------------------------------------
 * MR_PREC_3XTF32: tensor cores (tcgen05, kind::tf32), each fp32 operand split
 *                 into a tf32 high part and a residual; hi*hi + hi*lo + lo*hi
 *                 accumulate in fp32 (fp32-level accuracy).
 * MR_PREC_TF32:   tensor cores, one tf32 product (about 1e-3 relative).
 * MR_PREC_FFMA:   CUDA-core fp32 FMA (any shape; slowest).
 * MR_PREC_BF16X3: for bf16 activations (x_dtype MR_BF16): W is split once
 *                 per call into three bf16 planes W1 + W2 + W3 (equal to W
 *                 within 2^-24 relative), and x*W1 + x*W2 + x*W3 run as
 *                 bf16 tensor-core products, each exact in fp32, with fp32
 *                 accumulation: fp32-level accuracy at half the tensor time
 *                 and half the activation bytes of 3xTF32.                  */
#define MR_PREC_3XTF32 0
#define MR_PREC_TF32 1
#define MR_PREC_FFMA 2
#define MR_PREC_BF16X3 3

/* ---- scoring variants (flags of mr_router_forward_ex2) --------------------
 * From the DeepSeek-V3.2-Exp "Normalize weights" page (Gate.forward):
 * MR_SCORE_SOFTMAX  s = softmax(L) over all N_r experts instead of sigmoid;
 *                   the chosen experts' weights are route_scale * s, not
 *                   renormalised.
 * MR_GROUP_MAX      group score = the group's largest biased score (the
 *                   page's choice when there is no bias) instead of the sum
 *                   of its two largest.
 * MR_NORM_NO_EPS    renormalise by the plain sum of the k scores (the page)
 *                   instead of sum + 1e-20 (Kimi K2 MoEGate.forward); the two
 *                   differ only when every chosen score underflows.
 * The page's gate is MR_NORM_NO_EPS, plus MR_GROUP_MAX when there is no bias,
 * plus MR_SCORE_SOFTMAX for score_func "softmax".  0 is the Kimi K2 /
 * DeepSeek-V3 gate of mr_router_forward.                                    */
#define MR_SCORE_SOFTMAX 1
#define MR_GROUP_MAX 2
#define MR_NORM_NO_EPS 4

/* Library version, major*10000 + minor*100 + patch. */
int mr_version(void);

/* Static English text for a status code. */
const char *mr_status_string(int status);

/*
 * mr_router_forward -- gate forward for T tokens.
 *
 * Computes, per token t, the k chosen experts and their weights exactly as
 * the pages define them (see the file header).  Ties between equal selection
 * scores (groups or experts) go to the lower index.  The k slots of a token
 * are ordered by masked selection score descending, index ascending.
 * When n_group == 1 the group step is skipped (it keeps every expert).
 * A NULL bias means b = 0; the group score is still the top-2 sum.
 *
 *   x        [T, d] fp32 token rows (the fp32 cast of the hidden states).
 *   W        [N_r, d] fp32 gate weight (nn.Linear layout, no Linear bias).
 *   bias     [N_r] fp32 selection bias, or NULL.
 *   n_group  groups; N_r % n_group == 0; group size >= 2 when n_group > 1.
 *   topk_group  groups kept, 1 <= topk_group <= n_group.
 *   k        experts per token, 1 <= k <= 8; with MR_MASK_NEG_INF and
 *            n_group > 1 also k <= topk_group * (N_r / n_group).
 *   route_scale  multiplier applied after renormalisation.
 *   mask_mode    MR_MASK_NEG_INF or MR_MASK_ZERO.
 *   idx_out  [T, k] int32 expert ids (written).
 *   w_out    [T, k] fp32 weights (written).
 *
 * Limits: 1 <= N_r <= 512, n_group <= 32, d >= 1.  Uses 3xTF32 tensor-core
 * arithmetic when d % 4 == 0 and N_r % 16 == 0 (N_r % 32 == 0 above 256),
 * CUDA-core FMA otherwise.  The environment variable MR_TC_CLUSTER=1, 2 or
 * P pins how CTAs share the work of a 128-token tile (testing only): one CTA
 * with all experts, two CTAs splitting the experts, or (bf16x3) two CTAs
 * running one 256-token tensor-core MMA.
 *
 * The kernels are picked by T, with no workspace argument:
 *  - T > 256: one fused kernel (GEMM + routing in its epilogue; the logits
 *    never leave the SM).
 *  - T <= 256 (decode): the split-K path -- a K-sliced GEMM over all SMs
 *    whose slices are summed in clusters, then a reduce-and-route kernel (two
 *    launches) -- when its partial logits fit the library's fixed array of
 *    mr_router_forward_max_scratch() bytes (2 MiB; e.g. every T <= 256 at
 *    d = 7168, N_r = 256); otherwise the fused kernel.  That array is part of
 *    libmr.so's device image: every GPU that loads the library holds one copy
 *    until the process exits, and this entry point allocates nothing.  All
 *    calls on a device share it; the library orders them across streams (each
 *    use waits on the previous use's event and records its own), except while
 *    `stream` is being captured into a CUDA graph, where it adds no
 *    dependency: the caller then orders the graph's launches against other
 *    small-batch calls of this entry point on that device.  The first call on
 *    a device looks up the array's address and creates the event.
 * The results are the same 3xTF32 arithmetic on either path, summed in a
 * fixed order (deterministic).
 * Returns MR_OK or a negative status (nothing launched on an argument error).
 */
int mr_router_forward(const float *x, const float *W, const float *bias, int T,
                      int d, int N_r, int n_group, int topk_group, int k,
                      float route_scale, int mask_mode, int32_t *idx_out,
                      float *w_out, mr_stream_t stream);

/* Size in bytes of the fixed array mr_router_forward keeps its split-K
 * partial logits in (no counterpart on the pages). */
size_t mr_router_forward_max_scratch(void);

/*
 * mr_router_workspace_size -- bytes of device workspace that
 * mr_router_forward_ex may use for T tokens on the current device: the
 * largest of W's three bf16 planes (3 * N_r * d * 2 bytes, bf16 activations),
 * W's tf32 residuals (N_r * d * 4 bytes, fp32 activations; both computed once
 * per call so the fused kernel's CTAs do not each re-derive them) and, for
 * T <= 256, the split-K partial logits of the small-batch path (about
 * (number of SMs / ceil(N_r/128)) * T * N_r * 4 bytes).
 */
size_t mr_router_workspace_size(int T, int d, int N_r);

/*
 * mr_router_forward_ex -- mr_router_forward with explicit options.
 *
 *   x_dtype     MR_F32 ([T,d] fp32) or MR_BF16 ([T,d] bf16 hidden states,
 *               whose fp32 cast is exact).
 *   precision   MR_PREC_3XTF32, MR_PREC_TF32, MR_PREC_FFMA or MR_PREC_BF16X3.
 *               With MR_BF16 activations the tensor-core precisions (3XTF32
 *               or BF16X3) both run the bf16x3 decomposition, which needs a
 *               workspace of mr_router_workspace_size bytes (W's planes);
 *               MR_PREC_FFMA computes the fp32 cast on CUDA cores.
 *   logits_out  [T, N_r] fp32 logits, or NULL (debug / verification only).
 *   workspace   device buffer of workspace_bytes, or NULL.  With at least
 *               mr_router_workspace_size(T, d, N_r) bytes, batches of up to
 *               256 tokens on the tensor-core precisions use the split-K path
 *               for fp32 and bf16 rows alike (two launches: a K-sliced 3xTF32
 *               GEMM over all SMs whose slices are summed in clusters, then a
 *               reduce-and-route kernel); the result is the same arithmetic,
 *               summed in a fixed order (deterministic).
 *               Larger batches use it for W's tf32 residuals (one extra
 *               launch); results are identical with or without it.
 * Returns MR_ERR_UNSUPPORTED when the requested precision cannot run this
 * shape (tensor-core paths need d % 4 == 0 and N_r % 16 == 0, or
 * N_r % 32 == 0 when N_r > 256).
 */
int mr_router_forward_ex(const void *x, int x_dtype, const float *W,
                         const float *bias, int T, int d, int N_r, int n_group,
                         int topk_group, int k, float route_scale,
                         int mask_mode, int precision, int32_t *idx_out,
                         float *w_out, float *logits_out, void *workspace,
                         size_t workspace_bytes, mr_stream_t stream);

/*
 * mr_router_forward_ex2 -- mr_router_forward_ex with the scoring variants of
 * the DeepSeek-V3.2-Exp "Normalize weights" page (Gate.forward): `flags` is
 * a combination of MR_SCORE_SOFTMAX, MR_GROUP_MAX and MR_NORM_NO_EPS (0 gives
 * mr_router_forward_ex).  Every path (fused tensor-core, split-K, CUDA-core)
 * supports every combination; other bits give MR_ERR_INVALID_ARG.
 */
int mr_router_forward_ex2(const void *x, int x_dtype, const float *W,
                          const float *bias, int T, int d, int N_r, int n_group,
                          int topk_group, int k, float route_scale,
                          int mask_mode, int precision, int flags,
                          int32_t *idx_out, float *w_out, float *logits_out,
                          void *workspace, size_t workspace_bytes,
                          mr_stream_t stream);

/*
 * mr_router_forward_bf16w -- the gate with its weight stored in bf16.
 *
 * The Kimi K2 "Normalize weights" page's MoEGate.forward casts the stored
 * gate weight to fp32 at use (self.weight.type(torch.float32) inside
 * F.linear): the weight may be kept in a narrower type and the logits are
 * still fp32 dot products.  Here W is kept in bf16 -- half the bytes of the
 * decode-time weight read -- and the method is otherwise that of
 * mr_router_forward_ex2 on the widened (exact) fp32 values of W.
 *
 *   x          [T, d] rows: MR_BF16 (tensor cores) or MR_F32 (CUDA cores).
 *   W_bf16     [N_r, d] bf16 gate weight (bit patterns, nn.Linear layout).
 *   flags      as mr_router_forward_ex2.
 *   workspace  optional, mr_router_workspace_size(T, d, N_r) bytes: with it,
 *              or with NULL and the batch's partials within
 *              mr_router_forward_max_scratch() (the array mr_router_forward
 *              uses, shared and ordered the same way), batches of up to 256
 *              bf16 rows take the split-K path (two launches); larger batches
 *              take the fused kernel (one launch, no workspace).
 * Arithmetic: bf16 rows x bf16 W on the tensor cores (tcgen05 kind::f16, one
 * product per multiply-add, each exact in fp32, fp32 accumulation): the fp32
 * logits of the widened operands up to summation order, so the tolerances of
 * the fp32 path hold against the oracle fed the widened W.  fp32 rows, or
 * shapes the tensor-core kernels do not take (d % 8, N_r % 16 or, above 256,
 * N_r % 32 nonzero): CUDA-core FMA on the widened W.
 * Limits and errors as mr_router_forward_ex2.
 */
int mr_router_forward_bf16w(const void *x, int x_dtype, const void *W_bf16,
                            const float *bias, int T, int d, int N_r,
                            int n_group, int topk_group, int k,
                            float route_scale, int mask_mode, int flags,
                            int32_t *idx_out, float *w_out, float *logits_out,
                            void *workspace, size_t workspace_bytes,
                            mr_stream_t stream);

/*
 * mr_dispatch_workspace_size -- bytes of device workspace mr_dispatch needs:
 * 16 + ceil(T*k / 1024) * N_r * 4 + N_r * 4 (a barrier word, per-chunk
 * expert histograms, expert totals).
 */
size_t mr_dispatch_workspace_size(int T, int k, int N_r);

/*
 * mr_dispatch -- moe_infer's dispatch bookkeeping (Kimi K2 "Add shared
 * output" page, moe_infer: cnts.scatter_ / tokens_per_expert, idxs =
 * topk_ids.view(-1).argsort(), the running start_idx/end_idx of the expert
 * loop, and the inverse used by new_x[idxs] = outs).
 *
 *   idx       [T, k] int32 expert ids in [0, N_r).
 *   counts    [N_r] int32: counts[e] = #{(t, j) : idx[t, j] == e}.
 *   offsets   [N_r + 1] int32: exclusive prefix sum of counts.
 *   perm      [T*k] int32: perm[i] = flat slot t*k + j of the i-th entry in
 *             expert order; within an expert, ascending slot (stable), so
 *             the token of sorted row i is perm[i] / k.
 *   inv_perm  [T*k] int32 or NULL: inv_perm[perm[i]] = i.
 *   workspace at least mr_dispatch_workspace_size(T, k, N_r) bytes; its
 *             contents need no initialisation.
 * One cooperative kernel (histogram, per-expert chunk prefix, offsets and
 * stable scatter, separated by two grid barriers whose waits are bounded)
 * preceded by a 4-byte memset of the barrier word, when one CTA per
 * 1024-entry chunk fits on the device at once; three kernels otherwise.
 * Calls on different streams need different workspaces.
 * Limits: 1 <= N_r <= 1024, 1 <= k <= 32.
 * An id outside [0, N_r) is dropped: counts/offsets/perm cover the valid
 * entries only, perm[offsets[N_r] ..] and the dropped slots' inv_perm are -1,
 * and the device flag reports MR_ERR_DEVICE.
 */
int mr_dispatch(const int32_t *idx, int T, int k, int N_r, int32_t *counts,
                int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                void *workspace, size_t workspace_bytes, mr_stream_t stream);

/*
 * mr_dispatch_noalloc -- mr_dispatch for callers that cannot allocate device
 * memory when they dispatch.  The pages have no counterpart to this entry
 * point; it exists for the runtime around the path, not for the method.
 *
 * Some callers hold a stream and their input/output tensors but may not call
 * cudaMalloc (or any allocating routine) at that point: a serving loop whose
 * device memory is planned before requests start and treats an allocation
 * mid-request as an error (cudaMalloc can synchronise the device and fragment
 * a planned pool), or a plug-in running inside another framework's runtime,
 * which owns all device memory and hands the plug-in only tensors and a
 * stream.  Such a caller cannot provide mr_dispatch's workspace.  This entry
 * point takes the same inputs and outputs as mr_dispatch and computes the
 * same results, with the workspace taken from a fixed array compiled into
 * libmr.so instead.
 *
 * Limits: everything mr_dispatch allows, and additionally
 * ceil(T*k / 1024) * N_r * 4 <= mr_dispatch_noalloc_max_workspace()
 * (1 MiB: ceil(T*k / 1024) * N_r <= 262144, e.g. T*k up to 1,048,576 entries
 * at N_r = 256).  Larger sizes return MR_ERR_UNSUPPORTED before any launch;
 * use mr_dispatch with a workspace for them.  (It runs the three-kernel
 * counting sort.)
 *
 * The fixed array: every GPU that loads libmr.so holds one 1 MiB copy until
 * the process exits.  The first call on a device looks up the array's device
 * address with that device current (cudaGetSymbolAddress) and keeps it; a
 * lookup that fails returns MR_ERR_CUDA and is tried again by the next call.
 * The entry point itself calls no cudaMalloc, cudaFree or other allocating
 * routine.  All calls on a
 * device share the one array, and it keeps whatever the last call left in
 * it: nothing in it needs to start at zero (each call rewrites every entry it
 * later reads), but calls that may overlap on the GPU -- on different streams
 * without ordering between them -- race on it and must be serialised by the
 * caller.
 */
int mr_dispatch_noalloc(const int32_t *idx, int T, int k, int N_r,
                        int32_t *counts, int32_t *offsets, int32_t *perm,
                        int32_t *inv_perm, mr_stream_t stream);

/* Size in bytes of the fixed scratch array mr_dispatch_noalloc uses. */
size_t mr_dispatch_noalloc_max_workspace(void);

/*
 * mr_ep_recv_order -- receive-side order of the expert-parallel exchange
 * (Kimi K2 "Add shared output" page, moe_infer, ep_size > 1: the labels
 * gatherd_idxs of the received rows, their argsort, and
 * tokens_per_expert_post_gather).
 *
 * With ep ranks, rank r owns experts [r*E_loc, (r+1)*E_loc).  After the row
 * all-to-all it holds R rows, source by source, each source's rows in that
 * source's expert-sorted order.
 *   recv_counts    [ep, E_loc] int32 (device): recv_counts[s][e] = rows from
 *                  source s for local expert e (the all_to_all_single of
 *                  tokens_per_expert).
 *   R              the sum of recv_counts (the rows received).
 *   order          [R] int32: order[j] = the received row that goes j-th when
 *                  the rows are sorted by local expert (stable: by source,
 *                  then the source's order) -- sorted = received[order],
 *                  e.g. mr_gather_rows(received, k = 1, perm = order).
 *   inv_order      [R] int32 or NULL: inv_order[order[j]] = j -- the
 *                  scatter-back new_x[gatherd_idxs] = outs is
 *                  mr_gather_rows(outs, k = 1, inv_perm = order).
 *   local_counts   [E_loc] int32: rows per local expert.
 *   local_offsets  [E_loc + 1] int32: their exclusive prefix.
 * One kernel, no sort (the stable order has a closed form per segment).
 * Limits: ep * E_loc <= 1024.  A negative count or a sum other than R writes
 * nothing and raises the device flag (MR_ERR_DEVICE from mr_get_error).
 */
int mr_ep_recv_order(const int32_t *recv_counts, int ep, int E_loc, int R,
                     int32_t *order, int32_t *inv_order, int32_t *local_counts,
                     int32_t *local_offsets, mr_stream_t stream);

/*
 * Expert parallelism over peer memory (Kimi K2 "Add shared output" page,
 * moe_infer, ep_size > 1), without the two row all-to-alls and the
 * receive-side sort: every source writes each of its rows straight into the
 * owner's receive buffer at the row's final place, and the combine reads the
 * expert outputs straight out of the owners' output buffers.  Rank r owns
 * experts [r*E_loc, (r+1)*E_loc), E_loc = N_r / ep.  Owner o's receive
 * buffer holds, in order: its local experts; within an expert, the sources in
 * rank order; within a source, that source's rows in its own stable expert
 * order (token order) -- exactly the rows and the order the page's
 * all-to-all followed by the stable argsort of the received expert labels
 * produces.  The place of every row follows from all ranks' counts alone.
 *
 * The buffers are device pointers of this process: this GPU's own memory,
 * another GPU's memory with peer access enabled, or another process's buffer
 * opened with mr_ipc_import.  The caller orders the ranks' steps: every
 * rank's mr_ep_dispatch_p2p finished before any owner reads its receive
 * buffer, every owner's outputs complete before any mr_ep_combine_p2p reads
 * them, and every combine finished before an owner overwrites its output
 * buffer (e.g. a collective on the stream between the steps).  The kernels
 * never wait on another rank.
 */

/*
 * mr_ep_dispatch_p2p -- rows of this rank to their owners' receive buffers.
 *
 *   x             [T, d] token rows of `dtype` (MR_BF16 or MR_F32).
 *   idx           [T, k] int32 expert ids in [0, N_r).
 *   inv_perm, offsets   this rank's mr_dispatch of idx (inv_perm [T*k],
 *                 offsets [N_r + 1]).
 *   counts_all    [ep, N_r] int32 (device): every rank's counts from
 *                 mr_dispatch, rank-major (an all-gather of them).
 *   rank, ep      this rank and the number of ranks (N_r % ep == 0).
 *   recv_bufs     HOST array of ep device pointers: rank o's receive buffer,
 *                 [capacity, d] of `dtype`, 16-byte aligned for the vector
 *                 path.
 *   dest          [T*k] int32 out: the row of slot t*k+j in its owner's
 *                 buffer, -1 for a slot without one.
 *   local_counts  [E_loc] int32 out: rows this rank receives per local
 *                 expert; local_offsets [E_loc + 1] their exclusive prefix
 *                 (the segments of its own receive buffer, for its experts).
 * Two kernels: the destinations (every CTA rebuilds the per-expert bases
 * from counts_all in shared memory), then one CTA per token reads its row
 * once and stores it to its k destinations.
 * Limits: 1 <= k <= 32, ep <= 64, N_r <= 1024.  Data faults do not trap: ids
 * out of range and slots dropped by mr_dispatch get dest -1; counts below
 * zero, or a row of counts_all for `rank` that disagrees with offsets, set
 * every dest to -1 and the local counts to 0 (MR_ERR_DEVICE from
 * mr_get_error); rows past an owner's capacity are not written, get dest -1
 * and are not counted in local_counts (MR_ERR_OVERFLOW).  A capacity of
 * ep * T_max * min(k, E_loc) rows never overflows.
 */
int mr_ep_dispatch_p2p(const void *x, int dtype, int T, int d, int k,
                       const int32_t *idx, const int32_t *inv_perm,
                       const int32_t *offsets, const int32_t *counts_all,
                       int ep, int rank, int N_r, void *const *recv_bufs,
                       int capacity, int32_t *dest, int32_t *local_counts,
                       int32_t *local_offsets, mr_stream_t stream);

/*
 * mr_ep_combine_p2p -- the weighted combine and shared add of mr_combine,
 * reading slot (t, j)'s expert output from row dest[t*k+j] of the output
 * buffer of idx[t, j]'s owner.
 *
 *   out_bufs  HOST array of ep device pointers: rank o's expert outputs,
 *             [capacity, d] of `dtype`, row i the output of its receive row i.
 *   idx, dest [T*k] from this rank's mr_ep_dispatch_p2p.
 *   w, shared, y, and the arithmetic: as mr_combine (slots without a row
 *             contribute nothing).
 * One kernel; the peers' rows are loaded through L2, not the read-only path.
 * Limits: 1 <= k <= 32, ep <= 64.
 */
int mr_ep_combine_p2p(const void *const *out_bufs, int dtype, int d,
                      const float *w, const int32_t *idx, const int32_t *dest,
                      int ep, int N_r, int capacity, const void *shared,
                      void *y, int T, int k, mr_stream_t stream);

/*
 * Buffers shared between processes (one process per GPU): an owner exports
 * its receive and output buffers, every rank imports the others'.
 *   mr_ipc_export  fills *out for `bytes` of device memory at dev_ptr, which
 *                  must lie inside one allocation of the runtime allocator
 *                  (cudaMalloc, as under PyTorch's caching allocator):
 *                  MR_ERR_INVALID_ARG otherwise, MR_ERR_UNSUPPORTED for memory
 *                  the IPC handles cannot name (the virtual memory API).
 *   mr_ipc_import  opens a handle exported by ANOTHER process, on the current
 *                  device, with peer access enabled on demand; *ptr is the
 *                  buffer, *base the mapping to pass to mr_ipc_close.
 *   mr_ipc_close   unmaps *base.
 * The handle is plain bytes: send it through any channel (e.g. an
 * all-gather of the processes' handles).
 */
typedef struct mr_ipc_handle {
  unsigned char handle[64]; /* CUDA IPC handle of the allocation */
  uint64_t offset;          /* buffer start within the allocation */
  uint64_t bytes;           /* buffer size */
} mr_ipc_handle_t;

int mr_ipc_export(const void *dev_ptr, size_t bytes, mr_ipc_handle_t *out);
int mr_ipc_import(const mr_ipc_handle_t *h, void **base, void **ptr);
int mr_ipc_close(void *base);

/*
 * mr_expert_gemm_gather -- one expert layer over the expert-sorted rows, with
 * the row gather fused into the GEMM (Kimi K2 "Add shared output" page,
 * moe_infer: sorted_tokens = x[idxs // k], then
 * expert(sorted_tokens[start_idx:end_idx]) for each expert).
 *
 * The expert is one linear map per expert with caller-supplied (synthetic)
 * weights; the sorted row j belongs to expert e(j), the e with
 * offsets[e] <= j < offsets[e + 1], and
 *     out[j][n] = sum_c x[perm[j] / k][c] * W_exp[e(j)][n][c].
 * The gathered rows are never written: each 128-row block of an expert's
 * segment is loaded from x by tensor-memory-access gathers (four rows per
 * copy, the rows taken from perm).  bf16 operands, each product exact, fp32
 * accumulation in tensor memory, rounded to bf16 (nearest even) on output.
 *
 *   x        [T, d] bf16 token rows.
 *   perm     [T*k] int32, offsets [N_r + 1] int32: from mr_dispatch.  perm
 *            may be NULL: x is then [T*k, d], the rows already in
 *            expert-sorted order (row j = sorted row j; e.g. from
 *            mr_gather_rows), and the call is the plain grouped GEMM (one
 *            tiled copy per 128-row block instead of the gathers).
 *   W_exp    [N_r, n_out, d] bf16 (nn.Linear layout per expert).
 *   out      [T*k, n_out] bf16 in expert-sorted order; rows from offsets[N_r]
 *            on (dropped ids) are not written.
 * Limits: d % 8 == 0, n_out % 16 == 0, N_r <= 1024, 16-byte aligned x, W_exp
 * and out (else MR_ERR_UNSUPPORTED).  One kernel; no workspace.
 */
int mr_expert_gemm_gather(const void *x, const int32_t *perm,
                          const int32_t *offsets, const void *W_exp, int T,
                          int d, int k, int N_r, int n_out, void *out,
                          mr_stream_t stream);

/*
 * mr_expert_packed_bytes / mr_expert_pack_weights /
 * mr_expert_gemm_gather_packed -- the same expert layer with its weights
 * re-laid once (at weight-load time) so each tile the GEMM stages is one
 * contiguous block: W_exp [N_r, n_out, d] is cut into tiles of 256 output
 * rows x 64 K columns, tile (e, nt, kc) stored as a [256][64] bf16 block at
 * block index (e * ceil(n_out/256) + nt) * ceil(d/64) + kc, zero-padded past
 * n_out and d, each 128-byte row's 16-byte chunks permuted into the
 * 128-byte-swizzled order the tensor core reads (chunk c of row r at
 * position c ^ (r % 8)), so one bulk copy stages a tile.  The pages have no
 * counterpart (a storage layout, not a step of the method); results are
 * bit-identical to mr_expert_gemm_gather.
 * mr_expert_pack_weights writes mr_expert_packed_bytes(N_r, n_out, d) bytes
 * (caller-owned, 16-byte aligned; d % 8 == 0).
 */
size_t mr_expert_packed_bytes(int N_r, int n_out, int d);
int mr_expert_pack_weights(const void *W_exp, int N_r, int n_out, int d,
                           void *W_packed, size_t packed_bytes,
                           mr_stream_t stream);
int mr_expert_gemm_gather_packed(const void *x, const int32_t *perm,
                                 const int32_t *offsets, const void *W_packed,
                                 int T, int d, int k, int N_r, int n_out,
                                 void *out, mr_stream_t stream);

/*
 * mr_expert_gemm_gather_combine -- the expert layer of mr_expert_gemm_gather
 * with the weighted combine fused into its epilogue (Kimi K2 "Add shared
 * output" page, moe_infer: outs = expert(sorted rows), new_x[idxs] = outs,
 * new_x.view(T, k, d) cast to the weights' dtype, multiplied by topk_weight
 * and summed over k, cast back, then y + shared_experts(identity)): neither
 * the gathered rows nor the expert outputs are written to memory.
 *
 *   x, perm, offsets, T, d, k, N_r, n_out   as mr_expert_gemm_gather (perm
 *            required: it gives each sorted row's slot perm[j] = t*k + j').
 *   W        the expert weights: [N_r, n_out, d] bf16 (nn.Linear layout)
 *            when w_packed == 0, the layout of mr_expert_pack_weights when
 *            w_packed == 1.
 *   w        [T, k] fp32 router weights (row j is scaled by w[perm[j]]).
 *   shared   [T, n_out] bf16 shared-expert output, or NULL.
 *   acc      [T, n_out] fp32 scratch, caller-owned and 16-byte aligned; the
 *            call zeroes it and leaves the fp32 routed sums in it.
 *   y        [T, n_out] bf16 output, 16-byte aligned.
 * Per element: out_j = bf16(x[perm[j]/k] . W[e(j)]^T) (as
 * mr_expert_gemm_gather); acc[t] = sum over the token's routed slots of the
 * fp32 products w_j * out_j, added with fp32 atomic reductions, so the order
 * of the k terms is not fixed and acc can differ in its last bits from run to
 * run; y = bf16(bf16(acc) + shared) (bf16(acc) without shared), both
 * roundings to nearest even.  A token with no routed slot gets y = shared
 * (or 0).  Three launches on `stream`: a memset of acc, the GEMM, the
 * finalize.  Limits as mr_expert_gemm_gather; n_out % 16 == 0, shared 16-byte
 * aligned (else MR_ERR_UNSUPPORTED).
 */
int mr_expert_gemm_gather_combine(const void *x, const int32_t *perm,
                                  const int32_t *offsets, const void *W,
                                  int w_packed, const float *w,
                                  const void *shared, int T, int d, int k,
                                  int N_r, int n_out, float *acc, void *y,
                                  mr_stream_t stream);

/*
 * mr_gather_rows -- sorted_tokens = x[idxs // k] (Kimi K2 "Add shared output"
 * page, moe_infer).  Copies rows bit for bit.
 *
 *   x         [T, d] rows of `dtype` (MR_BF16 or MR_F32).
 *   perm      [T*k] from mr_dispatch (used when inv_perm is NULL).
 *   inv_perm  [T*k] from mr_dispatch or NULL.  When given, each token row is
 *             read once and written to its k sorted positions; a slot whose
 *             entry is -1 (an assignment mr_dispatch dropped) writes no row.
 *   xs        [T*k, d] output rows in expert-sorted order.
 * Limits: 1 <= k <= 32.
 */
int mr_gather_rows(const void *x, int dtype, int T, int d, int k,
                   const int32_t *perm, const int32_t *inv_perm, void *xs,
                   mr_stream_t stream);

/*
 * mr_combine -- scatter-back, weighted combine and shared add (Kimi K2 "Add
 * shared output" page: new_x[idxs] = outs, view(T,k,d) * topk_weight summed
 * over k, cast back to the row dtype, then y + shared_experts(identity)).
 *
 *   expert_out [T*k, d] expert outputs in expert-sorted order (row i belongs
 *              to slot perm[i]), `dtype` MR_BF16 or MR_F32.
 *   w          [T, k] fp32 router weights.
 *   inv_perm   [T*k] from mr_dispatch; a slot whose entry is -1 (an
 *              assignment mr_dispatch dropped) adds nothing.
 *   shared     [T, d] shared-expert output of `dtype`, or NULL.
 *   y          [T, d] output of `dtype`.
 * Per element: acc = sum_j w[t,j] * expert_out[inv_perm[t*k+j]] in fp32;
 * bf16 rows: y = bf16(bf16(acc) + shared) (both roundings to nearest even);
 * fp32 rows: y = acc + shared.
 * Limits: 1 <= k <= 32.
 */
int mr_combine(const void *expert_out, int dtype, const float *w,
               const int32_t *inv_perm, const void *shared, void *y, int T,
               int d, int k, mr_stream_t stream);

/*
 * mr_launch_count -- number of kernels this library has launched in this
 * process (all devices and streams), for accounting in benchmarks.
 */
uint64_t mr_launch_count(void);

/*
 * mr_selftest_bounded_wait -- exercises the failure path of the library's
 * bounded waits without a GPU fault: one small kernel waits on something that
 * nothing completes -- which = 0: an mbarrier phase (the wait of the
 * tensor-core router kernels); which = 1: a grid barrier that only one of two
 * CTAs reaches (the wait of the cooperative dispatch kernel).  The wait gives
 * up after the library's limit (1 s), raises the device flag and the kernel
 * returns; mr_get_error then reports MR_ERR_TIMEOUT and the context stays
 * usable.  The grid-barrier case counts arrivals in a word of the library's
 * device image (cleared by the kernel), so the call allocates nothing; two
 * self tests of that kind running at once would share the word.  The pages
 * have no counterpart to this entry point (it is a test hook).  Returns
 * MR_ERR_INVALID_ARG for another `which`.
 */
int mr_selftest_bounded_wait(int which, mr_stream_t stream);

/*
 * mr_get_error -- synchronise `stream`, then read and clear the current
 * device's sticky error flag.  Returns MR_OK, MR_ERR_DEVICE (a bad expert id
 * or inconsistent counts were seen), MR_ERR_TIMEOUT (a bounded wait inside a
 * kernel gave up), MR_ERR_OVERFLOW (rows past a receive buffer's capacity
 * were dropped) or MR_ERR_CUDA (the synchronisation itself failed).  When
 * several were raised, the first of TIMEOUT, DEVICE, OVERFLOW is returned.
 */
int mr_get_error(mr_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MR_H */
