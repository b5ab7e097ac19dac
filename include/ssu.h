/*
 * ssu.h -- C ABI of the B200 selective-state-update library (libssu.so).
 *
 * The Mamba selective state update over a paged recurrent-state pool, in its forms
 * (single-token decode, multi-token prefill with an optional replay stash, tree verify
 * of a draft tree, and the replay of accepted speculative tokens or tree nodes), plus
 * slot clear, slot copy and gather/scatter; and the gated delta-rule decode core over a
 * pool with the same conventions.
 *
 * Sources: the "Selective State Update" page of the TensorRT-Edge-LLM C++ API
 * (mamba_ssm::invokeSelectiveStateUpdate, invokeSelectiveStateUpdatePrefill,
 * invokeSelectiveStateUpdateDDTree, struct MambaReplayLayerInfo,
 * invokeMambaReplayReconstructBatched, invokeMambaStateClear, invokeMambaStateGather,
 * invokeMambaStateScatter), the padding contract of the FlashInfer page
 * "flashinfer.gdn_fused_decode_step" (parameters state_indices and ssm_state), and the
 * "Recurrent State Manager" page (clearSlot, clear, copySlotFrom).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Device pointers unless stated otherwise. The caller owns every buffer; the library
 *    allocates nothing and never synchronises the host. The only state it keeps is a
 *    per-device cache of facts about the device and each kernel (SM count, occupancy,
 *    the kernel's shared-memory limit), filled once under std::call_once, so first calls
 *    from several host threads are safe; it never affects results. All work is enqueued
 *    on `stream` (a cudaStream_t; NULL is the legacy default stream), so every entry
 *    point may be recorded into a CUDA graph.
 *  - Optional inputs are NULL when absent.
 *  - Layouts are dense, row-major and batch-major as written beside each argument.
 *    Names: batch rows b, tokens t, heads h < nheads (H), groups g < ngroups (G),
 *    dim index d < dim (Dm), state index n < dstate (N). Head h reads group
 *    g = h / (H / G); H must be a multiple of G.
 *  - The state pool is [P, H, Dm, N] with dstate innermost. Slot s starts at element
 *    s * slot_stride; slot_stride >= H*Dm*N allows padded slots (the padding is never
 *    touched). The pool pointer must be 16-byte aligned and slot_stride * element size
 *    a multiple of 16 bytes.
 *  - state_indices [batch] int32 maps row b to its pool slot (NULL: row b uses slot b).
 *    A negative index marks a padding row: its state is neither read nor written and
 *    its output rows are written as zero. Indices of the active rows that are >= 0 must
 *    be distinct (two rows updating one slot would race); the kernels do not check this,
 *    ssu_check_state_indices does (for debugging).
 *  - Only rows b < active_batch are visited; rows beyond it are left untouched, so a
 *    graph captured at the maximum batch can run a smaller live batch.
 *  - An index >= P, or a length outside [0, T], is a caller bug that the pages leave
 *    undefined. Here it never causes an out-of-bounds access: the row is skipped (index)
 *    or the length clamped, and a bit is OR-ed into the optional device int32 err_flags:
 *    SSU_FLAG_INDEX_RANGE, SSU_FLAG_ACCEPTED_RANGE, SSU_FLAG_CONTEXT_RANGE,
 *    SSU_FLAG_NEGATIVE_LENGTH. Kernels that wait on their own asynchronous copies bound
 *    every wait and report SSU_FLAG_TIMEOUT instead of hanging.
 *  - Return value: SSU_OK, or an ssu_status error, in which case nothing was launched
 *    (SSU_ERR_CUDA: the launch itself failed, as cudaLaunchKernelEx reported it for this
 *    launch; an error left by unrelated earlier work in the calling thread is neither
 *    reported nor cleared). Sizes and dtype codes are checked first;
 *    a call with nothing to do (active_batch == 0, or T == 0) then returns SSU_OK without
 *    looking at any pointer, since empty tensors may carry NULL data pointers.
 *  - Arithmetic is fp32; fp16/bf16 values are widened exactly and results are rounded
 *    to nearest-even once when stored.
 */
#ifndef SSU_H
#define SSU_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st *ssu_stream_t;

typedef enum { SSU_F32 = 0, SSU_F16 = 1, SSU_BF16 = 2 } ssu_dtype;

typedef enum {
    SSU_OK = 0,
    SSU_ERR_NULL = 1,         /* a required pointer is NULL, or the stash is partial */
    SSU_ERR_SHAPE = 2,        /* sizes inconsistent (H % G, active > batch, stride, ...) */
    SSU_ERR_DTYPE = 3,        /* dtype code not one of ssu_dtype */
    SSU_ERR_UNSUPPORTED = 4,  /* dstate not in {8,16,32,64,128,256}, or (ssu_ddtree) a
                                 tree whose tables exceed shared memory */
    SSU_ERR_CUDA = 5,         /* the kernel launch failed (or the device could not be
                                 queried before it) */
    SSU_ERR_ALIGN = 6         /* pool pointer or slot stride not 16-byte aligned, or (in
                                 ssu_prefill / ssu_replay / ssu_ddtree) B, C or the stash B
                                 not 16-byte aligned */
} ssu_status;

enum {
    SSU_FLAG_INDEX_RANGE = 1,     /* state_indices[b] >= P: row skipped */
    SSU_FLAG_ACCEPTED_RANGE = 2,  /* accepted_lengths[b] > T: clamped to T */
    SSU_FLAG_CONTEXT_RANGE = 4,   /* context_lengths[b] > T: clamped to T */
    SSU_FLAG_NEGATIVE_LENGTH = 8, /* a negative length: treated as 0 */
    SSU_FLAG_TIMEOUT = 16,        /* an internal wait gave up after 2 s (never expected);
                                     the outputs of that launch are incomplete */
    SSU_FLAG_LAYER = 32,          /* a per-layer pointer was NULL or not 16-byte aligned:
                                     that layer was skipped */
    SSU_FLAG_TREE = 64,           /* ssu_ddtree: a node's parent walk was malformed (its
                                     outputs are 0); replay: an accepted node id outside
                                     [0, T) (the row was left untouched) */
    SSU_FLAG_DUPLICATE_INDEX = 128 /* ssu_check_state_indices only: two active rows name
                                     the same slot */
};

/* Per-layer device pointers of a multi-layer replay: one entry per layer, in a device
 * array (Selective State Update page, struct MambaReplayLayerInfo). All layers share the
 * geometry, slot stride and pool size given to the call. */
typedef struct {
    void *state;          /* the layer's pool [P, H, Dm, N], 16-byte aligned */
    const float *st_dA;   /* the layer's replay stash, as written by ssu_prefill */
    const float *st_U;
    const float *st_B;    /* 16-byte aligned */
    const float *st_dt;
} ssu_replay_layer;

/* Per-layer device pointers of the recurrent and convolution states (Selective State
 * Update page, struct MambaStateLayerInfo), for the multi-layer slot clear. */
typedef struct {
    void *recurrent_state;
    void *conv_state;     /* may be NULL: the layer has no convolution state */
} ssu_layer_states;

/*
 * ssu_decode -- one token (seq_len == 1) for every active row.
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdate:
 *     dt_eff    = softplus(dt + dt_bias) if dt_softplus, else dt + dt_bias
 *     new_state = state * exp(A * dt_eff) + B * dt_eff * x        (in place, in the pool)
 *     out       = sum_n new_state[n] * C[n] + D * x,  times silu(z) if z is given
 *
 *   x        [batch, H, Dm]  x_dtype          A        [H] fp32
 *   B, C     [batch, G, N]   bc_dtype         dt       [batch, H] fp32
 *   dt_bias  [H] fp32 (optional)              D        [H] fp32 (optional)
 *   z        [batch, H, Dm]  x_dtype (optional gate)
 *   state    pool [P, H, Dm, N] state_dtype, slot stride slot_stride elements; in place
 *   out      [batch, H, Dm]  x_dtype; rows b >= active_batch are not written
 *   state_indices [batch] int32 (optional); err_flags int32 (optional)
 * The output is reduced from the fp32 new state before it is rounded to state_dtype.
 */
int ssu_decode(const void *x, int x_dtype, const float *A,
               const void *B, const void *C, int bc_dtype,
               const float *dt, const float *dt_bias, const float *D, const void *z,
               void *state, int state_dtype, int64_t slot_stride, int32_t P,
               void *out, const int32_t *state_indices,
               int32_t batch, int32_t active_batch, int32_t nheads, int32_t ngroups,
               int32_t dim, int32_t dstate, int dt_softplus, int32_t *err_flags,
               ssu_stream_t stream);

/*
 * ssu_prefill -- all T tokens (seq_len > 1) in one launch.
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdatePrefill:
 * the decode recurrence run over t < L_b = context_lengths[b] (all T when NULL), with
 * the state held on chip across the tokens.
 *
 *   x, z, out [batch, T, H, Dm] x_dtype;  B, C [batch, T, G, N] bc_dtype;
 *   dt [batch, T, H] fp32; other arguments as in ssu_decode.
 *   Without the stash: the state after L_b tokens is stored back once (not when L_b=0).
 *   With the replay stash (all four or none; fp32, written for t < L_b only):
 *     st_dA [batch, T, H]      = exp(A * dt_eff)   (the decay factor)
 *     st_U  [batch, T, H, Dm]  = x (unscaled, widened)
 *     st_B  [batch, T, G, N]   = B (widened)
 *     st_dt [batch, T, H]      = dt_eff
 *   and the committed state is only read, never written.
 *   Positions t >= L_b of out and of the stash are not written. A padding row writes
 *   zeros to out at every t < T and touches nothing else.
 */
int ssu_prefill(const void *x, int x_dtype, const float *A,
                const void *B, const void *C, int bc_dtype,
                const float *dt, const float *dt_bias, const float *D, const void *z,
                void *state, int state_dtype, int64_t slot_stride, int32_t P,
                void *out, const int32_t *state_indices, const int32_t *context_lengths,
                float *st_dA, float *st_U, float *st_B, float *st_dt,
                int32_t batch, int32_t active_batch, int32_t T, int32_t nheads,
                int32_t ngroups, int32_t dim, int32_t dstate, int dt_softplus,
                int32_t *err_flags, ssu_stream_t stream);

/*
 * ssu_replay -- re-apply accepted speculative tokens to the committed state.
 * Selective State Update page, struct MambaReplayLayerInfo and
 * invokeMambaReplayReconstructBatched: for t < k_b = accepted_lengths[b],
 *     state = state * st_dA[b,t,h] + st_B[b,t,g,n] * st_dt[b,t,h] * st_U[b,t,h,d]
 * in place; the state is written once, and not at all when k_b == 0.
 *   stash buffers as written by ssu_prefill (or ssu_ddtree), with T their token (node)
 *   extent; accepted_lengths [batch] int32 (required); no output.
 *   accepted_node_ids [batch, max_accept_len] int32 (optional; the acceptedNodeIds and
 *   maxAcceptLen arguments of invokeMambaReplayReconstructBatched): when given, the t-th
 *   replayed token is stash entry accepted_node_ids[b][t] instead of t (the accepted
 *   root-to-node path of a tree verify), and k_b is bounded by max_accept_len instead
 *   of T. A row with an id outside [0, T) among its first k_b is left untouched and
 *   flagged SSU_FLAG_TREE. When NULL, max_accept_len is ignored.
 */
int ssu_replay(void *state, int state_dtype, int64_t slot_stride, int32_t P,
               const float *st_dA, const float *st_U, const float *st_B,
               const float *st_dt, const int32_t *accepted_lengths,
               const int32_t *state_indices, int32_t batch, int32_t active_batch,
               int32_t T, int32_t nheads, int32_t ngroups, int32_t dim, int32_t dstate,
               const int32_t *accepted_node_ids, int32_t max_accept_len,
               int32_t *err_flags, ssu_stream_t stream);

/*
 * ssu_replay_layers -- ssu_replay over num_layers layers in one launch.
 * Selective State Update page, invokeMambaReplayReconstructBatched with a device array of
 * MambaReplayLayerInfo: every layer re-applies the first accepted_lengths[b] tokens of its
 * own stash to its own pool; accepted_lengths and state_indices are shared by the layers.
 *   layers      device array [num_layers] of ssu_replay_layer
 *   other arguments as in ssu_replay (their geometry applies to every layer)
 * A layer whose pointers are NULL or misaligned is skipped and flagged SSU_FLAG_LAYER.
 */
int ssu_replay_layers(const ssu_replay_layer *layers, int32_t num_layers, int state_dtype,
                      int64_t slot_stride, int32_t P, const int32_t *accepted_lengths,
                      const int32_t *state_indices, int32_t batch, int32_t active_batch,
                      int32_t T, int32_t nheads, int32_t ngroups, int32_t dim, int32_t dstate,
                      const int32_t *accepted_node_ids, int32_t max_accept_len,
                      int32_t *err_flags, ssu_stream_t stream);

/*
 * ssu_conv_decode -- the causal conv1d update of the raw xBC channels fused with one
 * decode token, over the same slot of a conv pool and a recurrent pool.
 * Selective State Update page (struct MambaStateLayerInfo: convState beside
 * recurrentState; invokeSelectiveStateUpdate for the decode) and the causal conv1d update
 * of the FlashInfer page flashinfer.gdn_fused_decode_step. For every channel c of a live
 * row (conv_dim = H*Dm + 2*G*N channels in the order x, B, C):
 *     window = (the slot's width-1 taps, oldest first, then xbc[b, c])
 *     v[c]   = sum_k conv_weight[c, k] * window[k] + conv_bias[c], times sigmoid(v[c]) if
 *              conv_silu;   the taps become window[1 ..]
 * then ssu_decode runs with x = v[0 : H*Dm] as [H, Dm], B and C = the next two G*N
 * blocks as [G, N] (kept in fp32, never stored).
 *   xbc          [batch, conv_dim] x_dtype (raw, pre-conv channels)
 *   conv_weight  [conv_dim, width] x_dtype;  conv_bias [conv_dim] x_dtype (optional)
 *   conv_state   conv pool of x_dtype, tap k of channel c of slot s at element
 *                s*conv_slot_stride + c*conv_stride_c + k*conv_stride_k (k < width-1):
 *                channel-major windows [P, conv_dim, width-1] use (.., width-1, 1),
 *                tap-major [P, width-1, conv_dim] use (.., 1, conv_dim); unused when
 *                width == 1
 *   width        1..16 taps;  other arguments as in ssu_decode (z, out [batch, H, Dm])
 * Both pools are indexed by state_indices; a padding row touches neither and outputs 0.
 * Two launches on `stream`: the fused conv + decode, which shifts the windows of the x
 * channels (each owned by one unit of work) and only reads the B and C taps (shared by
 * all heads of a group), then the shift of the B and C windows of every live row.
 */
int ssu_conv_decode(const void *xbc, int x_dtype, const void *conv_weight,
                    const void *conv_bias, void *conv_state, int64_t conv_slot_stride,
                    int64_t conv_stride_c, int64_t conv_stride_k, int32_t width, int conv_silu,
                    const float *A, const float *dt, const float *dt_bias, const float *D,
                    const void *z, void *state, int state_dtype, int64_t slot_stride,
                    int32_t P, void *out, const int32_t *state_indices, int32_t batch,
                    int32_t active_batch, int32_t nheads, int32_t ngroups, int32_t dim,
                    int32_t dstate, int dt_softplus, int32_t *err_flags, ssu_stream_t stream);

/*
 * gdn_decode -- one gated delta-rule decode token over a paged fp32 state pool.
 * The recurrent core of the FlashInfer page flashinfer.gdn_fused_decode_step (the b/a
 * projection, the conv1d update and the q/k/v split that the page folds around it are
 * not part of this call). Per active row b and value head hv, with key head
 * hk = hv / (num_v_heads / num_k_heads):
 *     q, k   [batch, num_k_heads, K] of head hk; with use_qk_l2norm each is divided by
 *            sqrt(sum of squares + 1e-6); q is then multiplied by scale (0: 1/sqrt(K))
 *     alpha  = exp(-exp(A_log[hv]) * softplus(a[b,hv] + dt_bias[hv]))
 *     beta   = 1 / (1 + exp(-b[b,hv]))
 *     every state row i < V (state [P, num_v_heads, V, K], K innermost, slot stride
 *     slot_stride elements, fp32, updated in place):
 *         d = beta * (v[b,hv,i] - alpha * (S_i . k));  S_i = alpha * S_i + d * k;
 *         out[b,hv,i] = S_i . q
 *   q, k [batch, num_k_heads, K]; v, out [batch, num_v_heads, V]; a, b
 *   [batch, num_v_heads]: all x_dtype;
 *   A_log, dt_bias (optional) [num_v_heads] fp32; K = head_k_dim in {8,...,256} (powers
 *   of two), V = head_v_dim any. Padding and index rules as in ssu_decode.
 */
int gdn_decode(const void *q, const void *k, const void *v, int x_dtype, const void *a,
               const void *b, const float *A_log, const float *dt_bias, float scale,
               int use_qk_l2norm, float *state, int64_t slot_stride, int32_t P, void *out,
               const int32_t *state_indices, int32_t batch, int32_t active_batch,
               int32_t num_k_heads, int32_t num_v_heads, int32_t head_k_dim,
               int32_t head_v_dim, int32_t *err_flags, ssu_stream_t stream);

/*
 * ssu_ddtree -- tree verify: every node of one draft tree per row, each evaluated from the
 * committed state along its own ancestor path.
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdateDDTree: the committed
 * state is only read; for node i of row b the recurrence of ssu_decode runs from the
 * committed state over the nodes on i's path (found by following tree_parent_ids from i
 * to the root), in root-to-node order, and out[b,i] is node i's output there (no z gate);
 * node i's own replay tuple goes to the stash at position i.
 *
 *   x, out [batch, T, H, Dm] x_dtype; B, C [batch, T, G, N] bc_dtype (B 16-byte
 *   aligned); dt [batch, T, H] fp32; T = nodes per tree, 1..128 (the verify budget).
 *   tree_parent_ids [batch, T] int32: parent node of each node, -1 for a node attached
 *   directly to the committed state.
 *   tree_depths [batch, T] int32: number of tree ancestors of each node (0 when its
 *   parent is -1). A node whose walk does not take exactly that many steps inside
 *   [0, T) and then reach -1 is malformed: its outputs are 0 and SSU_FLAG_TREE is set.
 *   Stash (required, fp32, every node of every non-padding row): st_dA [batch, T, H],
 *   st_U [batch, T, H, Dm], st_B [batch, T, G, N], st_dt [batch, T, H], as in
 *   ssu_prefill; replay an accepted path with ssu_replay and accepted_node_ids.
 *   A padding row writes zeros to out at every node and nothing else.
 *   With bf16 B and C (C 16-byte aligned) and dstate 64 or 128 the dense part, the dot
 *   products of the committed state with every node's C, runs on the tensor cores with
 *   the state split into bf16 pieces that sum to it exactly (fp32 state: to within 2^-24
 *   of each element), so either way the outputs carry fp32 accuracy.
 * Returns SSU_ERR_SHAPE for T > 128, SSU_ERR_UNSUPPORTED when the row's tables do not fit
 * in shared memory (about T (dstate + 4) x 4 + 5 T (T + 1) + T x 64 x element bytes of x
 * bytes must stay under 227 KB: every T up to 128 for dstate <= 128).
 */
int ssu_ddtree(const void *x, int x_dtype, const float *A, const void *B, const void *C,
               int bc_dtype, const float *dt, const float *dt_bias, const float *D,
               const void *state, int state_dtype, int64_t slot_stride, int32_t P, void *out,
               const int32_t *tree_parent_ids, const int32_t *tree_depths,
               const int32_t *state_indices, float *st_dA, float *st_U, float *st_B,
               float *st_dt, int32_t batch, int32_t active_batch, int32_t T, int32_t nheads,
               int32_t ngroups, int32_t dim, int32_t dstate, int dt_softplus,
               int32_t *err_flags, ssu_stream_t stream);

/*
 * pool_clear_slot -- zero one slot, or every slot when slot == -1.
 * Selective State Update page, invokeMambaStateClear; Recurrent State Manager page,
 * clearSlot / clear. slot_bytes is the slot stride in bytes; other slots are untouched.
 * Returns SSU_ERR_SHAPE for slot < -1 or slot >= P.
 */
int pool_clear_slot(void *pool, int64_t slot_bytes, int32_t P, int32_t slot,
                    ssu_stream_t stream);

/*
 * pool_copy_slot -- copy one slot between two pools with the same per-slot geometry
 * (slot_bytes), which may hold different slot counts.
 * Recurrent State Manager page, copySlotFrom. The two slot ranges must not overlap
 * partially (the same slot of the same pool is a no-op copy).
 * Returns SSU_ERR_SHAPE for a slot outside its pool.
 */
int pool_copy_slot(void *dst_pool, int32_t dst_P, int32_t dst_slot,
                   const void *src_pool, int32_t src_P, int32_t src_slot,
                   int64_t slot_bytes, ssu_stream_t stream);

/*
 * pool_clear_slot_layers -- pool_clear_slot over the recurrent and convolution states of
 * num_layers layers in one launch. Selective State Update page, invokeMambaStateClear.
 *   layers                device array [num_layers] of ssu_layer_states
 *   recurrent_slot_bytes  slot stride of every recurrent pool, in bytes
 *   conv_slot_bytes       slot stride of every convolution pool (0: none)
 * Returns SSU_ERR_SHAPE for slot < -1 or slot >= P.
 */
int pool_clear_slot_layers(const ssu_layer_states *layers, int32_t num_layers, int32_t P,
                           int32_t slot, int64_t recurrent_slot_bytes, int64_t conv_slot_bytes,
                           ssu_stream_t stream);

/*
 * pool_gather / pool_scatter -- copy active rows between the pool and a dense batch.
 * Selective State Update page, invokeMambaStateGather / invokeMambaStateScatter: for
 * b < active_batch, dense[b] = pool[state_indices[b]] (gather) or
 * pool[state_indices[b]] = dense[b] (scatter); rows are slot_bytes long, dense rows are
 * contiguous ([batch, slot_bytes]), pool rows sit slot_bytes apart.
 * A padding row (negative index): gather writes zeros to dense[b], scatter writes nothing.
 * An index >= P: the row is skipped and SSU_FLAG_INDEX_RANGE is set.
 */
int pool_gather(const void *pool, int64_t slot_bytes, int32_t P, void *dense,
                const int32_t *state_indices, int32_t batch, int32_t active_batch,
                int32_t *err_flags, ssu_stream_t stream);
int pool_scatter(const void *dense, void *pool, int64_t slot_bytes, int32_t P,
                 const int32_t *state_indices, int32_t batch, int32_t active_batch,
                 int32_t *err_flags, ssu_stream_t stream);

/*
 * ssu_check_state_indices -- debug check of a row-to-slot map before it is used.
 * The padding contract of the FlashInfer page flashinfer.gdn_fused_decode_step
 * (state_indices): every batch row reads and writes its own slot, so the active rows'
 * non-negative indices must be distinct (the other entry points take that as a
 * precondition and do not check it). One launch on `stream` that ORs into the device
 * int32 *err_flags (required): SSU_FLAG_DUPLICATE_INDEX when two rows b < active_batch
 * hold the same index >= 0, SSU_FLAG_INDEX_RANGE when one holds an index >= P. Negative
 * indices (padding) may repeat. O(active_batch^2) comparisons: meant for debugging and
 * tests, not for every step. Like every entry point it allocates nothing and does not
 * synchronise; the caller reads the flags when it chooses.
 * Returns SSU_ERR_NULL for a NULL state_indices or err_flags (when active_batch > 0),
 * SSU_ERR_SHAPE for active_batch outside [0, batch] or P < 0.
 */
int ssu_check_state_indices(const int32_t *state_indices, int32_t batch,
                            int32_t active_batch, int32_t P, int32_t *err_flags,
                            ssu_stream_t stream);

/* A constant string naming an ssu_status value. */
const char *ssu_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SSU_H */
