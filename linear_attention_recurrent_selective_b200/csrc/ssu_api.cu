// ssu_api.cu -- the extern "C" boundary of libssu: argument checks, then one launch.
//
// Every entry point validates its arguments on the host without touching device memory
// (so it stays legal under CUDA-graph capture), returns an ssu_status error without
// launching anything when a check fails, and otherwise enqueues its kernel on the
// caller's stream (one launch; ssu_conv_decode enqueues two). Kernels are launched with
// cudaLaunchKernelEx and the call returns that launch's own status: an error left by
// unrelated earlier work in the caller's thread is neither reported nor cleared. Values that live on the device (stateIndices, contextLengths,
// acceptedLengths, tree parents and depths, accepted node ids) are checked in-kernel,
// as the padding contract of the FlashInfer page flashinfer.gdn_fused_decode_step
// requires for graph replay.
#include "ssu_common.cuh"
#ifdef SSU_WAIT_TEST
#include "ssu_async.cuh"
#include "ssu_wait_test.h"
static_assert(SSU_WAIT_STREAM == ssu::kFaultStream && SSU_WAIT_PREFILL == ssu::kFaultPrefill &&
                  SSU_WAIT_TREE_STATE == ssu::kFaultTreeState &&
                  SSU_WAIT_TREE_X == ssu::kFaultTreeX && SSU_WAIT_TREE_MMA == ssu::kFaultTreeMma,
              "wait sites of the test header and the kernels agree");
#endif

namespace {

bool valid_dtype(int d) { return d == SSU_F32 || d == SSU_F16 || d == SSU_BF16; }

int elem_bytes(int d) { return d == SSU_F32 ? 4 : 2; }

bool supported_dstate(int n)
{
    return n == 8 || n == 16 || n == 32 || n == 64 || n == 128 || n == 256;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Sizes and dtypes only (no pointer is looked at), so that an empty batch, whose tensors
// may carry NULL data pointers, can be accepted before the pointer checks.
int check_sizes(int state_dtype, int64_t slot_stride, int32_t P, const int32_t *idx,
                int32_t batch, int32_t active, int32_t H, int32_t G, int32_t Dm, int32_t N)
{
    if (!valid_dtype(state_dtype))
        return SSU_ERR_DTYPE;
    if (batch < 0 || active < 0 || active > batch || P < 0)
        return SSU_ERR_SHAPE;
    if (H <= 0 || G <= 0 || Dm <= 0 || N <= 0 || H % G != 0)
        return SSU_ERR_SHAPE;
    if (slot_stride < (int64_t)H * Dm * N)
        return SSU_ERR_SHAPE;
    if (!idx && active > P)               // row b is slot b: every active row needs one
        return SSU_ERR_SHAPE;
    if (!supported_dstate(N))
        return SSU_ERR_UNSUPPORTED;
    return SSU_OK;
}

int check_pool_alignment(const void *state, int state_dtype, int64_t slot_stride)
{
    if (!aligned16(state) || (slot_stride * elem_bytes(state_dtype)) % 16 != 0)
        return SSU_ERR_ALIGN;
    return SSU_OK;
}

ssu::DecodeArgs pack_decode(const void *x, int x_dtype, const float *A, const void *B,
                            const void *C, int bc_dtype, const float *dt,
                            const float *dt_bias, const float *D, const void *z,
                            void *state, int64_t slot_stride, int32_t P, void *out,
                            const int32_t *idx, int32_t batch, int32_t active, int32_t H,
                            int32_t G, int32_t Dm, int32_t N, int softplus, int32_t *err)
{
    ssu::DecodeArgs a;
    a.x = x;
    a.A = A;
    a.B = B;
    a.C = C;
    a.dt = dt;
    a.dt_bias = dt_bias;
    a.D = D;
    a.z = z;
    a.state = state;
    a.out = out;
    a.idx = idx;
    a.err = err;
    a.slot_stride = slot_stride;
    a.P = P;
    a.batch = batch;
    a.active = active;
    a.H = H;
    a.G = G;
    a.Dm = Dm;
    a.N = N;
    a.x_dtype = x_dtype;
    a.bc_dtype = bc_dtype;
    a.softplus = softplus ? 1 : 0;
    return a;
}

}  // namespace

extern "C" {

int ssu_decode(const void *x, int x_dtype, const float *A, const void *B, const void *C,
               int bc_dtype, const float *dt, const float *dt_bias, const float *D,
               const void *z, void *state, int state_dtype, int64_t slot_stride, int32_t P,
               void *out, const int32_t *state_indices, int32_t batch,
               int32_t active_batch, int32_t nheads, int32_t ngroups, int32_t dim,
               int32_t dstate, int dt_softplus, int32_t *err_flags, ssu_stream_t stream)
{
    if (!valid_dtype(x_dtype) || !valid_dtype(bc_dtype))
        return SSU_ERR_DTYPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0)
        return rc;
    if (!x || !A || !B || !C || !dt || !state || !out)
        return SSU_ERR_NULL;
    if ((rc = check_pool_alignment(state, state_dtype, slot_stride)) != SSU_OK)
        return rc;
    ssu::DecodeArgs a = pack_decode(x, x_dtype, A, B, C, bc_dtype, dt, dt_bias, D, z, state,
                                    slot_stride, P, out, state_indices, batch, active_batch,
                                    nheads, ngroups, dim, dstate, dt_softplus, err_flags);
    return ssu::launch_decode(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_prefill(const void *x, int x_dtype, const float *A, const void *B, const void *C,
                int bc_dtype, const float *dt, const float *dt_bias, const float *D,
                const void *z, void *state, int state_dtype, int64_t slot_stride, int32_t P,
                void *out, const int32_t *state_indices, const int32_t *context_lengths,
                float *st_dA, float *st_U, float *st_B, float *st_dt, int32_t batch,
                int32_t active_batch, int32_t T, int32_t nheads, int32_t ngroups,
                int32_t dim, int32_t dstate, int dt_softplus, int32_t *err_flags,
                ssu_stream_t stream)
{
    if (!valid_dtype(x_dtype) || !valid_dtype(bc_dtype))
        return SSU_ERR_DTYPE;
    if (T < 0)
        return SSU_ERR_SHAPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0 || T == 0)
        return rc;
    if (!x || !A || !B || !C || !dt || !state || !out)
        return SSU_ERR_NULL;
    const int given = (st_dA != nullptr) + (st_U != nullptr) + (st_B != nullptr) +
                      (st_dt != nullptr);
    if (given != 0 && given != 4)
        return SSU_ERR_NULL;
    if ((rc = check_pool_alignment(state, state_dtype, slot_stride)) != SSU_OK)
        return rc;
    if (!aligned16(B) || !aligned16(C) || (st_B && !aligned16(st_B)))
        return SSU_ERR_ALIGN;
    ssu::PrefillArgs a;
    a.d = pack_decode(x, x_dtype, A, B, C, bc_dtype, dt, dt_bias, D, z, state, slot_stride,
                      P, out, state_indices, batch, active_batch, nheads, ngroups, dim,
                      dstate, dt_softplus, err_flags);
    a.ctx = context_lengths;
    a.st_dA = st_dA;
    a.st_U = st_U;
    a.st_B = st_B;
    a.st_dt = st_dt;
    a.T = T;
    return ssu::launch_prefill(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_replay(void *state, int state_dtype, int64_t slot_stride, int32_t P,
               const float *st_dA, const float *st_U, const float *st_B, const float *st_dt,
               const int32_t *accepted_lengths, const int32_t *state_indices,
               int32_t batch, int32_t active_batch, int32_t T, int32_t nheads,
               int32_t ngroups, int32_t dim, int32_t dstate,
               const int32_t *accepted_node_ids, int32_t max_accept_len, int32_t *err_flags,
               ssu_stream_t stream)
{
    if (T < 0 || (accepted_node_ids && max_accept_len < 0))
        return SSU_ERR_SHAPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0 || T == 0)
        return rc;
    if (!state || !st_dA || !st_U || !st_B || !st_dt || !accepted_lengths)
        return SSU_ERR_NULL;
    if ((rc = check_pool_alignment(state, state_dtype, slot_stride)) != SSU_OK)
        return rc;
    if (!aligned16(st_B))
        return SSU_ERR_ALIGN;
    ssu::ReplayArgs a;
    a.layers = nullptr;
    a.num_layers = 1;
    a.state = state;
    a.st_dA = st_dA;
    a.st_U = st_U;
    a.st_B = st_B;
    a.st_dt = st_dt;
    a.acc = accepted_lengths;
    a.idx = state_indices;
    a.nodes = accepted_node_ids;
    a.err = err_flags;
    a.slot_stride = slot_stride;
    a.P = P;
    a.batch = batch;
    a.active = active_batch;
    a.T = T;
    a.H = nheads;
    a.G = ngroups;
    a.Dm = dim;
    a.N = dstate;
    a.max_accept = accepted_node_ids ? max_accept_len : T;
    return ssu::launch_replay(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_replay_layers(const ssu_replay_layer *layers, int32_t num_layers, int state_dtype,
                      int64_t slot_stride, int32_t P, const int32_t *accepted_lengths,
                      const int32_t *state_indices, int32_t batch, int32_t active_batch,
                      int32_t T, int32_t nheads, int32_t ngroups, int32_t dim, int32_t dstate,
                      const int32_t *accepted_node_ids, int32_t max_accept_len,
                      int32_t *err_flags, ssu_stream_t stream)
{
    if (T < 0 || num_layers < 0 || (accepted_node_ids && max_accept_len < 0))
        return SSU_ERR_SHAPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0 || T == 0 || num_layers == 0)
        return rc;
    if (!layers || !accepted_lengths)
        return SSU_ERR_NULL;
    if ((slot_stride * elem_bytes(state_dtype)) % 16 != 0)
        return SSU_ERR_ALIGN;
    ssu::ReplayArgs a;
    a.layers = layers;                   // per-layer pointers are checked in-kernel
    a.num_layers = num_layers;
    a.state = nullptr;
    a.st_dA = a.st_U = a.st_B = a.st_dt = nullptr;
    a.acc = accepted_lengths;
    a.idx = state_indices;
    a.nodes = accepted_node_ids;
    a.err = err_flags;
    a.slot_stride = slot_stride;
    a.P = P;
    a.batch = batch;
    a.active = active_batch;
    a.T = T;
    a.H = nheads;
    a.G = ngroups;
    a.Dm = dim;
    a.N = dstate;
    a.max_accept = accepted_node_ids ? max_accept_len : T;
    return ssu::launch_replay(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_conv_decode(const void *xbc, int x_dtype, const void *conv_weight,
                    const void *conv_bias, void *conv_state, int64_t conv_slot_stride,
                    int64_t conv_stride_c, int64_t conv_stride_k, int32_t width, int conv_silu,
                    const float *A, const float *dt, const float *dt_bias, const float *D,
                    const void *z, void *state, int state_dtype, int64_t slot_stride,
                    int32_t P, void *out, const int32_t *state_indices, int32_t batch,
                    int32_t active_batch, int32_t nheads, int32_t ngroups, int32_t dim,
                    int32_t dstate, int dt_softplus, int32_t *err_flags, ssu_stream_t stream)
{
    if (!valid_dtype(x_dtype))
        return SSU_ERR_DTYPE;
    if (width < 1 || width > 16)
        return SSU_ERR_SHAPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0)
        return rc;
    const int64_t cd = (int64_t)nheads * dim + 2 * (int64_t)ngroups * dstate;
    if (width > 1) {
        if (conv_slot_stride < 0 || conv_stride_c < 0 || conv_stride_k < 0)
            return SSU_ERR_SHAPE;
        // every (channel, tap) of a slot must lie inside the slot's extent
        if ((cd - 1) * conv_stride_c + (int64_t)(width - 2) * conv_stride_k >= conv_slot_stride)
            return SSU_ERR_SHAPE;
    }
    if (!xbc || !conv_weight || !A || !dt || !state || !out || (width > 1 && !conv_state))
        return SSU_ERR_NULL;
    if ((rc = check_pool_alignment(state, state_dtype, slot_stride)) != SSU_OK)
        return rc;
    ssu::ConvArgs a;
    a.d = pack_decode(nullptr, x_dtype, A, nullptr, nullptr, x_dtype, dt, dt_bias, D, z, state,
                      slot_stride, P, out, state_indices, batch, active_batch, nheads, ngroups,
                      dim, dstate, dt_softplus, err_flags);
    a.xbc = xbc;
    a.w = conv_weight;
    a.bias = conv_bias;
    a.cstate = conv_state;
    a.cslot = conv_slot_stride;
    a.cc = conv_stride_c;
    a.ck = conv_stride_k;
    a.width = width;
    a.silu = conv_silu ? 1 : 0;
    return ssu::launch_conv_decode(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int gdn_decode(const void *q, const void *k, const void *v, int x_dtype, const void *a,
               const void *b, const float *A_log, const float *dt_bias, float scale,
               int use_qk_l2norm, float *state, int64_t slot_stride, int32_t P, void *out,
               const int32_t *state_indices, int32_t batch, int32_t active_batch,
               int32_t num_k_heads, int32_t num_v_heads, int32_t head_k_dim,
               int32_t head_v_dim, int32_t *err_flags, ssu_stream_t stream)
{
    if (!valid_dtype(x_dtype))
        return SSU_ERR_DTYPE;
    if (batch < 0 || active_batch < 0 || active_batch > batch || P < 0)
        return SSU_ERR_SHAPE;
    if (num_k_heads <= 0 || num_v_heads <= 0 || num_v_heads % num_k_heads != 0 ||
        head_k_dim <= 0 || head_v_dim <= 0)
        return SSU_ERR_SHAPE;
    if (slot_stride < (int64_t)num_v_heads * head_v_dim * head_k_dim)
        return SSU_ERR_SHAPE;
    if (!state_indices && active_batch > P)
        return SSU_ERR_SHAPE;
    if (!supported_dstate(head_k_dim))
        return SSU_ERR_UNSUPPORTED;
    if (active_batch == 0)
        return SSU_OK;
    if (!q || !k || !v || !a || !b || !A_log || !state || !out)
        return SSU_ERR_NULL;
    int rc;
    if ((rc = check_pool_alignment(state, SSU_F32, slot_stride)) != SSU_OK)
        return rc;
    ssu::GdnArgs g;
    g.q = q;
    g.k = k;
    g.v = v;
    g.a = a;
    g.b = b;
    g.A_log = A_log;
    g.dt_bias = dt_bias;
    g.state = state;
    g.out = out;
    g.idx = state_indices;
    g.err = err_flags;
    g.slot_stride = slot_stride;
    g.scale = scale != 0.f ? scale : 1.f / sqrtf((float)head_k_dim);
    g.P = P;
    g.batch = batch;
    g.active = active_batch;
    g.HK = num_k_heads;
    g.HV = num_v_heads;
    g.K = head_k_dim;
    g.V = head_v_dim;
    g.x_dtype = x_dtype;
    g.l2norm = use_qk_l2norm ? 1 : 0;
    return ssu::launch_gdn_decode(g, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_ddtree(const void *x, int x_dtype, const float *A, const void *B, const void *C,
               int bc_dtype, const float *dt, const float *dt_bias, const float *D,
               const void *state, int state_dtype, int64_t slot_stride, int32_t P, void *out,
               const int32_t *tree_parent_ids, const int32_t *tree_depths,
               const int32_t *state_indices, float *st_dA, float *st_U, float *st_B,
               float *st_dt, int32_t batch, int32_t active_batch, int32_t T, int32_t nheads,
               int32_t ngroups, int32_t dim, int32_t dstate, int dt_softplus,
               int32_t *err_flags, ssu_stream_t stream)
{
    if (!valid_dtype(x_dtype) || !valid_dtype(bc_dtype))
        return SSU_ERR_DTYPE;
    if (T < 0 || T > 128)
        return SSU_ERR_SHAPE;
    int rc = check_sizes(state_dtype, slot_stride, P, state_indices, batch, active_batch,
                         nheads, ngroups, dim, dstate);
    if (rc != SSU_OK || active_batch == 0 || T == 0)
        return rc;
    if (!x || !A || !B || !C || !dt || !state || !out || !tree_parent_ids || !tree_depths ||
        !st_dA || !st_U || !st_B || !st_dt)
        return SSU_ERR_NULL;
    if ((rc = check_pool_alignment(state, state_dtype, slot_stride)) != SSU_OK)
        return rc;
    if (!aligned16(B))
        return SSU_ERR_ALIGN;
    ssu::TreeArgs a;
    a.d = pack_decode(x, x_dtype, A, B, C, bc_dtype, dt, dt_bias, D, nullptr,
                      const_cast<void *>(state), slot_stride, P, out, state_indices, batch,
                      active_batch, nheads, ngroups, dim, dstate, dt_softplus, err_flags);
    a.parents = tree_parent_ids;
    a.depths = tree_depths;
    a.st_dA = st_dA;
    a.st_U = st_U;
    a.st_B = st_B;
    a.st_dt = st_dt;
    a.T = T;
    return ssu::launch_ddtree(a, state_dtype, reinterpret_cast<cudaStream_t>(stream));
}

int pool_clear_slot_layers(const ssu_layer_states *layers, int32_t num_layers, int32_t P,
                           int32_t slot, int64_t recurrent_slot_bytes, int64_t conv_slot_bytes,
                           ssu_stream_t stream)
{
    if (num_layers < 0 || P < 0 || slot < -1 || slot >= P || recurrent_slot_bytes < 0 ||
        conv_slot_bytes < 0)
        return SSU_ERR_SHAPE;
    if (num_layers == 0)
        return SSU_OK;
    if (!layers)
        return SSU_ERR_NULL;
    return ssu::launch_clear_layers(layers, num_layers, P, slot, recurrent_slot_bytes,
                                           conv_slot_bytes,
                                           reinterpret_cast<cudaStream_t>(stream));
}

static int gather_scatter(const void *pool, int64_t slot_bytes, int32_t P, void *dense,
                          const int32_t *state_indices, int32_t batch, int32_t active_batch,
                          int scatter, int32_t *err_flags, ssu_stream_t stream)
{
    if (slot_bytes < 0 || P < 0 || batch < 0 || active_batch < 0 || active_batch > batch)
        return SSU_ERR_SHAPE;
    if (!state_indices && active_batch > P)
        return SSU_ERR_SHAPE;
    if (active_batch == 0 || slot_bytes == 0)
        return SSU_OK;
    if (!pool || !dense)
        return SSU_ERR_NULL;
    return ssu::launch_gather(pool, slot_bytes, P, dense, state_indices, active_batch,
                                     scatter, err_flags, reinterpret_cast<cudaStream_t>(stream));
}

int pool_gather(const void *pool, int64_t slot_bytes, int32_t P, void *dense,
                const int32_t *state_indices, int32_t batch, int32_t active_batch,
                int32_t *err_flags, ssu_stream_t stream)
{
    return gather_scatter(pool, slot_bytes, P, dense, state_indices, batch, active_batch, 0,
                          err_flags, stream);
}

int pool_scatter(const void *dense, void *pool, int64_t slot_bytes, int32_t P,
                 const int32_t *state_indices, int32_t batch, int32_t active_batch,
                 int32_t *err_flags, ssu_stream_t stream)
{
    return gather_scatter(pool, slot_bytes, P, const_cast<void *>(dense), state_indices, batch,
                          active_batch, 1, err_flags, stream);
}

int pool_clear_slot(void *pool, int64_t slot_bytes, int32_t P, int32_t slot,
                    ssu_stream_t stream)
{
    if (!pool)
        return SSU_ERR_NULL;
    if (slot_bytes < 0 || P < 0 || slot < -1 || slot >= P)
        return SSU_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (slot == -1)
        return ssu::launch_clear(pool, slot_bytes * P, s);
    return ssu::launch_clear(static_cast<uint8_t *>(pool) + slot * slot_bytes,
                                    slot_bytes, s);
}

int pool_copy_slot(void *dst_pool, int32_t dst_P, int32_t dst_slot, const void *src_pool,
                   int32_t src_P, int32_t src_slot, int64_t slot_bytes, ssu_stream_t stream)
{
    if (!dst_pool || !src_pool)
        return SSU_ERR_NULL;
    if (slot_bytes < 0 || dst_slot < 0 || dst_slot >= dst_P || src_slot < 0 ||
        src_slot >= src_P)
        return SSU_ERR_SHAPE;
    return ssu::launch_copy(static_cast<uint8_t *>(dst_pool) + dst_slot * slot_bytes,
                                   static_cast<const uint8_t *>(src_pool) + src_slot * slot_bytes,
                                   slot_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int ssu_check_state_indices(const int32_t *state_indices, int32_t batch,
                            int32_t active_batch, int32_t P, int32_t *err_flags,
                            ssu_stream_t stream)
{
    if (batch < 0 || active_batch < 0 || active_batch > batch || P < 0)
        return SSU_ERR_SHAPE;
    if (active_batch == 0)
        return SSU_OK;
    if (!state_indices || !err_flags)
        return SSU_ERR_NULL;
    return ssu::launch_check_indices(state_indices, active_batch, P, err_flags,
                                     reinterpret_cast<cudaStream_t>(stream));
}

#ifdef SSU_WAIT_TEST
// Test build only (libssu_waittest.so; declared in include/ssu_wait_test.h).
int ssu_test_wait_fault(int site, int block, int warp, int index, unsigned long long limit_ns)
{
    if (limit_ns == 0)
        return SSU_ERR_SHAPE;
    const ssu::WaitFault f{limit_ns, site, block, warp, index};
    const int bad = ssu::wait_fault_set_decode(f) | ssu::wait_fault_set_replay(f) |
                    ssu::wait_fault_set_conv(f) | ssu::wait_fault_set_gdn(f) |
                    ssu::wait_fault_set_prefill(f) | ssu::wait_fault_set_prefill_tc(f) |
                    ssu::wait_fault_set_ddtree(f);
    return bad ? SSU_ERR_CUDA : SSU_OK;
}
#endif

const char *ssu_status_string(int status)
{
    switch (status) {
    case SSU_OK: return "SSU_OK";
    case SSU_ERR_NULL: return "SSU_ERR_NULL: a required pointer is NULL or the stash is partial";
    case SSU_ERR_SHAPE: return "SSU_ERR_SHAPE: inconsistent sizes";
    case SSU_ERR_DTYPE: return "SSU_ERR_DTYPE: unknown dtype code";
    case SSU_ERR_UNSUPPORTED:
        return "SSU_ERR_UNSUPPORTED: dstate not in {8,16,32,64,128,256}, or a tree too large "
               "for shared memory";
    case SSU_ERR_CUDA: return "SSU_ERR_CUDA: kernel launch failed";
    case SSU_ERR_ALIGN: return "SSU_ERR_ALIGN: pool or slot stride not 16-byte aligned";
    default: return "unknown ssu_status";
    }
}

}  // extern "C"
