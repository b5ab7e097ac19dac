// ssu_replay.cu -- re-apply accepted speculative tokens to the committed state.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API), struct MambaReplayLayerInfo
// and invokeMambaReplayReconstructBatched: re-run the recurrence over the first
// acceptedLengths[b] tokens of the replay stash written by the prefill, in place on the
// committed state; a row whose accepted count is 0 is left untouched, and the loop is
// bounded by activeBatchSize. The stash carries the finished factors of each token:
//     state = state * dA[t] + B[t][n] * (dt[t] * U[t][d])
// (dA = exp(A * dt_eff), dt = dt_eff, U = x), the same association the decode and
// prefill kernels use, so fp32 results agree bit for bit with the decode steps.
//
// With acceptedNodeIds ([batch, maxAcceptLen], the tree-accept form written for the tree
// verify's stash), the t-th replayed token is stash entry acceptedNodeIds[b][t] and the
// accepted count is bounded by maxAcceptLen; a row with an id outside [0, T) among its
// accepted tokens is left untouched and flagged.
//
// invokeMambaReplayReconstructBatched also takes a device array of per-layer pointers
// (MambaReplayLayerInfo) and replays every layer in the same launch; units are numbered
// layer-major, so consecutive warps stream through one layer's pool at a time.
//
// With a handful of tokens per row the work is one read and one write of every touched
// state row, so the kernel runs on the per-warp bulk-copy pipeline of ssu_stream.cuh;
// rows with nothing accepted are never copied. The stash values are read through L1
// (B and dA/dt are shared by all tiles of a unit). Units are numbered over the live rows
// only (a valid slot, something accepted, node ids inside the stash): every CTA lists
// them in shared memory from the device lengths at launch, so each warp gets the same
// number of units that move state (within one) instead of a share of the batch in which
// rows with nothing accepted leave holes; batches of more than kLiveMax rows are
// numbered over all rows.
#include "ssu_stream.cuh"

namespace ssu {
namespace {

using namespace stream;

// Units of up to 4 tiles (16 KB). With units numbered over the live rows every warp
// gets an even share anyway, so the unit only has to be long enough to hide the loads
// of its first stashed tokens (measured on the batch-64 replay: 1 tile 0.072 ms, 2 tiles
// 0.064 ms, 4 tiles 0.061 ms, 8 tiles 0.073 ms). Both counts can be overridden at build
// time for tuning sweeps.
#ifndef SSU_REPLAY_UT
#define SSU_REPLAY_UT 4
#endif
#ifndef SSU_REPLAY_PRE
#define SSU_REPLAY_PRE 4
#endif
constexpr int kUT = SSU_REPLAY_UT;
constexpr int kPre = SSU_REPLAY_PRE;   // stashed tokens per unit held in registers
constexpr int kLiveMax = 1024;         // batches up to this size number units over live rows

// The lane's E columns of an fp32 [N] row, as 16-byte loads.
template <typename G>
__device__ __forceinline__ void load_cols(const float *row, int ln, float *dst)
{
#pragma unroll
    for (int v = 0; v < G::NV; ++v)
#pragma unroll
        for (int e4 = 0; e4 < G::VEC; e4 += 4) {
            const float4 q = *reinterpret_cast<const float4 *>(row + G::col(v, ln, e4));
            dst[v * G::VEC + e4] = q.x;
            dst[v * G::VEC + e4 + 1] = q.y;
            dst[v * G::VEC + e4 + 2] = q.z;
            dst[v * G::VEC + e4 + 3] = q.w;
        }
}

__device__ __forceinline__ bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15) == 0;
}

// The pointers of one layer (from the layer array, or the single-layer arguments).
struct LayerPtrs {
    char *state;
    const float *dA, *U, *B, *dt;
    bool ok;
};

__device__ __forceinline__ LayerPtrs layer_ptrs(const ReplayArgs &a, int layer)
{
    LayerPtrs L;
    if (a.layers) {
        const ssu_replay_layer &l = a.layers[layer];
        L.state = static_cast<char *>(l.state);
        L.dA = l.st_dA;
        L.U = l.st_U;
        L.B = l.st_B;
        L.dt = l.st_dt;
    } else {
        L.state = static_cast<char *>(a.state);
        L.dA = a.st_dA;
        L.U = a.st_U;
        L.B = a.st_B;
        L.dt = a.st_dt;
    }
    L.ok = L.state && L.dA && L.U && L.B && L.dt && aligned16(L.state) && aligned16(L.B);
    return L;
}

// Accepted count of a row whose accepted node ids are not all inside [0, T): the row is
// left untouched and SSU_FLAG_TREE reported.
constexpr int kBadNodes = -0x40000000;

// Stash entry of the t-th replayed token of row b: t itself, or acceptedNodeIds[b][t]
// (the tree-accept form); ids outside [0, T) map to entry 0 so that a prefetch never
// leaves the stash (such rows never use the values).
__device__ __forceinline__ int entry_of(const ReplayArgs &a, int b, int t)
{
    if (!a.nodes)
        return t;
    const int e = a.nodes[(int64_t)b * a.max_accept + t];
    return e >= 0 && e < a.T ? e : 0;
}

struct ReplayRows {
    const ReplayArgs *a;
    const int *live;     // live rows (shared memory), or NULL: units over all active rows
    __device__ __forceinline__ LUnit unit(int u, int upl, int cph, int CR, int H, int Dm) const
    {
        LUnit lu = lunit_at(u, upl, cph, CR, H, Dm);
        if (live)
            lu.un.b = live[lu.un.b];
        return lu;
    }
    __device__ __forceinline__ UnitRes resolve(const LUnit &lu) const
    {
        const LayerPtrs L = layer_ptrs(*a, lu.layer);
        const int b = lu.un.b;
        int acc = a->acc[b];
        if (a->nodes) {
            const int k = min(acc, a->max_accept);
            for (int t = 0; t < k; ++t) {
                const int e = a->nodes[(int64_t)b * a->max_accept + t];
                if (e < 0 || e >= a->T) {
                    acc = kBadNodes;
                    break;
                }
            }
        }
        return UnitRes{L.ok ? L.state : nullptr, a->idx ? a->idx[b] : b, acc};
    }
    __device__ __forceinline__ bool moves(const UnitRes &r) const
    {
        return r.pool != nullptr && r.slot >= 0 && r.slot < a->P &&
               min(r.extra, a->max_accept) > 0;
    }
};

// The rows whose state moves, in row order, into list[]; returns their count. All
// threads of the CTA take part. CTA 0 also reports every row's caller bugs (index >= P,
// node id outside the stash, accepted length out of range) and every layer whose pointers
// are unusable, since units of rows that do not move are never visited.
__device__ int list_live_rows(const ReplayArgs &a, int *list, int *wcount)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reporter = blockIdx.x == 0 && a.err;
    if (reporter)
        for (int l = tid; l < a.num_layers; l += kWarps * 32)
            if (!layer_ptrs(a, l).ok)
                atomicOr(a.err, SSU_FLAG_LAYER);
    int total = 0;
    for (int b0 = 0; b0 < a.active; b0 += kWarps * 32) {
        const int b = b0 + tid;
        bool live = false;
        if (b < a.active) {
            const int slot = a.idx ? a.idx[b] : b;
            const int acc = a.acc[b];
            const int k = min(acc, a.max_accept);
            bool bad = false;
            if (a.nodes && slot >= 0 && slot < a.P)
                for (int t = 0; t < k && !bad; ++t) {
                    const int e = a.nodes[(int64_t)b * a.max_accept + t];
                    bad = e < 0 || e >= a.T;
                }
            live = slot >= 0 && slot < a.P && k > 0 && !bad;
            if (reporter) {
                if (slot >= a.P)
                    atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
                else if (slot >= 0 && bad)
                    atomicOr(a.err, SSU_FLAG_TREE);
                else if (slot >= 0 && acc > a.max_accept)
                    atomicOr(a.err, SSU_FLAG_ACCEPTED_RANGE);
                else if (slot >= 0 && acc < 0)
                    atomicOr(a.err, SSU_FLAG_NEGATIVE_LENGTH);
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, live);
        if (lane == 0)
            wcount[warp] = __popc(m);
        __syncthreads();
        int before = total;
        for (int v = 0; v < kWarps; ++v) {
            if (v < warp)
                before += wcount[v];
            total += wcount[v];
        }
        if (live)
            list[before + __popc(m & ((1u << lane) - 1u))] = b;
        __syncthreads();                 // wcount is reused by the next chunk of rows
    }
    return total;
}

template <typename S, int N>
__global__ void __launch_bounds__(kWarps * 32)
ssu_replay_kernel(const __grid_constant__ ReplayArgs a, const int cph)
{
    using G = Geo<S, N, kUT>;
    using V = Vec16<S>;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_live[kLiveMax];
    __shared__ int s_wcount[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WarpViews w = warp_views(smem, warp);
    init_ring(w, lane);

    const int H = a.H, Dm = a.Dm, T = a.T, hpg = H / a.G;
    const int gw = blockIdx.x * kWarps + warp;
    const int nw = gridDim.x * kWarps;
    const bool listed = a.active <= kLiveMax;
    const int nrows = listed ? list_live_rows(a, s_live, s_wcount) : a.active;
    const int upl = nrows * H * cph;     // units per layer (the host checked the full count)
    const int nunits = upl * a.num_layers;
    const ReplayRows rows{&a, listed ? s_live : nullptr};
    Producer<G, N, ReplayRows> prod;
    if (lane == 0) {
        prod.start(rows, gw, nw, upl, cph, nunits, H, Dm);
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            prod.issue(rows, a.slot_stride, gw, nw, upl, cph, nunits, H, Dm, w, s);
    }

    const int ln = lane % G::LPR, sub = lane / G::LPR;
    int c = 0;
    for (int u = gw; u < nunits; u += nw) {
        const LUnit lu = rows.unit(u, upl, cph, G::CR, H, Dm);
        const Unit &un = lu.un;
        const int tiles = (un.rows + G::RT - 1) / G::RT;
        const int g = un.h / hpg;
        const LayerPtrs L = layer_ptrs(a, lu.layer);

        // ---- the unit's first kPre stashed tokens, loaded before its first tile is
        // waited for (addresses stay inside the stash whatever the accepted count is)
        float pdA[kPre], pdt[kPre], pB[kPre][G::E], pU[kPre][G::XR];
#pragma unroll
        for (int t = 0; t < kPre; ++t) {
            if (t < a.max_accept && L.ok) {
                const int64_t bt = (int64_t)un.b * T + entry_of(a, un.b, t);
                pdA[t] = L.dA[bt * H + un.h];
                pdt[t] = L.dt[bt * H + un.h];
                load_cols<G>(L.B + (bt * a.G + g) * N, ln, pB[t]);
                const float *Ut = L.U + (bt * H + un.h) * Dm + un.row0;
#pragma unroll
                for (int m = 0; m < G::XR; ++m)
                    pU[t][m] = lane + 32 * m < un.rows ? Ut[lane + 32 * m] : 0.f;
            }
        }

        int2 r2 = make_int2(-1, 0);
        for (int j = 0; j < tiles; ++j, ++c) {
            if (!wait_tile(w, c, lane == 0 ? prod.issued : 0, lane, a.err))
                return;
            const int s = c % kStages;
            r2 = make_int2(w.ctl->slot[s], w.ctl->extra[s]);
            if (w.ctl->moves[s]) {
                const int k = min(r2.y, a.max_accept);
                const int rt = min(G::RT, un.rows - j * G::RT);
                const int r0 = un.row0 + j * G::RT;
                const uint8_t *buf = w.ring + s * kTileBytes;
                float st[G::RPT][G::E];
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
#pragma unroll
                    for (int v = 0; v < G::NV; ++v) {
                        const uint4 q = r < rt ? *reinterpret_cast<const uint4 *>(
                                                     buf + r * G::ROW_BYTES + (v * G::LPR + ln) * 16)
                                               : make_uint4(0, 0, 0, 0);
                        V::unpack(q, &st[i][v * G::VEC]);
                    }
                }
                // tokens held in registers; U of unit row q lives in lane q % 32, slot
                // q / 32, and the rows of one warp access never straddle 32, so the slot
                // index is warp-uniform
#pragma unroll
                for (int t = 0; t < kPre; ++t) {
                    if (t < k) {
#pragma unroll
                        for (int i = 0; i < G::RPT; ++i) {
                            const int q = j * G::RT + i * G::RPW + sub;
                            float um = pU[t][0];
#pragma unroll
                            for (int m = 1; m < G::XR; ++m)
                                um = (q >> 5) == m ? pU[t][m] : um;
                            const float uq = __shfl_sync(0xffffffffu, um, q & 31);
                            const float dtu = pdt[t] * uq;
#pragma unroll
                            for (int e = 0; e < G::E; ++e)
                                st[i][e] = fmaf(st[i][e], pdA[t], pB[t][e] * dtu);
                        }
                    }
                }
                // longer acceptances: the remaining tokens straight from the stash
                for (int t = kPre; t < k; ++t) {
                    const int64_t bt = (int64_t)un.b * T + entry_of(a, un.b, t);
                    const float dA = L.dA[bt * H + un.h];
                    const float dte = L.dt[bt * H + un.h];
                    const float *Ut = L.U + (bt * H + un.h) * Dm + r0;
                    float Bn[G::E];
                    load_cols<G>(L.B + (bt * a.G + g) * N, ln, Bn);
#pragma unroll
                    for (int i = 0; i < G::RPT; ++i) {
                        const int r = i * G::RPW + sub;
                        const float dtu = r < rt ? dte * Ut[r] : 0.f;
#pragma unroll
                        for (int e = 0; e < G::E; ++e)
                            st[i][e] = fmaf(st[i][e], dA, Bn[e] * dtu);
                    }
                }
                S *dst = reinterpret_cast<S *>(L.state) + (int64_t)r2.x * a.slot_stride +
                         ((int64_t)un.h * Dm + r0) * N;
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
                    if (r < rt) {
#pragma unroll
                        for (int v = 0; v < G::NV; ++v)
                            *reinterpret_cast<uint4 *>(dst + (int64_t)r * N + G::col(v, ln, 0)) =
                                V::pack(&st[i][v * G::VEC]);
                    }
                }
            }
            __syncwarp();                        // every lane is done with buffer s
            if (lane == 0)
                prod.issue(rows, a.slot_stride, gw, nw, upl, cph, nunits, H, Dm, w, s);
        }
        // ---- caller bugs, reported once per row (or layer): clamped or skipped (listed
        // launches reported them while listing the rows)
        if (!listed && lane == 0 && un.h == 0 && un.row0 == 0 && a.err) {
            if (!L.ok && un.b == 0)
                atomicOr(a.err, SSU_FLAG_LAYER);
            if (lu.layer == 0) {
                if (r2.x >= a.P)
                    atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
                else if (r2.x >= 0 && r2.y == kBadNodes)
                    atomicOr(a.err, SSU_FLAG_TREE);
                else if (r2.x >= 0 && r2.y > a.max_accept)
                    atomicOr(a.err, SSU_FLAG_ACCEPTED_RANGE);
                else if (r2.x >= 0 && r2.y < 0)
                    atomicOr(a.err, SSU_FLAG_NEGATIVE_LENGTH);
            }
        }
    }
}

template <typename S, int N>
int launch_n(const ReplayArgs &a, cudaStream_t stream)
{
    using G = Geo<S, N, kUT>;
    const int64_t cph = (a.Dm + G::CR - 1) / G::CR;
    const int64_t upl = (int64_t)a.active * a.H * cph;
    const int64_t nunits = upl * a.num_layers;
    if (nunits == 0 || a.T == 0)
        return SSU_OK;
    if (nunits > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    // sized for every active row; a listed launch may have fewer units that move
    const int grid = persistent_grid<ssu_replay_kernel<S, N>>(nunits);
    if (grid < 0)
        return SSU_ERR_CUDA;
    return launch_kernel(ssu_replay_kernel<S, N>, grid, kWarps * 32, kSmemBytes, stream, a,
                         (int)cph);
}

template <typename S>
int launch_s(const ReplayArgs &a, cudaStream_t s)
{
    switch (a.N) {
    case 8: return launch_n<S, 8>(a, s);
    case 16: return launch_n<S, 16>(a, s);
    case 32: return launch_n<S, 32>(a, s);
    case 64: return launch_n<S, 64>(a, s);
    case 128: return launch_n<S, 128>(a, s);
    case 256: return launch_n<S, 256>(a, s);
    default: return SSU_ERR_UNSUPPORTED;
    }
}

}  // namespace

#ifdef SSU_WAIT_TEST
SSU_WAIT_FAULT_SETTER(wait_fault_set_replay)
#endif

int launch_replay(const ReplayArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
