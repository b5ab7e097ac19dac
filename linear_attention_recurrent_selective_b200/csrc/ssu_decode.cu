// ssu_decode.cu -- single-token selective state update over a paged state pool.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdate:
//     new_state = state * exp(A * dt) + B * dt * x
//     output    = sum_n new_state[n] * C[n] + D * x, times silu(z) when z is given,
// with dt optionally passed through softplus(dt + dt_bias), and the padding contract of
// the FlashInfer page flashinfer.gdn_fused_decode_step (a negative state index is a
// padding row: no state access, output zero), checked in-kernel so that it holds under
// CUDA-graph replay.
//
// The step is a pure stream over the state pool: every state element is read once and
// written once (5 FLOP per 8 bytes of fp32 traffic), so the kernel is bound by HBM. It
// runs on the per-warp bulk-copy pipeline of ssu_stream.cuh and keeps every dependent
// load off the per-tile path:
//   * the per-unit scalars (dt_eff, exp(A dt_eff), D), the lane's B and C columns and the
//     unit's x and z are loaded once per unit, at addresses that do not depend on the
//     slot index, before the unit's first tile is waited for;
//   * a tile is read with conflict-free 16-byte shared loads, updated in registers and
//     written straight back to the pool with coalesced 16-byte global stores (each warp
//     instruction covers 512 contiguous bytes); the input term is formed as B * (dt * x),
//     the association the prefill and replay kernels use too, so fp32 states agree bit
//     for bit across the three forms;
//   * the dstate reductions of a tile's rows share one transposing butterfly of warp
//     shuffles inside each lane group (RPT - 1 + log2(LPR / RPT) shuffles for RPT rows
//     instead of RPT log2(LPR)); the per-row sums are collected in shared memory and the
//     unit's outputs (skip term and gate applied) are written with one coalesced store per
//     32 rows.
#include "ssu_stream.cuh"

namespace ssu {
namespace {

using namespace stream;

// Units of up to 8 tiles (32 KB): one unit is a whole head of the batch-256 workload,
// so its metadata is loaded once per 64 KB of traffic.
constexpr int kUT = 8;

struct DecodeRows : UnitsInOrder {
    const void *pool;
    const int32_t *idx;
    int32_t P;
    __device__ __forceinline__ UnitRes resolve(const LUnit &lu) const
    {
        return UnitRes{static_cast<const char *>(pool), idx ? idx[lu.un.b] : lu.un.b, 0};
    }
    __device__ __forceinline__ bool moves(const UnitRes &r) const
    {
        return r.slot >= 0 && r.slot < P;
    }
};

template <typename S, int N>
__global__ void __launch_bounds__(kWarps * 32)
ssu_decode_kernel(const DecodeArgs a, const int cph, const int nunits)
{
    using G = Geo<S, N, kUT>;
    using V = Vec16<S>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WarpViews w = warp_views(smem, warp);
    float *xs = w.f0;                           // unit x, [CR]
    float *ys = w.f1;                           // unit row sums, [CR]
    init_ring(w, lane);

    const int H = a.H, Dm = a.Dm, hpg = H / a.G;
    const int gw = blockIdx.x * kWarps + warp;
    const int nw = gridDim.x * kWarps;
    const DecodeRows rows{{}, a.state, a.idx, a.P};
    Producer<G, N, DecodeRows> prod;
    if (lane == 0) {
        prod.start(rows, gw, nw, nunits, cph, nunits, H, Dm);
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            prod.issue(rows, a.slot_stride, gw, nw, nunits, cph, nunits, H, Dm, w, s);
    }

    const int ln = lane % G::LPR, sub = lane / G::LPR;
    int c = 0;                                  // tiles consumed by this warp
    for (int u = gw; u < nunits; u += nw) {
        const Unit un = unit_at(u, cph, G::CR, H, Dm);
        const int tiles = (un.rows + G::RT - 1) / G::RT;
        const int64_t xrow = ((int64_t)un.b * H + un.h) * Dm + un.row0;

        // ---- per-unit inputs: addresses independent of the slot index
        const float dte = effective_dt(a.dt[(int64_t)un.b * H + un.h], a.dt_bias, un.h,
                                       a.softplus);
        const float dA = expf(a.A[un.h] * dte);
        const float Dh = a.D ? a.D[un.h] : 0.f;
        float Bn[G::E], Cn[G::E], xo[G::XR], zo[G::XR];
        {
            const int64_t bc = ((int64_t)un.b * a.G + un.h / hpg) * N;
#pragma unroll
            for (int v = 0; v < G::NV; ++v)
#pragma unroll
                for (int e = 0; e < G::VEC; ++e) {
                    Bn[v * G::VEC + e] = ld_f32(a.B, a.bc_dtype, bc + G::col(v, ln, e));
                    Cn[v * G::VEC + e] = ld_f32(a.C, a.bc_dtype, bc + G::col(v, ln, e));
                }
        }
#pragma unroll
        for (int m = 0; m < G::XR; ++m) {
            const int r = lane + 32 * m;
            const bool in = r < un.rows;
            xo[m] = in ? ld_f32(a.x, a.x_dtype, xrow + r) : 0.f;
            zo[m] = (in && a.z) ? ld_f32(a.z, a.x_dtype, xrow + r) : 0.f;
            if (r < G::CR)
                xs[r] = xo[m];
        }
        __syncwarp();

        int slot = -1;
        for (int j = 0; j < tiles; ++j, ++c) {
            if (!wait_tile(w, c, lane == 0 ? prod.issued : 0, lane, a.err))
                return;
            const int s = c % kStages;
            slot = w.ctl->slot[s];
            if (w.ctl->moves[s]) {
                const int rt = min(G::RT, un.rows - j * G::RT);
                const uint8_t *buf = w.ring + s * kTileBytes;
                S *dst = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride +
                         ((int64_t)un.h * Dm + un.row0 + j * G::RT) * N;
                uint4 raw[G::RPT][G::NV];
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
#pragma unroll
                    for (int v = 0; v < G::NV; ++v)
                        raw[i][v] = r < rt ? *reinterpret_cast<const uint4 *>(
                                                 buf + r * G::ROW_BYTES + (v * G::LPR + ln) * 16)
                                           : make_uint4(0, 0, 0, 0);
                }
                float acc[G::RPT];
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
                    const float dtx = r < rt ? dte * xs[j * G::RT + r] : 0.f;
                    acc[i] = 0.f;
#pragma unroll
                    for (int v = 0; v < G::NV; ++v) {
                        float f[G::VEC];
                        V::unpack(raw[i][v], f);
#pragma unroll
                        for (int e = 0; e < G::VEC; ++e) {
                            const float sn = fmaf(f[e], dA, Bn[v * G::VEC + e] * dtx);
                            f[e] = sn;
                            acc[i] = fmaf(sn, Cn[v * G::VEC + e], acc[i]);
                        }
                        if (r < rt)
                            *reinterpret_cast<uint4 *>(dst + (int64_t)r * N + G::col(v, ln, 0)) =
                                V::pack(f);
                    }
                }
                // the rows' dstate sums: one transposing butterfly for the whole tile
                if constexpr (G::RPT <= G::LPR) {
                    int i = 0;
                    bool wr = false;
                    const float y = row_sums<G::RPT, G::LPR>(acc, ln, i, wr);
                    const int r = i * G::RPW + sub;
                    if (wr && r < rt)
                        ys[j * G::RT + r] = y;
                } else {
#pragma unroll
                    for (int i0 = 0; i0 < G::RPT; ++i0) {
                        int i = i0;
                        bool wr = false;
                        const float y = row_sums<G::RPT, G::LPR>(acc, ln, i, wr);
                        const int r = i0 * G::RPW + sub;
                        if (wr && r < rt)
                            ys[j * G::RT + r] = y;
                    }
                }
            }
            __syncwarp();                        // every lane is done with buffer s
            if (lane == 0)
                prod.issue(rows, a.slot_stride, gw, nw, nunits, cph, nunits, H, Dm, w, s);
        }

        // ---- the unit's outputs, one coalesced store per 32 rows
        if (slot >= a.P) {                       // caller bug: skip the row and report it
            if (lane == 0 && un.h == 0 && un.row0 == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
        } else {
#pragma unroll
            for (int m = 0; m < G::XR; ++m) {
                const int r = lane + 32 * m;
                if (r < un.rows) {
                    float y = 0.f;               // padding row: zero
                    if (slot >= 0) {
                        y = ys[r] + Dh * xo[m];
                        if (a.z)
                            y *= silu_f(zo[m]);
                    }
                    st_f32(a.out, a.x_dtype, xrow + r, y);
                }
            }
        }
        __syncwarp();                            // xs / ys are reused by the next unit
    }
}

template <typename S, int N>
int launch_n(const DecodeArgs &a, cudaStream_t stream)
{
    using G = Geo<S, N, kUT>;
    const int64_t cph = (a.Dm + G::CR - 1) / G::CR;
    const int64_t nunits = (int64_t)a.active * a.H * cph;
    if (nunits == 0)
        return SSU_OK;
    if (nunits > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    const int grid = persistent_grid<ssu_decode_kernel<S, N>>(nunits);
    if (grid < 0)
        return SSU_ERR_CUDA;
    return launch_kernel(ssu_decode_kernel<S, N>, grid, kWarps * 32, kSmemBytes, stream, a,
                         (int)cph, (int)nunits);
}

template <typename S>
int launch_s(const DecodeArgs &a, cudaStream_t s)
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
SSU_WAIT_FAULT_SETTER(wait_fault_set_decode)
#endif

int launch_decode(const DecodeArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
