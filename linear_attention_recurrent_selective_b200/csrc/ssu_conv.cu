// ssu_conv.cu -- the causal conv1d update of the xBC channels fused with the decode.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API): a slot carries a convolution
// state beside the recurrent state (struct MambaStateLayerInfo, convState), and the
// decode of invokeSelectiveStateUpdate consumes x, B and C. The causal conv1d update is
// the one of the FlashInfer page flashinfer.gdn_fused_decode_step: depthwise weights
// [conv_dim, width], bias [conv_dim], a conv pool of the last width-1 raw inputs of every
// channel, updated in place and indexed by the same state index as the recurrent pool,
// padding rows (negative index) touching neither pool. Per channel c of a live row:
//     window = (taps of the slot, oldest first, then the new raw input xbc[b, c])
//     v[c]   = sum_k w[c, k] window[k] + bias[c], then v * sigmoid(v)
//     taps   = window[1 ..]
// and x = v[0, H*Dm), B = v[H*Dm, +G*N), C = v[H*Dm+G*N, +G*N) feed the decode.
//
// The conv outputs are never stored: every unit of the decode pipeline (up to 128 dim
// rows of one head, see ssu_stream.cuh) computes the conv outputs it needs -- its x rows
// and its group's B and C columns -- in fp32 from the old taps, then streams its state
// tiles as the decode kernel does. Each warp takes a contiguous range of units, so that
// consecutive units share their batch row: the row's slot index and the lane's B and C
// conv outputs are computed once per (row, group) and reused. A unit owns its x channels
// and advances their windows itself. B and C channels are shared by all heads of a group,
// so no unit may shift their taps while another might still read them; their shift runs
// as a second, short launch on the same stream after the first has finished (2*G*N
// channels per row).
#include "ssu_stream.cuh"

namespace ssu {
namespace {

using namespace stream;

constexpr int kUT = 8;   // units of up to 8 tiles, as in the decode
constexpr int kMaxConvWidth = 16;   // the widest window ssu_conv_decode accepts

struct ConvRows : UnitsInOrder {
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

// Conv output of channel ch of batch row b (slot's taps at tap0 = slot * cslot). With
// `shift`, the caller owns the channel and its window is advanced here as well: in
// ascending order tap k takes tap k+1 (read before it is overwritten), the last tap the
// new input.
__device__ __forceinline__ float conv_out(const ConvArgs &c, int dtype, int64_t xrow,
                                          int64_t tap0, int64_t ch, bool shift = false)
{
    if (c.width <= 4) {
        // windows of up to 4 (the common case): every input loaded at once into registers
        // (one round trip instead of one per dependent step), the taps reused by the shift
        const int W = c.width;
        const int64_t w0 = ch * W, t0 = tap0 + ch * c.cc;
        uint32_t tap[3], wt[4];
#pragma unroll
        for (int k = 0; k < 3; ++k)
            tap[k] = k + 1 < W ? ld_bits(c.cstate, dtype, t0 + k * c.ck) : 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            wt[k] = k < W ? ld_bits(c.w, dtype, w0 + k) : 0u;
        const uint32_t xin = ld_bits(c.xbc, dtype, xrow + ch);
        float acc = c.bias ? ld_f32(c.bias, dtype, ch) : 0.f;
#pragma unroll
        for (int k = 0; k < 3; ++k)
            if (k + 1 < W)
                acc = fmaf(bits_f32(wt[k], dtype), bits_f32(tap[k], dtype), acc);
        const uint32_t wl = W == 4 ? wt[3] : W == 3 ? wt[2] : W == 2 ? wt[1] : wt[0];
        acc = fmaf(bits_f32(wl, dtype), bits_f32(xin, dtype), acc);
        if (shift) {
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                if (k + 1 < W) {
                    const uint32_t v = k + 2 < W ? tap[k + 1 < 3 ? k + 1 : 2] : xin;
                    if (dtype == SSU_F32)
                        static_cast<uint32_t *>(c.cstate)[t0 + k * c.ck] = v;
                    else
                        static_cast<uint16_t *>(c.cstate)[t0 + k * c.ck] = static_cast<uint16_t>(v);
                }
            }
        }
        return c.silu ? silu_f(acc) : acc;
    }
    float acc = c.bias ? ld_f32(c.bias, dtype, ch) : 0.f;
    const int64_t w0 = ch * c.width;
    const int64_t t0 = tap0 + ch * c.cc;
#pragma unroll 4
    for (int k = 0; k + 1 < c.width; ++k)
        acc = fmaf(ld_f32(c.w, dtype, w0 + k), ld_f32(c.cstate, dtype, t0 + k * c.ck), acc);
    const uint32_t xin = ld_bits(c.xbc, dtype, xrow + ch);
    acc = fmaf(ld_f32(c.w, dtype, w0 + c.width - 1), bits_f32(xin, dtype), acc);
    if (shift) {
        for (int k = 0; k + 1 < c.width; ++k) {
            const uint32_t v = k + 2 < c.width ? ld_bits(c.cstate, dtype, t0 + (k + 1) * c.ck)
                                               : xin;
            if (dtype == SSU_F32)
                static_cast<uint32_t *>(c.cstate)[t0 + k * c.ck] = v;
            else
                static_cast<uint16_t *>(c.cstate)[t0 + k * c.ck] = static_cast<uint16_t>(v);
        }
    }
    return c.silu ? silu_f(acc) : acc;
}

template <typename S, int N>
__global__ void __launch_bounds__(kWarps * 32)
ssu_conv_decode_kernel(const __grid_constant__ ConvArgs ca, const int cph, const int nunits)
{
    using G = Geo<S, N, kUT>;
    using V = Vec16<S>;
    extern __shared__ __align__(128) uint8_t smem[];
    const DecodeArgs &a = ca.d;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WarpViews w = warp_views(smem, warp);
    float *xs = w.f0;                           // unit x (conv outputs), [CR]
    float *ys = w.f1;                           // unit row sums, [CR]
    init_ring(w, lane);
    grid_launch_dependents();                   // the B/C window shift may start loading

    const int H = a.H, Dm = a.Dm, hpg = H / a.G;
    const int64_t cd = (int64_t)H * Dm + 2 * (int64_t)a.G * N;   // conv channels
    // this warp's contiguous range of units [first, last): the producer walks it with a
    // stride of 1 (its "unit count" is the range end)
    const int gw = blockIdx.x * kWarps + warp;
    const int nw = gridDim.x * kWarps;
    const int first = (int)((int64_t)nunits * gw / nw);
    const int last = (int)((int64_t)nunits * (gw + 1) / nw);
    const ConvRows rows{{}, a.state, a.idx, a.P};
    Producer<G, N, ConvRows> prod;
    if (lane == 0) {
        prod.start(rows, first, 1, nunits, cph, last, H, Dm);
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            prod.issue(rows, a.slot_stride, first, 1, nunits, cph, last, H, Dm, w, s);
    }

    const int ln = lane % G::LPR, sub = lane / G::LPR;
    int c = 0;                                  // tiles consumed by this warp
    int cur_b = -1, cur_g = -1, slot0 = -1;
    float Bn[G::E], Cn[G::E];
    for (int u = first; u < last; ++u) {
        const Unit un = unit_at(u, cph, G::CR, H, Dm);
        const int tiles = (un.rows + G::RT - 1) / G::RT;
        const int64_t orow = ((int64_t)un.b * H + un.h) * Dm + un.row0;
        if (un.b != cur_b)
            slot0 = a.idx ? a.idx[un.b] : un.b;
        const bool live = slot0 >= 0 && slot0 < a.P;
        const int64_t tap0 = (int64_t)(live ? slot0 : 0) * ca.cslot;
        const int64_t xb = (int64_t)un.b * cd;

        // ---- per-unit inputs: dt, the conv outputs of the unit's x rows and of the
        // lane's B and C columns, z
        const float dte = effective_dt(a.dt[(int64_t)un.b * H + un.h], a.dt_bias, un.h,
                                       a.softplus);
        const float dA = expf(a.A[un.h] * dte);
        const float Dh = a.D ? a.D[un.h] : 0.f;
        float xo[G::XR], zo[G::XR];
        if (un.b != cur_b || un.h / hpg != cur_g) {     // B and C conv of a new (row, group)
            cur_b = un.b;
            cur_g = un.h / hpg;
            const int64_t bch = (int64_t)H * Dm + (int64_t)(un.h / hpg) * N;
            const int64_t cch = bch + (int64_t)a.G * N;
#pragma unroll
            for (int v = 0; v < G::NV; ++v)
#pragma unroll
                for (int e = 0; e < G::VEC; ++e) {
                    const int n = G::col(v, ln, e);
                    Bn[v * G::VEC + e] = live ? conv_out(ca, a.x_dtype, xb, tap0, bch + n) : 0.f;
                    Cn[v * G::VEC + e] = live ? conv_out(ca, a.x_dtype, xb, tap0, cch + n) : 0.f;
                }
        }
#pragma unroll
        for (int m = 0; m < G::XR; ++m) {
            const int r = lane + 32 * m;
            const bool in = r < un.rows;
            xo[m] = (in && live) ? conv_out(ca, a.x_dtype, xb, tap0,
                                            (int64_t)un.h * Dm + un.row0 + r, true)
                                 : 0.f;
            zo[m] = (in && a.z) ? ld_f32(a.z, a.x_dtype, orow + r) : 0.f;
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
                if constexpr (G::RPT <= G::LPR) {         // one transposing butterfly
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
                prod.issue(rows, a.slot_stride, first, 1, nunits, cph, last, H, Dm, w, s);
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
                    st_f32(a.out, a.x_dtype, orow + r, y);
                }
            }
        }
        __syncwarp();                            // xs / ys are reused by the next unit
    }
}

// Shift the conv windows of the B and C channels of every live row by one raw input (the
// x channels were shifted by their owning units in the fused decode). Launched as a
// programmatic dependent of the fused decode, which never writes these taps: the old taps
// and the new input are loaded while the decode runs, and the stores wait until it has
// completed, so that no unit can still be reading a tap.
__global__ void __launch_bounds__(256)
conv_shift_kernel(const __grid_constant__ ConvArgs ca, const int64_t cd, const int64_t ch0)
{
    // block (x, y): row y, B/C channels ch0 + 256 x + threadIdx.x
    const DecodeArgs &a = ca.d;
    const int64_t b = blockIdx.y;
    const int64_t ch = ch0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int slot = a.idx ? a.idx[b] : (int)b;
    if (ch >= cd || slot < 0 || slot >= a.P)
        return;
    const int64_t t0 = (int64_t)slot * ca.cslot + ch * ca.cc;
    const int W = ca.width, dty = a.x_dtype;
    // every old tap first (registers: the loops are unrolled to the widest window), then
    // every store: tap k takes tap k+1, the last tap the new input
    uint32_t tap[kMaxConvWidth - 1];
#pragma unroll
    for (int k = 0; k < kMaxConvWidth - 1; ++k)
        tap[k] = k + 1 < W ? ld_bits(ca.cstate, dty, t0 + k * ca.ck) : 0u;
    const uint32_t xin = ld_bits(ca.xbc, dty, b * cd + ch);
    grid_dependency_wait();
#pragma unroll
    for (int k = 0; k < kMaxConvWidth - 1; ++k) {
        if (k + 1 < W) {
            const uint32_t v = k + 2 < W ? tap[k + 1 < kMaxConvWidth - 1 ? k + 1 : 0] : xin;
            if (dty == SSU_F32)
                static_cast<uint32_t *>(ca.cstate)[t0 + k * ca.ck] = v;
            else
                static_cast<uint16_t *>(ca.cstate)[t0 + k * ca.ck] = static_cast<uint16_t>(v);
        }
    }
}

template <typename S, int N>
int launch_n(const ConvArgs &ca, cudaStream_t stream)
{
    using G = Geo<S, N, kUT>;
    const DecodeArgs &a = ca.d;
    const int64_t cph = (a.Dm + G::CR - 1) / G::CR;
    const int64_t nunits = (int64_t)a.active * a.H * cph;
    if (nunits == 0)
        return SSU_OK;
    if (nunits > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    const int grid = persistent_grid<ssu_conv_decode_kernel<S, N>>(nunits);
    if (grid < 0)
        return SSU_ERR_CUDA;
    int rc = launch_kernel(ssu_conv_decode_kernel<S, N>, grid, kWarps * 32, kSmemBytes, stream,
                           ca, (int)cph, (int)nunits);
    if (rc == SSU_OK && ca.width > 1) {
        const int64_t ch0 = (int64_t)a.H * a.Dm;
        const int64_t cd = ch0 + 2 * (int64_t)a.G * N;
        const dim3 blocks((unsigned)((cd - ch0 + 255) / 256), (unsigned)a.active);
        rc = launch_kernel_dependent(conv_shift_kernel, blocks, 256, 0, stream, ca, cd, ch0);
    }
    return rc;
}

template <typename S>
int launch_s(const ConvArgs &a, cudaStream_t s)
{
    switch (a.d.N) {
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
SSU_WAIT_FAULT_SETTER(wait_fault_set_conv)
#endif

int launch_conv_decode(const ConvArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
