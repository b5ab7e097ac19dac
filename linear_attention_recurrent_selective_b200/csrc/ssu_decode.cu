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
// written once (8 FLOP per 4 bytes of fp32 state), so the kernel is HBM-bound. Design:
//   * one CTA (8 warps) per (row b, head h, dim tile); consecutive CTAs walk the heads of
//     one slot, i.e. contiguous memory;
//   * a row of N state elements is covered by LPR lanes with 16-byte accesses, so each
//     warp instruction moves 512 contiguous bytes; each thread keeps RPT rows in flight
//     (all loads are issued before any arithmetic) to hold enough bytes in flight per SM;
//   * B and C for the lane's state columns and the per-(b,h) decay live in registers;
//     the input term is formed as B * (dt * x), the association the prefill and replay
//     kernels use too, so fp32 states agree bit for bit across the three forms;
//   * the dstate reduction is a butterfly of warp shuffles inside each lane group;
//   * the new state is stored back to the same addresses with 16-byte stores.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kDecodeWarps = 8;

template <typename S, int N, int RPT>
__global__ void __launch_bounds__(kDecodeWarps * 32)
ssu_decode_kernel(const DecodeArgs a)
{
    using V = Vec16<S>;
    constexpr int VEC = V::kElems;                       // state elements per 16 bytes
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;  // lanes per state row
    constexpr int E = N / LPR;                           // elements per lane and row
    constexpr int NV = E / VEC;                          // 16-byte vectors per lane and row
    constexpr int RPW = 32 / LPR;                        // rows per warp instruction
    constexpr int RPP = kDecodeWarps * RPW;              // rows per CTA pass
    constexpr int RT = RPP * RPT;                        // rows per CTA (dim tile)

    const int H = a.H, Dm = a.Dm;
    const int dtiles = (Dm + RT - 1) / RT;
    int unit = blockIdx.x;
    const int dtile = unit % dtiles;
    unit /= dtiles;
    const int h = unit % H;
    const int b = unit / H;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ln = lane % LPR;
    const int rbase = dtile * RT + warp * RPW + lane / LPR;
    const int64_t xrow = ((int64_t)b * H + h) * Dm;

    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0) {                       // padding row: output zero, state untouched
        if (ln == 0) {
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int r = rbase + i * RPP;
                if (r < Dm)
                    st_f32(a.out, a.x_dtype, xrow + r, 0.f);
            }
        }
        return;
    }
    if (slot >= a.P) {                    // caller bug: skip the row and report it
        if (threadIdx.x == 0 && dtile == 0 && h == 0 && a.err)
            atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
        return;
    }

    // ---- issue every state load of this thread first
    S *base = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride + (int64_t)h * Dm * N;
    uint4 raw[RPT][NV];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rbase + i * RPP;
        const uint4 *rp = reinterpret_cast<const uint4 *>(base + (int64_t)r * N);
#pragma unroll
        for (int v = 0; v < NV; ++v)
            raw[i][v] = r < Dm ? rp[v * LPR + ln] : make_uint4(0, 0, 0, 0);
    }

    // ---- per-(b, h) scalars and the lane's columns of B and C
    const int g = h / (H / a.G);
    const float dte = effective_dt(a.dt[(int64_t)b * H + h], a.dt_bias, h, a.softplus);
    const float dA = expf(a.A[h] * dte);
    const float Dh = a.D ? a.D[h] : 0.f;
    const int64_t bc = ((int64_t)b * a.G + g) * N;
    float Bn[E], Cn[E];
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const int n = (v * LPR + ln) * VEC + k;
            Bn[v * VEC + k] = ld_f32(a.B, a.bc_dtype, bc + n);
            Cn[v * VEC + k] = ld_f32(a.C, a.bc_dtype, bc + n);
        }
    float xv[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rbase + i * RPP;
        xv[i] = r < Dm ? ld_f32(a.x, a.x_dtype, xrow + r) : 0.f;
    }

    // ---- update, reduce, store
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rbase + i * RPP;
        const float dtx = dte * xv[i];
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            float f[VEC];
            V::unpack(raw[i][v], f);
#pragma unroll
            for (int k = 0; k < VEC; ++k) {
                const float s = fmaf(f[k], dA, Bn[v * VEC + k] * dtx);
                f[k] = s;
                acc = fmaf(s, Cn[v * VEC + k], acc);
            }
            raw[i][v] = V::pack(f);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
            acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (r < Dm) {
            uint4 *rp = reinterpret_cast<uint4 *>(base + (int64_t)r * N);
#pragma unroll
            for (int v = 0; v < NV; ++v)
                rp[v * LPR + ln] = raw[i][v];
            if (ln == 0) {
                float y = acc + Dh * xv[i];
                if (a.z)
                    y *= silu_f(ld_f32(a.z, a.x_dtype, xrow + r));
                st_f32(a.out, a.x_dtype, xrow + r, y);
            }
        }
    }
}

template <typename S, int N, int RPT>
int launch_rpt(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int VEC = Vec16<S>::kElems;
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;
    constexpr int RT = kDecodeWarps * (32 / LPR) * RPT;
    const int64_t dtiles = (a.Dm + RT - 1) / RT;
    const int64_t grid = (int64_t)a.active * a.H * dtiles;
    if (grid == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    ssu_decode_kernel<S, N, RPT><<<(unsigned)grid, kDecodeWarps * 32, 0, s>>>(a);
    return SSU_OK;
}

// Rows per thread: as many as the dim extent fills (up to 8), so that small dims do not
// leave most of the CTA idle and large dims keep 128 bytes in flight per thread.
template <typename S, int N>
int launch_n(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int VEC = Vec16<S>::kElems;
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;
    constexpr int RPP = kDecodeWarps * (32 / LPR);
    if (a.Dm >= 8 * RPP)
        return launch_rpt<S, N, 8>(a, s);
    if (a.Dm >= 4 * RPP)
        return launch_rpt<S, N, 4>(a, s);
    if (a.Dm >= 2 * RPP)
        return launch_rpt<S, N, 2>(a, s);
    return launch_rpt<S, N, 1>(a, s);
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
