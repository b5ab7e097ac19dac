// ssu_replay.cu -- re-apply accepted speculative tokens to the committed state.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API), struct MambaReplayLayerInfo
// and invokeMambaReplayReconstructBatched: re-run the recurrence over the first
// acceptedLengths[b] tokens of the replay stash written by the prefill, in place on the
// committed state; a row whose accepted count is 0 is left untouched, and the loop is
// bounded by activeBatchSize.
//
// With at most a handful of tokens per row the work is dominated by one read and one
// write of each touched state row, so the kernel has the decode kernel's streaming
// layout (16-byte accesses, several rows in flight per thread, loads issued first) and
// keeps the state in registers while the stashed tokens are applied.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kReplayWarps = 8;

template <typename S, int N, int RPT>
__global__ void __launch_bounds__(kReplayWarps * 32)
ssu_replay_kernel(const ReplayArgs a)
{
    using V = Vec16<S>;
    constexpr int VEC = V::kElems;
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;
    constexpr int E = N / LPR;
    constexpr int NV = E / VEC;
    constexpr int RPW = 32 / LPR;
    constexpr int RPP = kReplayWarps * RPW;
    constexpr int RT = RPP * RPT;

    const int H = a.H, Dm = a.Dm, T = a.T;
    const int dtiles = (Dm + RT - 1) / RT;
    int unit = blockIdx.x;
    const int dtile = unit % dtiles;
    unit /= dtiles;
    const int h = unit % H;
    const int b = unit / H;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ln = lane % LPR;
    const int rbase = dtile * RT + warp * RPW + lane / LPR;
    const bool reporter = threadIdx.x == 0 && dtile == 0 && h == 0;

    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0)
        return;                           // padding row: nothing to commit
    if (slot >= a.P) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
        return;
    }
    int k = a.acc[b];
    if (k > T) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_ACCEPTED_RANGE);
        k = T;
    }
    if (k < 0) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_NEGATIVE_LENGTH);
        k = 0;
    }
    if (k == 0)
        return;                           // nothing accepted: row untouched

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
    float s[RPT][E];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int v = 0; v < NV; ++v)
            V::unpack(raw[i][v], &s[i][v * VEC]);

    const int g = h / (H / a.G);
    for (int t = 0; t < k; ++t) {
        const int64_t bt = (int64_t)b * T + t;
        const float dA = a.st_dA[bt * H + h];
        const float dte = a.st_dt[bt * H + h];
        const float *Bt = a.st_B + (bt * a.G + g) * N;
        float Bn[E];
#pragma unroll
        for (int v = 0; v < NV; ++v)
#pragma unroll
            for (int k4 = 0; k4 < VEC; k4 += 4) {
                const float4 q = *reinterpret_cast<const float4 *>(Bt + (v * LPR + ln) * VEC + k4);
                Bn[v * VEC + k4] = q.x;
                Bn[v * VEC + k4 + 1] = q.y;
                Bn[v * VEC + k4 + 2] = q.z;
                Bn[v * VEC + k4 + 3] = q.w;
            }
        const float *Ut = a.st_U + (bt * H + h) * Dm;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rbase + i * RPP;
            const float dtu = r < Dm ? dte * Ut[r] : 0.f;
#pragma unroll
            for (int j = 0; j < E; ++j)
                s[i][j] = fmaf(s[i][j], dA, Bn[j] * dtu);
        }
    }

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rbase + i * RPP;
        if (r < Dm) {
            uint4 *rp = reinterpret_cast<uint4 *>(base + (int64_t)r * N);
#pragma unroll
            for (int v = 0; v < NV; ++v)
                rp[v * LPR + ln] = V::pack(&s[i][v * VEC]);
        }
    }
}

template <typename S, int N, int RPT>
int launch_rpt(const ReplayArgs &a, cudaStream_t s)
{
    constexpr int VEC = Vec16<S>::kElems;
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;
    constexpr int RT = kReplayWarps * (32 / LPR) * RPT;
    const int64_t dtiles = (a.Dm + RT - 1) / RT;
    const int64_t grid = (int64_t)a.active * a.H * dtiles;
    if (grid == 0 || a.T == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    ssu_replay_kernel<S, N, RPT><<<(unsigned)grid, kReplayWarps * 32, 0, s>>>(a);
    return SSU_OK;
}

template <typename S, int N>
int launch_n(const ReplayArgs &a, cudaStream_t s)
{
    constexpr int VEC = Vec16<S>::kElems;
    constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;
    constexpr int RPP = kReplayWarps * (32 / LPR);
    if (a.Dm >= 8 * RPP)
        return launch_rpt<S, N, 8>(a, s);
    if (a.Dm >= 4 * RPP)
        return launch_rpt<S, N, 4>(a, s);
    if (a.Dm >= 2 * RPP)
        return launch_rpt<S, N, 2>(a, s);
    return launch_rpt<S, N, 1>(a, s);
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
