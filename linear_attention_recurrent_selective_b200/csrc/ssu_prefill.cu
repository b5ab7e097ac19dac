// ssu_prefill.cu -- multi-token selective state update (seq_len > 1) in one launch.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdatePrefill: the decode recurrence over the tokens
// t < contextLengths[b] of a [batch, seq_len, ...] input. With the replay stash
// (replayDA, replayU, replayB, replayDT) the committed state stays read-only and the
// per-token replay inputs are written instead.
//
// The state of one (row, head, dim tile) stays in registers for the whole token loop,
// so the pool is read once and (without the stash) written once. Per token every state
// element costs a multiply and two FMAs plus a short shuffle reduction: the kernel is
// bound by FP32 issue, not by HBM. Design:
//   * one CTA of 128 threads per (row b, head h, dim tile of RT rows); a thread owns
//     E = min(N, 32) state columns of one row, LPR = N / E lanes share a row;
//   * tokens are staged in chunks of kChunk: B and C (widened to fp32), x of the tile's
//     rows, dt_eff and exp(A * dt_eff) go to shared memory once per chunk and are read as
//     broadcast float4s by every row of the CTA;
//   * per-token outputs are collected in shared memory and written per chunk with the
//     D skip term and the silu(z) gate applied in the same pass;
//   * the stash is written in the staging pass (B by one CTA per group, dA/dt by one CTA
//     per head, U by every CTA for its rows).
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kPrefillThreads = 128;
constexpr int kChunk = 16;

template <typename S, int N>
__global__ void __launch_bounds__(kPrefillThreads)
ssu_prefill_kernel(const PrefillArgs pa)
{
    constexpr int E = N < 32 ? N : 32;        // state columns per thread
    constexpr int LPR = N / E;                // lanes per row
    constexpr int RT = kPrefillThreads / LPR; // rows per CTA
    constexpr int Q = E / 4;                  // quads of columns per thread

    __shared__ __align__(16) float sB[kChunk][N];
    __shared__ __align__(16) float sC[kChunk][N];
    __shared__ float sx[kChunk][RT];
    __shared__ float sy[kChunk][RT];
    __shared__ float sdA[kChunk], sdt[kChunk];

    const DecodeArgs &a = pa.d;
    const int H = a.H, Dm = a.Dm, T = pa.T, G = a.G;
    const int dtiles = (Dm + RT - 1) / RT;
    int unit = blockIdx.x;
    const int dtile = unit % dtiles;
    unit /= dtiles;
    const int h = unit % H;
    const int b = unit / H;
    const int tid = threadIdx.x;
    const int ln = tid % LPR, rloc = tid / LPR;
    const int r = dtile * RT + rloc;
    const bool reporter = tid == 0 && dtile == 0 && h == 0;

    const int slot = a.idx ? a.idx[b] : b;
    if (slot < 0) {                    // padding row: zero outputs at every position
        for (int i = tid; i < T * RT; i += kPrefillThreads) {
            const int t = i / RT, row = dtile * RT + i % RT;
            if (row < Dm)
                st_f32(a.out, a.x_dtype, (((int64_t)b * T + t) * H + h) * Dm + row, 0.f);
        }
        return;
    }
    if (slot >= a.P) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
        return;
    }
    int L = pa.ctx ? pa.ctx[b] : T;
    if (L > T) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_CONTEXT_RANGE);
        L = T;
    }
    if (L < 0) {
        if (reporter && a.err)
            atomicOr(a.err, SSU_FLAG_NEGATIVE_LENGTH);
        L = 0;
    }
    if (L == 0)
        return;

    const bool stash = pa.st_dA != nullptr;
    const int hpg = H / G;
    const int g = h / hpg;
    const bool write_group = stash && dtile == 0 && h % hpg == 0;
    const bool write_head = stash && dtile == 0;
    const float Dh = a.D ? a.D[h] : 0.f;
    const float Ah = a.A[h];

    // ---- state of this thread's row into registers
    S *base = static_cast<S *>(a.state) + (int64_t)slot * a.slot_stride + (int64_t)h * Dm * N;
    float st[E];
    if (r < Dm) {
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const float4 v = Quad<S>::load(base + (int64_t)r * N + (q * LPR + ln) * 4);
            st[4 * q] = v.x;
            st[4 * q + 1] = v.y;
            st[4 * q + 2] = v.z;
            st[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < E; ++j)
            st[j] = 0.f;
    }

    for (int t0 = 0; t0 < L; t0 += kChunk) {
        const int nt = min(kChunk, L - t0);
        __syncthreads();                 // previous chunk fully consumed
        // ---- stage the chunk
        if (tid < nt) {
            const int64_t bth = ((int64_t)b * T + t0 + tid) * H + h;
            const float dte = effective_dt(a.dt[bth], a.dt_bias, h, a.softplus);
            const float dA = expf(Ah * dte);
            sdt[tid] = dte;
            sdA[tid] = dA;
            if (write_head) {
                pa.st_dA[bth] = dA;
                pa.st_dt[bth] = dte;
            }
        }
        for (int i = tid; i < nt * N; i += kPrefillThreads) {
            const int tt = i / N, n = i % N;
            const int64_t off = (((int64_t)b * T + t0 + tt) * G + g) * N + n;
            const float bv = ld_f32(a.B, a.bc_dtype, off);
            sB[tt][n] = bv;
            sC[tt][n] = ld_f32(a.C, a.bc_dtype, off);
            if (write_group)
                pa.st_B[off] = bv;
        }
        for (int i = tid; i < nt * RT; i += kPrefillThreads) {
            const int tt = i / RT, rr = i % RT, row = dtile * RT + rr;
            float xv = 0.f;
            if (row < Dm) {
                const int64_t xi = (((int64_t)b * T + t0 + tt) * H + h) * Dm + row;
                xv = ld_f32(a.x, a.x_dtype, xi);
                if (stash)
                    pa.st_U[xi] = xv;
            }
            sx[tt][rr] = xv;
        }
        __syncthreads();
        // ---- the recurrence, token by token, state in registers
        for (int tt = 0; tt < nt; ++tt) {
            const float dA = sdA[tt];
            const float dtx = sdt[tt] * sx[tt][rloc];
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const int n = (q * LPR + ln) * 4;
                const float4 bq = *reinterpret_cast<const float4 *>(&sB[tt][n]);
                const float4 cq = *reinterpret_cast<const float4 *>(&sC[tt][n]);
                st[4 * q] = fmaf(st[4 * q], dA, bq.x * dtx);
                st[4 * q + 1] = fmaf(st[4 * q + 1], dA, bq.y * dtx);
                st[4 * q + 2] = fmaf(st[4 * q + 2], dA, bq.z * dtx);
                st[4 * q + 3] = fmaf(st[4 * q + 3], dA, bq.w * dtx);
                acc = fmaf(st[4 * q], cq.x, acc);
                acc = fmaf(st[4 * q + 1], cq.y, acc);
                acc = fmaf(st[4 * q + 2], cq.z, acc);
                acc = fmaf(st[4 * q + 3], cq.w, acc);
            }
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1)
                acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (ln == 0)
                sy[tt][rloc] = acc;
        }
        __syncthreads();
        // ---- outputs of the chunk: skip term and gate, coalesced along dim
        for (int i = tid; i < nt * RT; i += kPrefillThreads) {
            const int tt = i / RT, rr = i % RT, row = dtile * RT + rr;
            if (row < Dm) {
                const int64_t xi = (((int64_t)b * T + t0 + tt) * H + h) * Dm + row;
                float y = sy[tt][rr] + Dh * sx[tt][rr];
                if (a.z)
                    y *= silu_f(ld_f32(a.z, a.x_dtype, xi));
                st_f32(a.out, a.x_dtype, xi, y);
            }
        }
    }

    // ---- final state, once (the stash mode leaves the committed state read-only)
    if (!stash && r < Dm) {
#pragma unroll
        for (int q = 0; q < Q; ++q)
            Quad<S>::store(base + (int64_t)r * N + (q * LPR + ln) * 4,
                           make_float4(st[4 * q], st[4 * q + 1], st[4 * q + 2], st[4 * q + 3]));
    }
}

template <typename S, int N>
int launch_n(const PrefillArgs &a, cudaStream_t s)
{
    constexpr int E = N < 32 ? N : 32;
    constexpr int RT = kPrefillThreads / (N / E);
    const int64_t dtiles = (a.d.Dm + RT - 1) / RT;
    const int64_t grid = (int64_t)a.d.active * a.d.H * dtiles;
    if (grid == 0 || a.T == 0)
        return SSU_OK;
    if (grid > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    ssu_prefill_kernel<S, N><<<(unsigned)grid, kPrefillThreads, 0, s>>>(a);
    return SSU_OK;
}

template <typename S>
int launch_s(const PrefillArgs &a, cudaStream_t s)
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

int launch_prefill(const PrefillArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
